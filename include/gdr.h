/*
 * gdr.h -- C ABI of libgdr.so: the key-axis-gated delta-rule recurrence on B200.
 *
 * The operation (one head of one sequence, tokens t = 1..T, state S_t in R^{dv x dk}):
 *
 *     S_t = S_{t-1} D_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,     o_t = S_t (scale * q_t)
 *
 *   - "Semidirect Fourier Delta Attention" page, section "Core architecture":
 *     the state is decayed, then erased along k_t, then written with
 *     beta_t k_t v_t^*.  The page's state is dk x dv and is acted on from the left;
 *     this library stores its transpose (value rows, key columns), as the
 *     "CARVE" page does in section 1.
 *   - "CARVE" page, section 2.3: the decay is a key-axis exponential gate,
 *     D_t = diag(exp(g_t)), g_t <= 0 (rotation off).
 *   - "Semidirect Fourier Delta Attention" page, "Core architecture", real
 *     implementation: with rotation on, D_t is a direct sum of 2x2 rotation-decay
 *     blocks.  Key pair j = (2j, 2j+1) of every row of S, read as x + i y, is
 *     multiplied by alpha_{t,j} e^{i theta_{t,j}}, alpha = exp(g_{t,j}).  That is
 *     the transpose of the page's Lambda_t = diag(alpha_t e^{i theta_t}).
 *   - The readout uses the post-update state S_t.
 *
 * Gate activation (fused in the kernels; "CARVE" page, section 2.3, gate in
 * kernel): GDR_GATE_LOGDECAY reads g itself; GDR_GATE_NEG_SOFTPLUS reads a raw
 * gate a and uses g = -softplus(a) = log sigmoid(-a).
 *
 * Common conventions
 *   - Every pointer is a DEVICE pointer unless stated otherwise.  The caller owns
 *     all buffers and the stream.  The library allocates no memory.
 *   - All calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream).  Argument checks are synchronous and
 *     return before anything is launched.
 *   - Layouts are dense row-major, last index fastest.  Every pointer must be
 *     16-byte aligned.
 *   - Element types: q, k, v use `qkv_dtype`; o uses `out_dtype`; g, beta, theta,
 *     S0, S_T and the decode state S are always fp32.
 *   - Errors: GDR_ERR_INVALID_ARG / GDR_ERR_UNSUPPORTED mean nothing was
 *     launched.  GDR_ERR_CUDA means a launch failed (see gdr_last_error_detail).
 *     No call aborts or throws.
 */
#ifndef GDR_H
#define GDR_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDR_ABI_VERSION 5

#if defined(__GNUC__)
#define GDR_API __attribute__((visibility("default")))
#else
#define GDR_API
#endif

typedef void* gdr_stream_t; /* a cudaStream_t */

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or enum; nothing launched */
    GDR_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. dk not in {32,64,128}) */
    GDR_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    GDR_ERR_TIMEOUT = 4,     /* a kernel gave up on a bounded wait (device status word) */
    GDR_ERR_WORKSPACE = 5,   /* workspace pointer NULL or smaller than required */
    GDR_ERR_RANGE = 6,       /* a decay factor left the factored range (device status word) */
    GDR_ERR_BOUNDS = 7       /* an index check of the debug build failed (device status word) */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

typedef enum { GDR_GATE_LOGDECAY = 0, GDR_GATE_NEG_SOFTPLUS = 1 } gdr_gate_mode;

typedef enum {
    GDR_ALGO_AUTO = 0,    /* for bf16 q/k/v and dk = dv = 128: the fused kernel for a single
                             chunk; the sequence-parallel form (GDR_ALGO_TCGEN05_SEGMENTS) when a
                             few heads have long sequences, so that one chain per head would be
                             the bound; else the split kernel when 2*B*H <= SM count, the waves
                             mix when B*H exceeds the SM count and its remainder would take the
                             split kernel, the fused kernel otherwise.  The CUDA-core kernel for
                             every other shape and for fp32 mode */
    GDR_ALGO_SIMT = 1,    /* fp32 CUDA-core chunk-WY kernel (every supported shape) */
    GDR_ALGO_TCGEN05 = 2, /* tcgen05/TMEM chunk-WY kernel, one CTA per (batch, head):
                             bf16 q/k/v, dk = dv = 128 */
    GDR_ALGO_TCGEN05_SPLIT = 3 /* same method; one CTA per head runs only the state chain
                             while every other SM prepares chunks (two at a time), handed
                             over through a ring in the workspace (needs B*H < SM count;
                             cooperative launch); results agree with GDR_ALGO_TCGEN05 to
                             rounding */,
    GDR_ALGO_TCGEN05_WAVES = 4 /* more heads than SMs: the fused kernel for whole waves of
                             SM-count heads, then the split kernel for the last partial wave
                             when it is at most half the SM count (else fused throughout);
                             workspace for the split part */,
    GDR_ALGO_TCGEN05_SEGMENTS = 5 /* sequence-parallel: each head's sequence is cut into
                             desc->segments segments (0: chosen by the library) that run as
                             separate chains, from the zero state and from the identity; an
                             affine scan over the segments and an output correction combine
                             them (see gdr_chunk_fwd) */,
    GDR_ALGO_TCGEN05_CHAINS = 6 /* the chain kernel the segments run on, for any number of
                             heads: a cooperative grid of one CTA per SM, nc of them state chains
                             (heads in waves of nc, one after another, nc from a cost model) and
                             every other SM a prep worker whose elementwise and solve warp groups
                             work on consecutive chunks; T > 64 */
} gdr_algo;

/* Shape and mode of one chunked forward call. */
typedef struct {
    int B, H, T;          /* batch, heads, tokens (T >= 0; T = 0 only copies S0 to S_T) */
    int dk, dv;           /* key / value head dims, each in {32, 64, 128} */
    int chunk;            /* chunk length; must be 64 */
    gdr_dtype qkv_dtype;  /* storage of q, k, v */
    gdr_dtype out_dtype;  /* storage of o */
    gdr_gate_mode gate_mode;
    int rotation;         /* 0: real key-axis decay; 1: 2x2 rotation-decay blocks */
    float scale;          /* multiplies q (1.0 for none) */
    gdr_algo algo;
    int qk_l2norm;        /* 1: the kernels L2-normalise q_t and k_t per token and head first,
                             x / sqrt(sum x^2 + 1e-6) in fp32, before the scale (0: as given) */
    int segments;         /* GDR_ALGO_TCGEN05_SEGMENTS: number of segments per sequence (>= 2; 0
                             lets the library choose); ignored by the other algorithms */
} gdr_fwd_desc;

/* Shape and mode of one decode step over N independent sequences. */
typedef struct {
    int N, H;             /* sequences, heads */
    int dk, dv;           /* each in {32, 64, 128} */
    gdr_dtype qkv_dtype, out_dtype;
    gdr_gate_mode gate_mode;
    int rotation;
    float scale;
    int qk_l2norm;        /* as in gdr_fwd_desc */
} gdr_dec_desc;

/* GDR_ABI_VERSION of the loaded library. */
GDR_API int gdr_abi_version(void);

/* Static, NUL-terminated name of a status code. */
GDR_API const char* gdr_status_string(gdr_status s);

/* Detail of the last GDR_ERR_* returned on the calling host thread (static
 * thread-local string; empty when there is none). */
GDR_API const char* gdr_last_error_detail(void);

/* Bytes of device workspace gdr_chunk_fwd needs for this descriptor (0 = none;
 * the workspace argument may then be NULL).  Returns 0 for an invalid desc.  The split
 * tensor-core kernel needs, for each of its nc state chains (1 <= nc <= min(B*H, SMs / 2),
 * chosen from B*H, T and the SM count), a ring of 8 slots of 91,136 bytes plus 36 bytes of
 * flags, and one 4-byte task counter; it resets the flags itself (on the call's stream) and
 * the buffer may be reused by later calls on the same stream.  Uses the current device's
 * SM count. */
GDR_API size_t gdr_chunk_fwd_workspace_bytes(const gdr_fwd_desc* desc);

/*
 * Chunk-parallel forward over whole sequences (chunk-WY / UT-transform solver).
 *
 * Source: the WY-form triangular chunk solver that batches a chunk's tokens into
 * one linear system ("CARVE" page, section 1 item 3, section 3 item 1), in the
 * constructive form of the "Semidirect Fourier Delta Attention" page (section
 * "Constructive Chunk-WY Theorem": the in-chunk correction has rank <= chunk;
 * section "Main contributions": exact affine chunk transfer of the state).
 *
 *   q, k  [B,T,H,dk]  qkv_dtype          v  [B,T,H,dv]  qkv_dtype
 *   g     [B,T,H,dk]  fp32 (rotation: [B,T,H,dk/2], one decay per key pair)
 *   beta  [B,T,H]     fp32, the write strength (0 <= beta <= 1 expected)
 *   theta [B,T,H,dk/2] fp32 angles; must be NULL unless rotation
 *   S0    [B,H,dv,dk] fp32 initial state, or NULL for zeros
 *   o     [B,T,H,dv]  out_dtype (written)
 *   S_T   [B,H,dv,dk] fp32 final state, or NULL to skip (may alias S0)
 *   workspace / workspace_bytes: see gdr_chunk_fwd_workspace_bytes.
 *
 * Numerical range: the kernels factor exp(Gamma_r - Gamma_i) through per-chunk
 * reference points; a key dim whose log-decay over 32 consecutive tokens is
 * below -80 may overflow the factored form (tensor-core kernels; reported as
 * GDR_ERR_RANGE by gdr_query_device_status).
 *
 * GDR_ALGO_TCGEN05_SEGMENTS (sequence parallelism; "Semidirect Fourier Delta Attention"
 * page, "Main contributions": the exact affine transfer S_end = S_start A + B): each
 * sequence is cut into segments of a whole number of chunks (the last one may be shorter).
 * Every segment runs from the zero state (segment 0 from S0), giving o0 and its end state
 * B, and segments 1.. also from the identity with zero values, giving y_t = A q_t and the
 * transition A; a scan over the segments forms their true start states St (fp32) and S_T,
 * and o_t = o0_t + St y_t (tf32 products) for t in segments 1..  The workspace
 * (gdr_chunk_fwd_workspace_bytes) then also holds the per-segment states and y (4 bytes per
 * token, head and key dim) and must be 256-byte aligned.
 */
GDR_API gdr_status gdr_chunk_fwd(const gdr_fwd_desc* desc,
                         const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const float* theta,
                         const float* S0, void* o, float* S_T,
                         void* workspace, size_t workspace_bytes,
                         gdr_stream_t stream);

/*
 * One recurrent decode step: the token update above applied once to each of
 * N*H states, in place.  Reads and writes S exactly once.
 *
 *   q, k [N,H,dk] qkv_dtype;  v [N,H,dv] qkv_dtype;  g [N,H,dk] (rotation: [N,H,dk/2]);
 *   beta [N,H];  theta [N,H,dk/2] or NULL;  S [N,H,dv,dk] fp32, in/out;  o [N,H,dv] out_dtype.
 */
GDR_API gdr_status gdr_decode_step(const gdr_dec_desc* desc,
                           const void* q, const void* k, const void* v,
                           const float* g, const float* beta, const float* theta,
                           float* S, void* o, gdr_stream_t stream);

/*
 * Separate erase and write strengths ("CARVE" page, sections 2.1-2.2: an erase gate and a
 * scalar value write gate per head and token).  The token update becomes
 *
 *   S_t = S_{t-1} D_t (I - beta_t k_t k_t^T) + w_t v_t k_t^T,     o_t = S_t (scale q_t)
 *
 * with beta the erase strength and w [B,T,H] (decode: [N,H]) fp32 the write strength,
 * 16-byte aligned.  w = NULL is the tied rule above (w = beta): gdr_chunk_fwd and
 * gdr_decode_step are these calls with w = NULL.  Every kernel supports it; the chunk solver
 * is unchanged (A still uses beta), only U = (I + A)^{-1} diag(w) V changes.  The
 * content-aware erase of that page (beta modulated by the previous chunk's mean output)
 * is left to the caller, which passes the resulting beta; gdr_chunk_fwd_ex below also
 * returns the chunk means it needs.  Other arguments, layouts, errors
 * and ownership as for gdr_chunk_fwd / gdr_decode_step.  (gdr_chunk_fwd_noalloc is tied only.)
 */
GDR_API gdr_status gdr_chunk_fwd_untied(const gdr_fwd_desc* desc,
                                        const void* q, const void* k, const void* v,
                                        const float* g, const float* beta, const float* w,
                                        const float* theta, const float* S0, void* o, float* S_T,
                                        void* workspace, size_t workspace_bytes,
                                        gdr_stream_t stream);
GDR_API gdr_status gdr_decode_step_untied(const gdr_dec_desc* desc,
                                          const void* q, const void* k, const void* v,
                                          const float* g, const float* beta, const float* w,
                                          const float* theta, float* S, void* o,
                                          gdr_stream_t stream);

/*
 * gdr_chunk_fwd_untied with one more output: the mean of o over each chunk, the content
 * signal of the content-aware erase ("CARVE" page, section 2.1: the chunk mean of the
 * outputs the kernel already writes, fed through a zero-initialised low-rank projection
 * into the next chunk's erase gate).
 *
 *   chunk_mean[b, c, h, :] = (1 / L_c) * sum over tokens t of chunk c of o[b, t, h, :]
 *
 * with chunks of desc->chunk (64) tokens and L_c the number of tokens of chunk c inside T
 * (the last chunk may be shorter).  chunk_mean is fp32 [B, ceil(T/64), H, dv], 16-byte
 * aligned, written whole; NULL = not computed (this call is then gdr_chunk_fwd_untied).  The
 * kernels sum the fp32 outputs before rounding them to the output dtype, in the epilogue that
 * writes o, so the only extra HBM traffic is the write of chunk_mean itself.  The projection
 * and the gate (beta for chunk c + 1 from chunk_mean of chunk c) belong to the layer that
 * produces beta.  Every kernel supports it.  Other arguments, layouts, errors and ownership
 * as for gdr_chunk_fwd_untied.
 */
GDR_API gdr_status gdr_chunk_fwd_ex(const gdr_fwd_desc* desc,
                                    const void* q, const void* k, const void* v,
                                    const float* g, const float* beta, const float* w,
                                    const float* theta, const float* S0, void* o, float* S_T,
                                    float* chunk_mean, void* workspace, size_t workspace_bytes,
                                    gdr_stream_t stream);

/*
 * gdr_chunk_fwd_ex on HOST buffers: q, k, v, g, beta, w, theta and S0 are read from host
 * memory and o, S_T and chunk_mean are written to host memory; only the workspace is device
 * memory.  Same arguments, layouts and results as gdr_chunk_fwd_ex (NULL = absent for w,
 * theta, S0, S_T, chunk_mean), computed slice by slice over the batch: the B entries are cut
 * into at most 8 slices of equal size (the last may be smaller), and each slice is one
 * gdr_chunk_fwd_ex call with B = its entry count, so its kernel is the one AUTO (or
 * desc->algo) picks for that B.
 *
 * Slice i's inputs are copied into device slot i % 2 on a copy stream of the library's, its
 * forward runs on `stream`, and its outputs are copied back on a second copy stream, so the
 * host-to-device copies, the device-to-host copies and the kernels of neighbouring slices
 * overlap.  The copies run asynchronously (and overlap) only from page-locked host memory
 * (cudaHostAlloc / cudaHostRegister); pageable buffers work but each copy then blocks the
 * host thread.
 *
 * Ordering: the copies start after the work already queued on `stream`, and `stream` is
 * complete only once every output is in host memory (synchronise it, or an event recorded
 * on it, before reading o).  Host buffers must stay valid and unchanged until then.  The
 * library's copy streams and events are created on a device's first call and kept until
 * the process exits; calls from several host threads are enqueued one at a time.
 *
 * workspace: device memory of at least gdr_chunk_fwd_host_workspace_bytes(desc, ...) bytes,
 * 16-byte aligned, given the same presence flags (non-zero when that argument is not NULL),
 * else GDR_ERR_WORKSPACE.  It holds the split kernel's ring (if any) and two slots of
 * per-slice inputs and outputs; like the ring it may be reused by later calls on the same
 * stream.  Errors: as gdr_chunk_fwd_ex; GDR_ERR_CUDA if a copy cannot be queued (the outputs
 * are then undefined, and `stream` still waits for the copies already queued, so host buffers
 * may be released once it has completed).
 */
GDR_API size_t gdr_chunk_fwd_host_workspace_bytes(const gdr_fwd_desc* desc, int with_w, int with_S0,
                                                  int with_S_T, int with_chunk_mean);
GDR_API gdr_status gdr_chunk_fwd_host(const gdr_fwd_desc* desc,
                                      const void* q, const void* k, const void* v,
                                      const float* g, const float* beta, const float* w,
                                      const float* theta, const float* S0, void* o, float* S_T,
                                      float* chunk_mean, void* workspace, size_t workspace_bytes,
                                      gdr_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word that
 * kernels set when a bounded wait gives up (GDR_ERR_TIMEOUT) or when the tensor-core
 * kernel meets a decay outside its factored range (GDR_ERR_RANGE; the outputs of that
 * call are not valid).  Returns GDR_OK, GDR_ERR_TIMEOUT, GDR_ERR_RANGE or GDR_ERR_CUDA
 * (a sticky CUDA error on the context).  Uses the current device.
 */
GDR_API gdr_status gdr_query_device_status(gdr_stream_t stream);

/*
 * gdr_chunk_fwd without a workspace argument: the library allocates nothing, ever.
 *
 * The pages have no counterpart to this call; it serves callers that cannot hand the
 * library device memory.  Examples: plain-C hosts whose own memory manager owns all of
 * the GPU's memory and forbids further cudaMalloc, and serving loops that must not
 * call cudaMalloc or cudaFree on their latency path, because those calls can
 * synchronise the device.
 *
 * It runs the split tensor-core kernel (same arithmetic and results as
 * gdr_chunk_fwd with GDR_ALGO_TCGEN05_SPLIT) with the kernel's hand-off ring in a scratch
 * array compiled into the library: at most GDR_NOALLOC_MAX_HEADS rings of 8 slots of 91,136
 * bytes plus flags (about 22.3 MiB), which every GPU that loads the library holds until the
 * process exits.
 *   - desc->algo must be GDR_ALGO_AUTO or GDR_ALGO_TCGEN05_SPLIT; q, k, v must be bf16 with
 *     dk = dv = 128; B*H must not exceed GDR_NOALLOC_MAX_HEADS, else GDR_ERR_UNSUPPORTED with
 *     a message (nothing launched).  Other arguments as for gdr_chunk_fwd.
 *   - The first call on each device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it with the context's id;
 *     a context destroyed and created again (cudaDeviceReset) is seen by its new id and the
 *     address is looked up again.  Make the first call in each context before any stream
 *     capture.
 *   - Every call shares the one scratch array, which keeps the last call's contents; each
 *     call clears the flags it needs on its own stream first.  Calls that overlap on the
 *     GPU (other streams, other host threads) race on the array and must be serialised by
 *     the caller.
 */
#define GDR_NOALLOC_MAX_HEADS 32
GDR_API gdr_status gdr_chunk_fwd_noalloc(const gdr_fwd_desc* desc,
                                         const void* q, const void* k, const void* v,
                                         const float* g, const float* beta, const float* theta,
                                         const float* S0, void* o, float* S_T,
                                         gdr_stream_t stream);

/* The gdr_algo a descriptor would run with (GDR_ALGO_AUTO resolved), or -1 if the
 * descriptor is invalid.  No GPU work. */
GDR_API int gdr_chunk_fwd_algo(const gdr_fwd_desc* desc);

/* The number of kernels one forward call with this descriptor launches on the stream
 * (the zeroing of the split kernel's flags by cudaMemsetAsync not counted): 1 for the
 * SIMT, fused and split kernels, 2 for TCGEN05_WAVES with a partial last wave, 4 for
 * TCGEN05_SEGMENTS with more than one segment (two split passes, the scan and the
 * correction), 0 when B or H is 0; a call with T = 0 counts 1 (it writes S_T).  -1 if
 * the descriptor is invalid.  No GPU work (the segment plan reads the device's SM
 * count). */
GDR_API int gdr_chunk_fwd_kernel_launches(const gdr_fwd_desc* desc);

/*
 * Backward pass of gdr_chunk_fwd: the gradients of a loss L with respect to every input, given
 * dO = dL/do and dS_T = dL/dS_T (the training use that the "CARVE" page, section 4, measures).
 * It follows the chain rule through the chunk-WY algebra ("CARVE" page, section 1 item 3;
 * "Semidirect Fourier Delta Attention" page, "Constructive Chunk-WY Theorem" and the exact
 * affine chunk transfer) in three launches: every chunk's transfer coefficients in parallel
 * (S_L = S0 A_c + B_c and dS0 = G_c + dS_L A_c^T need no state), one short chain per (batch,
 * head) for the chunk start states and the end-state gradients (on tcgen05 at d = 128), then
 * every chunk's gradients in parallel.  fp32 throughout (tensor-core products with split-tf32 operands).  With rotation
 * ("Semidirect Fourier Delta Attention" page, "Core architecture", 2x2 rotation-decay blocks) the
 * key pairs are complex numbers and the adjoints of the complex decay products are their
 * conjugates; with qk_l2norm the gradients of q and k are taken through the normalisation
 * x / sqrt(sum x^2 + 1e-6).
 *
 *   desc            as for gdr_chunk_fwd; dk = dv (32, 64 or 128), else GDR_ERR_UNSUPPORTED;
 *                   rotation, qk_l2norm, gate_mode and scale as in the forward; algo and
 *                   segments are ignored.  dO has the dtype desc->out_dtype; q, k, v
 *                   desc->qkv_dtype.
 *   q, k, v, g, beta, w, theta, S0   the forward's inputs, layouts as in gdr_chunk_fwd (w may be
 *                   NULL: w = beta; theta [B,T,H,dk/2] exactly with rotation; S0 may be NULL:
 *                   zero).
 *   dO [B,T,H,dv]   gradient of o, or NULL (zero).
 *   dS_T [B,H,dv,dk] fp32 gradient of the final state, or NULL (zero).
 *   dq, dk [B,T,H,dk], dv [B,T,H,dv], dg [B,T,H,dk] (rotation: [B,T,H,dk/2]; of the gate input
 *                   as given: g itself with GDR_GATE_LOGDECAY, the raw gate a with
 *                   GDR_GATE_NEG_SOFTPLUS), dbeta [B,T,H]: fp32 outputs, required when T > 0.
 *   dw [B,T,H]      fp32, required exactly when w is given (then dbeta is the erase strength's
 *                   gradient alone).
 *   dtheta [B,T,H,dk/2]  fp32, required exactly with rotation (when T > 0).
 *   dS0 [B,H,dv,dk] fp32 gradient of S0, or NULL (not written).
 *   workspace       device memory of gdr_chunk_bwd_workspace_bytes(desc) bytes, 16-byte aligned
 *                   (five dk x dv fp32 matrices per chunk and about 1 MB of chunk matrices per
 *                   SM at d = 128: 1.47 GB at B=4, H=16, T=4096).
 * All pointers are device pointers, 16-byte aligned, owned by the caller; the call is
 * asynchronous on `stream` and allocates nothing.  With T = 0, dS0 = dS_T.  Errors: argument
 * checks return before any launch; a decay too strong for the factored form over half a chunk
 * (a factor above 3e38) sets the device status word's range bit (gdr_query_device_status ->
 * GDR_ERR_RANGE).
 */
GDR_API size_t gdr_chunk_bwd_workspace_bytes(const gdr_fwd_desc* desc);
GDR_API gdr_status gdr_chunk_bwd(const gdr_fwd_desc* desc,
                                 const void* q, const void* k, const void* v,
                                 const float* g, const float* beta, const float* w,
                                 const float* theta, const float* S0, const void* dO,
                                 const float* dS_T, float* dq, float* dk, float* dv, float* dg,
                                 float* dbeta, float* dw, float* dtheta, float* dS0,
                                 void* workspace, size_t workspace_bytes, gdr_stream_t stream);

/*
 * Raven's routed slot memory ("Raven: High-Recall Sequence Modeling with Sparse Memory Routing"
 * page, section 2.1, routing slot memories, and section 2.2, the Raven architecture): per
 * (batch, head) a key state Sk and a value state Sv of M = 64 slots (rows) of d values.  Token t:
 *   - the router keeps the top K of the logits z_t (ties to the lower slot index), takes the
 *     sigmoid m of the kept ones and normalises them, r_t[i] = m_i / sum of the kept m (zero on the
 *     other slots); the logits are an input (the projection W x_t belongs to the layer);
 *   - only the chosen slots decay and are written: with a_t the log-decay of the gate g_t
 *     (g itself for GDR_GATE_LOGDECAY, -softplus(g) for GDR_GATE_NEG_SOFTPLUS),
 *     S[i] <- e^{a_t r_t[i]} S[i] + (1 - e^{a_t r_t[i]}) x_t, x = k_t for Sk and v_t for Sv;
 *     an unchosen slot (r = 0) stays as it is;
 *   - the readout is softmax attention over the slots of the updated states,
 *     o_t = sum_i softmax_i(scale q_t . Sk[i]) Sv[i] (with a one-hot router that cycles through
 *     the slots and a decay that empties the chosen slot, exactly sliding-window attention over
 *     the last M tokens, the special case the page's section 2.1 names).
 * The library runs it in chunks of 32 tokens (per-slot cumulative decays, bf16 tensor-core
 * products, the chunk's writes as sums over the tokens that chose each slot, fp32 states), and
 * splits long sequences into segments whose start states it composes from the earlier segments'
 * end states (the chunk transition is diagonal in the slots).
 */
typedef struct {
    int B, H, T;          /* batch, heads, tokens (T >= 0) */
    int d;                /* head dim of q, k, v and the slot states: 64 or 128 */
    int slots;            /* M: must be 64 */
    int topk;             /* K: 1 .. 16 */
    gdr_dtype qkv_dtype;  /* must be GDR_BF16 */
    gdr_dtype out_dtype;  /* GDR_BF16 or GDR_F32 */
    gdr_gate_mode gate_mode;
    float scale;          /* multiplies q . Sk[i] inside the softmax */
    int segments;         /* 0: the library chooses; n >= 1: n segments per sequence (at most one
                             per 32-token chunk) */
} gdr_raven_desc;

/* Segments per sequence a descriptor runs with, or -1 if it is invalid.  No GPU work. */
GDR_API int gdr_raven_fwd_segments(const gdr_raven_desc* desc);
/* Device workspace for gdr_raven_fwd: every token's routing record (B*T*H * 144 bytes, rounded up
 * to 256), then (B*H) * units * (2*64*d + 64) floats, where the units are the pieces (a divisor of
 * the segment length, at least 4 chunks of 32 tokens, short enough for about two waves of CTAs)
 * of the chunks before the last segment whose end states the state pass computes; 0 when
 * B, H or T is 0, or for an invalid descriptor. */
GDR_API size_t gdr_raven_fwd_workspace_bytes(const gdr_raven_desc* desc);
/*
 *   q, k, v [B,T,H,d] bf16;  z [B,T,H,64] fp32 router logits (finite or -inf);  g [B,T,H] fp32;
 *   S0k, S0v [B,H,64,d] fp32 initial states or NULL (zero);  o [B,T,H,d] out_dtype;
 *   Sk_T, Sv_T [B,H,64,d] fp32 final states or NULL (not written).
 * All device pointers, 16-byte aligned, owned by the caller; asynchronous on `stream`; nothing
 * is allocated.  Errors: GDR_ERR_INVALID_ARG / GDR_ERR_UNSUPPORTED / GDR_ERR_WORKSPACE before any
 * launch.  Two launches with one segment (the router for every token, then the outputs), three
 * otherwise (the router, the state units, the outputs).
 */
GDR_API gdr_status gdr_raven_fwd(const gdr_raven_desc* desc, const void* q, const void* k, const void* v,
                                 const float* z, const float* g, const float* S0k, const float* S0v,
                                 void* o, float* Sk_T, float* Sv_T, void* workspace,
                                 size_t workspace_bytes, gdr_stream_t stream);

/*
 * Test hook for the bounded waits of the tensor-core kernel (process-wide, not
 * thread-safe).  wait_limit_ns bounds every mbarrier wait (0 restores the 2 s
 * default).  With skip_first_commit != 0, each later launch never signals its first
 * MMA completion: the wait gives up after wait_limit_ns, the kernel frees its tensor
 * memory and returns, and gdr_query_device_status reports GDR_ERR_TIMEOUT.  Outputs of
 * such a launch are not valid.  Nothing faults or traps.
 */
/* Debug build (libgdr_debug.so, compiled with -DGDR_BOUNDS_CHECK): every kernel tests the
 * index of each global-memory access that it computes (ring slots and flags, outputs, the
 * states, beta) before making it; a failing test skips the access, records its site number and
 * sets the status word's bounds bit (gdr_query_device_status -> GDR_ERR_BOUNDS).  Returns and
 * clears the first failing site (0: none), or -1 in the default build, which has no checks. */
GDR_API int gdr_debug_bounds_site(void);

GDR_API void gdr_debug_set_tc_fault(int skip_first_commit, unsigned long long wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H */
