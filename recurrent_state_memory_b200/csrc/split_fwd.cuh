// split_fwd.cuh -- chunk-WY forward with the chunk preparation and the state chains on
// separate SMs (tcgen05 + TMEM, bf16 operands, fp32 accumulation, dk = dv = 128, chunk 64).
//
// The WY/UT-transform triangular chunk solver ("CARVE" page, section 1 item 3 and section 3
// item 1; "Semidirect Fourier Delta Attention" page, "Constructive Chunk-WY Theorem" and the
// exact affine chunk transfer).  Per chunk, with P_r = D_1 ... D_r and the reference token
// m = 31, every decay factor is split around P_m so that none exceeds the decay of half a chunk:
//   Ktil_r = (P_m^{-1} P_r) k_r,  Qtil_r = (P_m^{-1} P_r) q_r,  Khat_i = (P_i^{-1} P_m)^T k_i
//   [A' ; Pm] = [Ktil ; Qtil] Khat^T,  T = (I + diag(beta) strict_lower(A'))^{-1}
//   Tb = T diag(beta), Tw = T diag(w),  Wm^T = Ktil^T Tb^T                    (prep worker)
//   U^T = V^T Tw^T,  E^T = U^T - Stil Wm^T,  S_acc = Stil + E^T Khat,
//   O^T = Stil Qtil^T + E^T masked(Pm)^T,  S_next = S_acc (P_m^{-1} P_C)      (state chain)
// where Stil = S P_m is the state at the chunk start prescaled by the reference decay.
//
// Grid: one CTA per SM, all resident (cooperative launch).  CTAs [0, nc) are state chains,
// the others prep workers.  Heads are processed in waves of nc: chain j runs heads
// j, j + nc, j + 2 nc, ... one after another, so any number of heads fits.  A worker task is
// one 64-token chunk of one head; tasks are numbered wave by wave, chunk-major within a wave,
// and claimed in increasing order (from a global counter, or at a fixed stride).  A worker
// writes a finished chunk's operands into a ring slot of its head's chain (RING slots per
// chain, in the shared-memory layouts the chain's MMAs read) and publishes the slot with a
// release store; the chain copies the slot into shared memory, drops its lines from L2 and
// hands it back.  Every task a worker waits on has a lower number than its own, and a chain
// waits only on its own chunks in order, so no wait is circular.
//
// Prep worker (512 threads):
//   warps 0-7   elementwise: gate activation, decay products, the bf16 operand tiles of the
//               first MMA (shared memory), Qtil and Khat^T into the ring; thread 0 stages the
//               next task's inputs with tensor-map copies and issues the first MMA.
//   warps 12-15 solve: read [A' ; Pm] back from TMEM (Pm into the ring), invert the unit
//               lower-triangular 64x64 matrix, form Tb / Tw, issue Wm^T = Ktil^T Tb^T and move
//               Wm^T into the ring, then publish the slot.
//   The two groups work on consecutive tasks at once (double-buffered tiles and accumulators).
// State chain (512 threads):
//   warp 0      loader: ring slot -> shared memory (bulk copies), V tile (tensor map).
//   warp 1      MMA issuer (one thread).
//   warps 4-7   o: O^T (TMEM) -> global o (16-byte stores after in-register transposes); chunk
//               means of o.
//   warps 8-15  state: S_acc -> S_next -> next chunk's prescaled state (fp32 and bf16 copy).
//   The first state MMA leaves E^T in TMEM in fp32; the state update and the second output
//   MMA read it there directly as the tf32 A operand, so each chunk has a single round trip
//   through the threads (the rescale of the state).
// Every wait is bounded; a role that gives up sets the CTA's abort flag and the device status
// word, and the other roles give up on their own bounded waits.
#pragma once

#include <cuda.h>   // CUtensorMap

#include "common.cuh"
#include "tc_ptx.cuh"

// Optional event timeline for profiling builds (compiled with -DGDR_TIMELINE): the %globaltimer
// of selected events, per CTA and iteration, into a device array the host reads back.  The
// default build records nothing.
#ifdef GDR_TIMELINE
namespace gdr {
constexpr int TL_ITERS = 256, TL_EVENTS = 16;
__device__ unsigned long long g_timeline[148 * TL_ITERS * TL_EVENTS];
}
#define GDR_TL(on, it, ev)                                                                            \
    do {                                                                                              \
        if ((on) && (it) < ::gdr::TL_ITERS)                                                           \
            ::gdr::g_timeline[((size_t)blockIdx.x * ::gdr::TL_ITERS + (it)) * ::gdr::TL_EVENTS + (ev)] = \
                ::gdr::tc::globaltimer_ns();                                                          \
    } while (0)
#else
#define GDR_TL(on, it, ev) \
    do {                   \
    } while (0)
#endif

namespace gdr {
namespace spl {

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 512;
constexpr int RING = 8;          // ring slots per chain
constexpr int AS = 68;           // row stride (floats) of the fp32 solve matrices

// Ring slot (bytes); the chain copies it as is into a shared-memory buffer.
constexpr uint32_t SL_Q = 0;         // Qtil bf16 K-major: 2 kblocks (dk halves) x 64 rows x 128 B
constexpr uint32_t SL_W = 16384;     // Wm^T bf16 MN-major: 128 dk rows x 128 B (64 tokens)
constexpr uint32_t SL_H = 32768;     // Khat^T fp32 K-major: 2 kblocks (token halves) x 128 dk rows x 128 B
constexpr uint32_t SL_P = 65536;     // masked Pm fp32 K-major: 2 kblocks (i halves) x 64 rows x 128 B
constexpr uint32_t SL_T = 81920;     // Tw bf16 K-major (Tb when w = beta): 64 rows x 128 B
constexpr uint32_t SL_VEC = 90112;   // P_m [128] then P_m^{-1} P_C [128] fp32 (rotation: re[64], im[64] each)
constexpr uint32_t SLOT_BYTES = SL_VEC + 1024;

// Chain CTA shared memory: two slot buffers, the V tile, a ring of decay vectors, barriers.
constexpr uint32_t CH_V = 2 * SLOT_BYTES;
constexpr uint32_t CH_VEC = CH_V + 16384;    // 4 chunks' decay vectors (P_m, P_m^{-1} P_C), 1 KB each
constexpr uint32_t CH_BAR = CH_VEC + 4096;
// Worker CTA shared memory.
constexpr uint32_t IN_Q = 0, IN_K = 16384, IN_G = 32768, IN_TH = 49152;   // staged inputs (64 KB)
constexpr uint32_t WK_KQ = 65536;        // x2: [Ktil ; Qtil] K-major, 2 kblocks x 128 rows x 128 B
constexpr uint32_t WK_KH = 131072;       // Khat K-major, 2 kblocks x 64 rows x 128 B
constexpr uint32_t WK_PMS = 147456;      // masked Pm staged in its ring layout (fp32, 16 KB)
constexpr uint32_t WK_AF = 163840;       // fp32 A [64][AS]
constexpr uint32_t WK_TF = WK_AF + 64 * AS * 4;   // fp32 T [64][AS] (blocks above the diagonal: scratch);
                                                  // after the solve, Wm^T staged in its ring layout
constexpr uint32_t WK_TB = 198656;       // Tb bf16 K-major 64 rows x 128 B
constexpr uint32_t WK_TW = WK_TB + 8192; // Tw bf16
constexpr uint32_t WK_QT = WK_TW + 8192; // segment products [8 segments][32 dim groups][8]
constexpr uint32_t WK_VEC = WK_QT + 8192;   // x2: beta[64], w[64]
constexpr uint32_t WK_BAR = WK_VEC + 1024;
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM_BYTES = (WK_BAR > CH_BAR ? WK_BAR : CH_BAR) + BAR_BYTES + 1024;   // + base alignment
static_assert(WK_TF + 64 * AS * 4 <= WK_TB, "solve matrices overlap Tb");
static_assert(SMEM_BYTES <= 232448, "shared memory exceeds 227 KB");
static_assert((SLOT_BYTES & 1023) == 0, "slot buffers must stay 1024-byte aligned");

// Tensor memory.  Chain (512 columns): S fp32 | Stil bf16 x2 | E^T x2 | O^T x2.
constexpr uint32_t COL_S = 0, COL_SB = 128, COL_E = 256, COL_O = 384;
// Worker (256 columns): [A' ; Pm] x2 | Wm^T.
constexpr uint32_t COL_ACC = 0, COL_WM = 128;

// 4-D tensor maps {inner dim, H, T, B} with boxes of 64 tokens: q, k bf16 {128,1,64,1}; g fp32
// {128,...} ({64,...} with rotation); theta fp32 {64,...}; v bf16 {64,1,64,1} with 128-byte
// swizzle (the MN-major V tile).
struct Maps {
    CUtensorMap q, k, g, th, v;
};

struct Cfg {
    uint8_t* ring;             // [nc][RING][SLOT_BYTES]
    unsigned int* ready;       // [nc][RING]: sequence number + 1 of the chunk a slot holds
    unsigned int* consumed;    // [nc]: chunks the chain has copied out of its ring
    unsigned int* next_task;   // [1]: next task to hand out (dynamic order)
    int nc;                    // chain CTAs
    int dynamic;               // 1: tasks from the counter; 0: worker w takes w, w + W, ...
    unsigned long long wait_limit_ns;
    int fault_skip_commit;     // test hook: the first MMA completion of each worker is never signalled
    int discard;               // 1: the ring is 128-byte aligned, so consumed slots are dropped from L2
};

// Flag words after the ring (zeroed before every launch): ready, consumed, next_task.
__host__ __device__ constexpr size_t flag_words(size_t nc) { return nc * RING + nc + 1; }
__host__ __device__ constexpr size_t workspace_bytes(size_t nc) {
    return nc * RING * SLOT_BYTES + flag_words(nc) * sizeof(unsigned int);
}

constexpr unsigned STATUS_TIMEOUT = 1u;
constexpr unsigned STATUS_RANGE = 2u;

struct Task {
    int j;      // chain
    int gh;     // head (local index in [0, nheads))
    int s;      // sequence number of the chunk in its chain
    int c;      // chunk within the head
};

// Task t -> chain, head, chunk: waves of nc heads, chunk-major within a wave.
__device__ __forceinline__ Task decode_task(int t, int nc, int nheads, int nchunks) {
    const int per_wave = nc * nchunks;
    const int w = t / per_wave;
    const int tin = t - w * per_wave;
    const int nw = min(nc, nheads - w * nc);
    const int c = tin / nw;
    const int jj = tin - c * nw;
    return Task{jj, w * nc + jj, w * nchunks + c, c};
}

// Virtual heads: with p.nseg > 1 each head's sequence runs as segments of p.seg_len tokens
// (segments p.seg0 .. p.nseg - 1), each segment its own chain; otherwise a virtual head is a head.
struct Geo {
    int nv;        // virtual heads
    int ns;        // segments run per head
    int nchunks;   // chunks per virtual head
};
__device__ __forceinline__ Geo geometry(const FwdParams& p) {
    Geo g;
    g.ns = p.nseg > 1 ? p.nseg - p.seg0 : 1;
    g.nchunks = p.nseg > 1 ? p.seg_len / C : (p.T + C - 1) / C;
    g.nv = p.nheads * g.ns;
    return g;
}
__device__ __forceinline__ int vh_head(const FwdParams& p, const Geo& g, int vh) { return p.head0 + vh / g.ns; }
__device__ __forceinline__ int vh_seg(const FwdParams& p, const Geo& g, int vh) {
    return p.nseg > 1 ? p.seg0 + vh % g.ns : 0;
}
__device__ __forceinline__ int vh_t0(const FwdParams& p, const Geo& g, int vh) { return vh_seg(p, g, vh) * p.seg_len; }
// tokens of chunk c of a virtual head inside the sequence (0 for chunks past its end)
__device__ __forceinline__ int vh_chunk_len(const FwdParams& p, const Geo& g, int vh, int c) {
    const int len = p.nseg > 1 ? min(p.seg_len, p.T - vh_t0(p, g, vh)) : p.T;
    return max(0, min(C, len - c * C));
}
// flat index of token t of global head gx in a [B, T, H, ...] tensor (in units of rows)
__device__ __forceinline__ size_t tok_row(const FwdParams& p, int gx, int t) {
    return ((size_t)(gx / p.H) * p.T + t) * p.H + (gx % p.H);
}

__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// fp32 -> tf32 bits, round to nearest (ties away), with two integer operations.  Finite inputs.
__device__ __forceinline__ uint32_t to_tf32(float x) { return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u; }

__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// In-register transpose of an 8x8 block held by 8 consecutive lanes: lane j (j = lane & 7)
// enters with row j in v[0..7] and leaves with column j.
__device__ __forceinline__ void transpose8(float (&v)[8], int j) {
#pragma unroll
    for (int st = 4; st >= 1; st >>= 1) {
        const bool up = (j & st) != 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if ((e & st) == 0) {
                const float send = up ? v[e] : v[e | st];
                const float recv = __shfl_xor_sync(0xffffffffu, send, st);
                if (up) v[e] = recv; else v[e | st] = recv;
            }
        }
    }
}

__device__ __forceinline__ uint4 pack8(const float* m8) {
    using tc::pack_bf16x2;
    return make_uint4(pack_bf16x2(m8[0], m8[1]), pack_bf16x2(m8[2], m8[3]), pack_bf16x2(m8[4], m8[5]),
                      pack_bf16x2(m8[6], m8[7]));
}
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Columns [col0, col0 + n) of one state row times the per-column decay rho (real: one factor
// per key dim; rotation: key pair j multiplied by the complex rho_j = rho[j] + i rho[64 + j]).
template <bool ROT, int N>
__device__ __forceinline__ void scale_cols(float* s, int col0, const float* rho) {
    if (!ROT) {
#pragma unroll
        for (int u = 0; u < N; u += 4) {
            const float4 f = *reinterpret_cast<const float4*>(rho + col0 + u);
            s[u] *= f.x; s[u + 1] *= f.y; s[u + 2] *= f.z; s[u + 3] *= f.w;
        }
    } else {
#pragma unroll
        for (int u = 0; u < N; u += 2) {
            const int pr = (col0 + u) >> 1;
            const float cr = rho[pr], ci = rho[64 + pr];
            const float xr = s[u], xi = s[u + 1];
            s[u] = xr * cr - xi * ci;
            s[u + 1] = xr * ci + xi * cr;
        }
    }
}

// ======================================================================= prep worker ====

// Worker mbarriers (bars[i]).
constexpr int WB_IN = 0;         // inputs of the next task staged (producer: expect_tx; or a bare arrival: no task)
constexpr int WB_MMA1 = 1;       // [2] first MMA of a task done (commit), or a bare arrival: stop
constexpr int WB_ACCFREE = 3;    // [2] accumulator read back
constexpr int WB_EWDONE = 5;     // [2] elementwise group's part of a task written
constexpr int WB_WM = 7;         // [2] Wm^T MMA done (commit)
constexpr int WB_DUMMY = 9;      // [3] commits whose completion only the exit waits for
constexpr int WB_INFREE = 12;    // input tiles read into registers
constexpr int WB_SOLVED = 13;    // [2] solve group's part of a task staged (or a bare arrival: stop)
constexpr int WB_PUBREAD = 15;   // [2] publisher's copies have read a task's staged tiles
constexpr int WB_COUNT = 17;

template <bool ROT, bool EXT>
__device__ __forceinline__ void worker_elementwise(const FwdParams& p, const Cfg& cf, uint8_t* base, uint32_t sb,
                                                   uint32_t tbase, uint64_t* bars, int* abort_f, int* range_f,
                                                   const int* tk_ring) {
    // abort_f: this group's flag (set by thread 0 only, read by all after a group barrier)
    using namespace tc;
    uint64_t* b_in = bars + WB_IN;
    uint64_t* b_mma1 = bars + WB_MMA1;
    uint64_t* b_accfree = bars + WB_ACCFREE;
    uint64_t* b_ewdone = bars + WB_EWDONE;
    uint64_t* b_dummy = bars + WB_DUMMY;
    uint64_t* b_infree = bars + WB_INFREE;
    uint64_t* b_pubread = bars + WB_PUBREAD;
    const int tid = threadIdx.x, sg = tid >> 5, dg = tid & 31;
    const Geo geo = geometry(p);
    const int nchunks = geo.nchunks, NV = geo.nv, NC = cf.nc, total = NV * nchunks;
    const unsigned long long lim = cf.wait_limit_ns;
    const bool untied = EXT && p.w != nullptr;
    const bool qkn = EXT && p.qk_norm != 0;
    const float L2E = 1.4426950408889634f;
    const uint32_t kb = (uint32_t)(dg >> 4), ch = (uint32_t)((dg & 15) >> 1), in_ch = (uint32_t)(dg & 1) * 8u;
    const uint32_t ID_KK = idesc_bf16(128, 64, 0, 0, 0);
    float* QT = reinterpret_cast<float*>(base + WK_QT);
    int n_dummy = 0;
    bool skip_commit = cf.fault_skip_commit != 0;
    bool bad = false;
    int it = 0;
    bool stopped = false;     // left the loop by running out of tasks
    for (;; ++it) {
        const int pb = it & 1;
        // inputs of task it staged by the producer (or no task left)
        if (tid == 0) {
            if (!mbar_wait_bounded(b_in, (uint32_t)(it & 1), lim)) atomicExch(abort_f, 1);
            GDR_TL(true, it, 0);
        }
        named_bar(1, 256);
        if (*abort_f) break;
        const int task = tk_ring[it & 3];
        if (task >= total) {
            stopped = true;
            break;
        }
        const Task tk = decode_task(task, NC, NV, nchunks);
        const int gx = vh_head(p, geo, tk.gh);
        const int tc0 = vh_t0(p, geo, tk.gh) + tk.c * C;     // first token of the chunk
        const int Lc = vh_chunk_len(p, geo, tk.gh, tk.c);
        uint8_t* slot = cf.ring + ((size_t)tk.j * RING + tk.s % RING) * SLOT_BYTES;
        const bool slot_ok = GDR_INB(tk.j >= 0 && tk.j < NC && tk.s >= 0, 101);
        float beta_r = 0.f, w_r = 0.f;
        if (tid < Lc && GDR_INB(gx < p.B * p.H && tc0 + tid < p.T, 102)) {
            beta_r = __ldg(p.beta + tok_row(p, gx, tc0 + tid));
            w_r = untied ? __ldg(p.w + tok_row(p, gx, tc0 + tid)) : beta_r;
        }
        // ---- raw inputs of this thread's 8 tokens x 4 dims (tokens past T arrive as zeros) ----
        uint2 rk[8], rq[8];
        float4 ra[8];       // real: 4 gates; rotation: gates of the 2 pairs, then their 2 angles
#pragma unroll
        for (int s_ = 0; s_ < 8; ++s_) {
            const int r = 8 * sg + s_;
            rk[s_] = *reinterpret_cast<const uint2*>(base + IN_K + (uint32_t)(r * D + 4 * dg) * 2u);
            rq[s_] = *reinterpret_cast<const uint2*>(base + IN_Q + (uint32_t)(r * D + 4 * dg) * 2u);
            if (!ROT) {
                ra[s_] = *reinterpret_cast<const float4*>(base + IN_G + (uint32_t)(r * D + 4 * dg) * 4u);
            } else {
                const float2 g2 = *reinterpret_cast<const float2*>(base + IN_G + (uint32_t)(r * 64 + 2 * dg) * 4u);
                const float2 t2 = *reinterpret_cast<const float2*>(base + IN_TH + (uint32_t)(r * 64 + 2 * dg) * 4u);
                ra[s_] = make_float4(g2.x, g2.y, t2.x, t2.y);
            }
        }
        named_bar(1, 256);           // the input tiles are free: the producer may stage the next task
        if (tid == 0) mbar_arrive(b_infree);

        // ---- gate pass: 1/alpha per token (real: per dim; rotation: per pair, with the phase) ----
        // x = 1/alpha = 1 + e^{a} (raw gate a, g = -softplus(a)) or e^{-g} (log-decay g); the
        // segment products of x (and of e^{i theta}) go to the table QT.
        float xv[8][4], sn[8][2];
        float nk[8], nq[8];
        float X[4] = {1.f, 1.f, 1.f, 1.f};
        float Zr[2] = {1.f, 1.f}, Zi[2] = {0.f, 0.f};
#pragma unroll
        for (int s_ = 0; s_ < 8; ++s_) {
            const bool ok = 8 * sg + s_ < Lc;
            const float ga[4] = {ra[s_].x, ra[s_].y, ra[s_].z, ra[s_].w};
#pragma unroll
            for (int d = 0; d < (ROT ? 2 : 4); ++d) {
                float x = 1.f;
                if (ok) x = (p.gate_mode == 1) ? 1.f + ex2_approx(ga[d] * L2E) : ex2_approx(-ga[d] * L2E);
                xv[s_][d] = x;
                X[d] *= x;
            }
            if (ROT) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float cs = 1.f, sv = 0.f;
                    if (ok) __sincosf(ga[2 + j], &sv, &cs);
                    xv[s_][2 + j] = cs;
                    sn[s_][j] = sv;
                    const float zr = Zr[j] * cs - Zi[j] * sv, zi = Zi[j] * cs + Zr[j] * sv;
                    Zr[j] = zr; Zi[j] = zi;
                }
            }
            if (qkn) {       // inverse L2 norms of this token's k and q (the warp holds all 128 dims)
                const uint2 kr = rk[s_], qr = rq[s_];
                float skk = bf_lo(kr.x) * bf_lo(kr.x) + bf_hi(kr.x) * bf_hi(kr.x) + bf_lo(kr.y) * bf_lo(kr.y) +
                            bf_hi(kr.y) * bf_hi(kr.y);
                float sqq = bf_lo(qr.x) * bf_lo(qr.x) + bf_hi(qr.x) * bf_hi(qr.x) + bf_lo(qr.y) * bf_lo(qr.y) +
                            bf_hi(qr.y) * bf_hi(qr.y);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    skk += __shfl_xor_sync(0xffffffffu, skk, off);
                    sqq += __shfl_xor_sync(0xffffffffu, sqq, off);
                }
                nk[s_] = rsqrtf(skk + 1e-6f);
                nq[s_] = rsqrtf(sqq + 1e-6f);
            }
        }
        {
            float4* qt = reinterpret_cast<float4*>(QT + (sg * 32 + dg) * 8);
            if (!ROT) {
                qt[0] = make_float4(X[0], X[1], X[2], X[3]);
            } else {
                qt[0] = make_float4(X[0], X[1], Zr[0], Zr[1]);
                qt[1] = make_float4(Zi[0], Zi[1], 0.f, 0.f);
            }
        }
        // Before anything is rewritten: the ring slot must be free (its chain has copied out chunk
        // s - RING), the tiles [Ktil ; Qtil] of task it - 2 read by the Wm^T MMA and the publisher,
        // and Khat of task it - 1 read by its first MMA.
        if (tid == 0) {
            GDR_TL(true, it, 1);
            if (tk.s >= RING &&
                !spin_until_ge(cf.consumed + tk.j, (unsigned)(tk.s - RING + 1), lim))
                atomicExch(abort_f, 1);
            if (it >= 2 && !mbar_wait_bounded(b_pubread + pb, (uint32_t)(((it - 2) >> 1) & 1), lim))
                atomicExch(abort_f, 1);
            if (it >= 1 && !mbar_wait_bounded(b_mma1 + (pb ^ 1), (uint32_t)(((it - 1) >> 1) & 1), lim))
                atomicExch(abort_f, 1);
        }
        named_bar(1, 256);
        if (*abort_f) break;
        GDR_TL(tid == 0, it, 2);

        // ---- reference decays: P_m (tokens 0..31) and P_m^{-1} P_C (tokens 32..63) -> ring ----
        float* rvec = reinterpret_cast<float*>(slot + SL_VEC);
        if (!slot_ok) {
        } else if (!ROT) {
            if (tid < 128) {
                const int d = tid;
                float lo = 1.f, hi = 1.f;
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) lo *= QT[(s2 * 32 + (d >> 2)) * 8 + (d & 3)];
#pragma unroll
                for (int s2 = 4; s2 < 8; ++s2) hi *= QT[(s2 * 32 + (d >> 2)) * 8 + (d & 3)];
                rvec[d] = 1.f / lo;
                rvec[128 + d] = 1.f / hi;
            }
        } else if (tid < 64) {
            const int jp = tid, g4 = jp >> 1, j = jp & 1;
            float ml = 1.f, mh = 1.f, lr = 1.f, li = 0.f, hr = 1.f, hi_ = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
                const float* e = QT + (s2 * 32 + g4) * 8;
                const float m = e[j], zr = e[2 + j], zi = e[4 + j];
                if (s2 < 4) {
                    ml *= m;
                    const float nr = lr * zr - li * zi, ni = li * zr + lr * zi;
                    lr = nr; li = ni;
                } else {
                    mh *= m;
                    const float nr = hr * zr - hi_ * zi, ni = hi_ * zr + hr * zi;
                    hr = nr; hi_ = ni;
                }
            }
            const float il = 1.f / ml, ih = 1.f / mh;
            rvec[jp] = il * lr;
            rvec[64 + jp] = il * li;
            rvec[128 + jp] = ih * hr;
            rvec[192 + jp] = ih * hi_;
        }

        // ---- tile pass: factors around token 31; [Ktil ; Qtil], Khat -> tiles; Qtil, Khat^T -> ring ----
        {
            uint8_t* KQ = base + WK_KQ + pb * 32768;
            uint8_t* KH = base + WK_KH;
            const float sc = p.scale;
            float khb[4][4];        // Khat of 4 consecutive tokens, for the fp32 Khat^T store
            float Rre[2] = {1.f, 1.f}, Rim[2] = {0.f, 0.f};
            // one token: fk / fh magnitudes of the Ktil / Khat factors (rotation: times R)
            auto emit = [&](int s_, const float (&fk)[4], const float (&fh)[4]) {
                const int r = 8 * sg + s_;
                float kk[4] = {bf_lo(rk[s_].x), bf_hi(rk[s_].x), bf_lo(rk[s_].y), bf_hi(rk[s_].y)};
                float qv[4] = {bf_lo(rq[s_].x), bf_hi(rq[s_].x), bf_lo(rq[s_].y), bf_hi(rq[s_].y)};
                if (qkn) {
#pragma unroll
                    for (int d = 0; d < 4; ++d) { kk[d] *= nk[s_]; qv[d] *= nq[s_]; }
                }
                float kt[4], qt[4], kh[4];
                if (!ROT) {
#pragma unroll
                    for (int d = 0; d < 4; ++d) {
                        kt[d] = kk[d] * fk[d];
                        qt[d] = qv[d] * (sc * fk[d]);
                        kh[d] = kk[d] * fh[d];
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float fr = fk[j] * Rre[j], fi = fk[j] * Rim[j];
                        const float hr = fh[j] * Rre[j], hi = fh[j] * Rim[j];
                        const float k0 = kk[2 * j], k1 = kk[2 * j + 1], q0 = sc * qv[2 * j], q1 = sc * qv[2 * j + 1];
                        kt[2 * j] = fr * k0 - fi * k1; kt[2 * j + 1] = fr * k1 + fi * k0;
                        qt[2 * j] = fr * q0 - fi * q1; qt[2 * j + 1] = fr * q1 + fi * q0;
                        kh[2 * j] = hr * k0 - hi * k1; kh[2 * j + 1] = hr * k1 + hi * k0;
                    }
                }
                const uint32_t off = sw128_off((uint32_t)r, ch) + in_ch;
                const uint2 qpk = make_uint2(pack_bf16x2(qt[0], qt[1]), pack_bf16x2(qt[2], qt[3]));
                *reinterpret_cast<uint2*>(KQ + kb * 16384u + off) =
                    make_uint2(pack_bf16x2(kt[0], kt[1]), pack_bf16x2(kt[2], kt[3]));
                *reinterpret_cast<uint2*>(KQ + kb * 16384u + 8192u + off) = qpk;
                *reinterpret_cast<uint2*>(KH + kb * 8192u + off) =
                    make_uint2(pack_bf16x2(kh[0], kh[1]), pack_bf16x2(kh[2], kh[3]));
#pragma unroll
                for (int d = 0; d < 4; ++d) khb[s_ & 3][d] = kh[d];
            };
            // Khat^T (fp32, K-major over tokens) of tokens 8sg + 4h .. + 3, one 16-byte store per dim
            auto flush_khat = [&](int h) {
                const uint32_t kb2 = (uint32_t)(sg >> 2);                 // token half
                const uint32_t c16 = (uint32_t)(2 * (sg & 3) + h);        // 16-byte chunk of the row
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t d = (uint32_t)(4 * dg + e);
                    if (slot_ok) *reinterpret_cast<float4*>(slot + SL_H + kb2 * 16384u + sw128_off(d, c16)) =
                        make_float4(khb[0][e], khb[1][e], khb[2][e], khb[3][e]);
                }
            };
            float F[4] = {1.f, 1.f, 1.f, 1.f};
            if (sg < 4) {
                // backward from token 31: F = prod of x over tokens r+1..31 at token r
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    if (s2 <= sg) continue;
                    const float* e = QT + (s2 * 32 + dg) * 8;
                    if (!ROT) {
                        F[0] *= e[0]; F[1] *= e[1]; F[2] *= e[2]; F[3] *= e[3];
                    } else {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            F[j] *= e[j];
                            const float zr = e[2 + j], zi = e[4 + j];
                            const float nr = Rre[j] * zr - Rim[j] * zi, ni = Rim[j] * zr + Rre[j] * zi;
                            Rre[j] = nr; Rim[j] = ni;
                        }
                    }
                }
#pragma unroll
                for (int s_ = 7; s_ >= 0; --s_) {
                    float fh[4];
#pragma unroll
                    for (int d = 0; d < 4; ++d) fh[d] = rcp_approx(F[d]);
                    emit(s_, F, fh);
                    if (s_ == 4) flush_khat(1);
                    if (s_ == 0) flush_khat(0);
#pragma unroll
                    for (int d = 0; d < (ROT ? 2 : 4); ++d) F[d] *= xv[s_][d];
                    if (ROT) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float cs = xv[s_][2 + j], sv = sn[s_][j];
                            const float nr = Rre[j] * cs - Rim[j] * sv, ni = Rim[j] * cs + Rre[j] * sv;
                            Rre[j] = nr; Rim[j] = ni;
                        }
                    }
                }
            } else {
                // forward from token 32: F = prod of x over tokens 32..r (the Khat factor)
#pragma unroll
                for (int s2 = 4; s2 < 8; ++s2) {
                    if (s2 >= sg) continue;
                    const float* e = QT + (s2 * 32 + dg) * 8;
                    if (!ROT) {
                        F[0] *= e[0]; F[1] *= e[1]; F[2] *= e[2]; F[3] *= e[3];
                    } else {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            F[j] *= e[j];
                            const float zr = e[2 + j], zi = -e[4 + j];         // conjugate phase
                            const float nr = Rre[j] * zr - Rim[j] * zi, ni = Rim[j] * zr + Rre[j] * zi;
                            Rre[j] = nr; Rim[j] = ni;
                        }
                    }
                }
#pragma unroll
                for (int s_ = 0; s_ < 8; ++s_) {
#pragma unroll
                    for (int d = 0; d < (ROT ? 2 : 4); ++d) F[d] *= xv[s_][d];
                    if (ROT) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float cs = xv[s_][2 + j], sv = -sn[s_][j];
                            const float nr = Rre[j] * cs - Rim[j] * sv, ni = Rim[j] * cs + Rre[j] * sv;
                            Rre[j] = nr; Rim[j] = ni;
                        }
                    }
                    float fk[4];
#pragma unroll
                    for (int d = 0; d < 4; ++d) fk[d] = rcp_approx(F[d]);
                    emit(s_, fk, F);
                    if (s_ == 3) flush_khat(0);
                    if (s_ == 7) flush_khat(1);
                }
            }
            // The products grow monotonically away from token 31: the final ones bound every
            // factor this thread used.
#pragma unroll
            for (int d = 0; d < (ROT ? 2 : 4); ++d)
                if (!(F[d] < 3e38f)) bad = true;
        }
        {
            float* vsm = reinterpret_cast<float*>(base + WK_VEC) + pb * 128;
            if (tid < 64) {
                vsm[tid] = beta_r;
                vsm[64 + tid] = w_r;
            }
        }
        fence_proxy_async_smem();
        named_bar(1, 256);
        if (tid == 0) {
            GDR_TL(true, it, 3);
            mbar_arrive(b_ewdone + pb);      // ring parts, vectors and the task's beta / w are written
            if (it >= 2 && !mbar_wait_bounded(b_accfree + pb, (uint32_t)(((it - 2) >> 1) & 1), lim))
                atomicExch(abort_f, 1);
            if (*abort_f == 0) {
                // [A' ; Pm] = [Ktil ; Qtil] Khat^T (128 x 64 x 128) -> accumulator pb
                tc_fence_after();
                const uint32_t kq_s = sb + WK_KQ + pb * 32768, kh_s = sb + WK_KH;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t kbk = ks >> 2, kin = (ks & 3) * 32;
                    mma_bf16_ss(tbase + COL_ACC + pb * 64, sdesc_sw128(kq_s + kbk * 16384 + kin, 16, 1024),
                                sdesc_sw128(kh_s + kbk * 8192 + kin, 16, 1024), ID_KK, ks > 0);
                }
                if (skip_commit) {
                    mma_commit(b_dummy);
                    ++n_dummy;
                } else {
                    mma_commit(b_mma1 + pb);
                }
                skip_commit = false;
            }
        }
    }
    if (bad) atomicExch(range_f, 1);
    if (tid == 0) {
        if (stopped) {
            mbar_arrive(b_mma1 + (it & 1));     // tells the solve warps there is no task it
        } else {
            // gave up: MMAs still in flight finish before the CTA ends
            mma_commit(b_dummy);
            ++n_dummy;
        }
        if (n_dummy > 0) (void)mbar_wait_bounded(b_dummy, (uint32_t)((n_dummy - 1) & 1), lim);
    }
}

// Producer (one thread): claims tasks in increasing order, stages each one's q, k, gates (and
// angles) with tensor-map copies into the input tiles once the elementwise group has read the
// previous ones, and records the task in tk_ring; past the last task it records a value >= the
// task count and arrives on the input barrier without copies.
template <bool ROT>
__device__ __forceinline__ void worker_producer(const FwdParams& p, const Cfg& cf, const Maps& tm, uint32_t sb,
                                                uint64_t* bars, int* abort_f, int* tk_ring) {
    using namespace tc;
    uint64_t* b_in = bars + WB_IN;
    uint64_t* b_infree = bars + WB_INFREE;
    const Geo geo = geometry(p);
    const int nchunks = geo.nchunks, NV = geo.nv, NC = cf.nc, total = NV * nchunks;
    const unsigned long long lim = cf.wait_limit_ns;
    const int nworkers = (int)gridDim.x - NC;
    int fixed_next = (int)blockIdx.x - NC;
    auto claim = [&]() -> int {
        if (cf.dynamic) return min((int)atomicAdd(cf.next_task, 1u), total);
        const int t = fixed_next;
        fixed_next += nworkers;
        return min(t, total);
    };
    int staged = 0;
    bool gave_up = false;
    int t = claim();
    for (int i = 0;; ++i) {
        if (i >= 1 && !mbar_wait_bounded(b_infree, (uint32_t)((i - 1) & 1), lim)) {
            atomicExch(abort_f, 1);
            gave_up = true;
            break;
        }
        tk_ring[i & 3] = t;
        if (t >= total) {
            mbar_arrive(b_in);          // no task i: the elementwise group stops
            break;
        }
        const Task tk = decode_task(t, NC, NV, nchunks);
        const int gx = vh_head(p, geo, tk.gh), bb = gx / p.H, hh = gx % p.H;
        const int t0 = vh_t0(p, geo, tk.gh) + tk.c * C;     // tokens past T arrive as zeros
        mbar_arrive_expect_tx(b_in, 65536u);
        tma_load_4d(sb + IN_Q, &tm.q, 0, hh, t0, bb, b_in);
        tma_load_4d(sb + IN_K, &tm.k, 0, hh, t0, bb, b_in);
        tma_load_4d(sb + IN_G, &tm.g, 0, hh, t0, bb, b_in);
        if (ROT) tma_load_4d(sb + IN_TH, &tm.th, 0, hh, t0, bb, b_in);
        ++staged;
        t = claim();                    // the next claim overlaps these copies
    }
    // After giving up, copies still in flight land before the CTA ends.  (Otherwise the
    // elementwise group has waited for every one of them.)
    if (gave_up && staged > 0) (void)mbar_wait_bounded(b_in, (uint32_t)((staged - 1) & 1), lim);
}

// Publisher (one thread): once the solve group has staged a task's tiles, copies Pm, Wm2^T and
// Tw (Tb) into the task's ring slot with bulk copies, waits until they are written, and
// publishes the slot with a release store (the elementwise group's stores to the slot happened
// before, through the task's barriers).
template <bool EXT>
__device__ __forceinline__ void worker_publisher(const FwdParams& p, const Cfg& cf, uint32_t sb, uint64_t* bars,
                                                 int* abort_f, const int* tk_ring) {
    using namespace tc;
    uint64_t* b_solved = bars + WB_SOLVED;
    uint64_t* b_pubread = bars + WB_PUBREAD;
    const Geo geo = geometry(p);
    const int nchunks = geo.nchunks, NV = geo.nv, NC = cf.nc, total = NV * nchunks;
    const unsigned long long lim = cf.wait_limit_ns;
    const bool untied = EXT && p.w != nullptr;
    for (int i = 0;; ++i) {
        const int pb = i & 1;
        if (!mbar_wait_bounded(b_solved + pb, (uint32_t)((i >> 1) & 1), lim)) {
            atomicExch(abort_f, 1);
            break;
        }
        const int task = tk_ring[i & 3];
        if (task >= total) break;
        const Task tk = decode_task(task, NC, NV, nchunks);
        uint8_t* slot = cf.ring + ((size_t)tk.j * RING + tk.s % RING) * SLOT_BYTES;
        const uint32_t kq = sb + WK_KQ + (uint32_t)pb * 32768u;
        if (!GDR_INB(tk.j >= 0 && tk.j < NC && tk.s >= 0, 104)) {      // neither copy nor publish
            mbar_arrive(b_pubread + pb);
            continue;
        }
        bulk_s2g(slot + SL_Q, kq + 8192u, 8192u);                  // Qtil, dk 0..63
        bulk_s2g(slot + SL_Q + 8192u, kq + 16384u + 8192u, 8192u); // Qtil, dk 64..127
        bulk_s2g(slot + SL_P, sb + WK_PMS, 16384u);
        bulk_s2g(slot + SL_W, sb + WK_TF, 16384u);
        bulk_s2g(slot + SL_T, sb + (untied ? WK_TW : WK_TB), 8192u);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(b_pubread + pb);    // the staged tiles may be rewritten
        bulk_wait_all();
        fence_proxy_async_global();
        st_release_gpu(cf.ready + (size_t)tk.j * RING + tk.s % RING, (unsigned)(tk.s + 1));
        GDR_TL(true, i, 9);
    }
    bulk_wait_all();
}

template <bool EXT>
__device__ __forceinline__ void worker_solve(const FwdParams& p, const Cfg& cf, uint8_t* base, uint32_t sb,
                                             uint32_t tbase, uint64_t* bars, int* abort_f, const int* tk_ring) {
    using namespace tc;
    uint64_t* b_mma1 = bars + WB_MMA1;
    uint64_t* b_accfree = bars + WB_ACCFREE;
    uint64_t* b_ewdone = bars + WB_EWDONE;
    uint64_t* b_wm = bars + WB_WM;
    uint64_t* b_dummy2 = bars + WB_DUMMY + 1;
    uint64_t* b_solved = bars + WB_SOLVED;
    uint64_t* b_pubread = bars + WB_PUBREAD;
    const int stid = (int)threadIdx.x - 384;     // warps 12-15
    const int sw = stid >> 5, lane = stid & 31;
    const int qd = sw;                           // TMEM lane quadrant of this warp (warp & 3)
    const Geo geo = geometry(p);
    const int total = geo.nv * geo.nchunks;
    const unsigned long long lim = cf.wait_limit_ns;
    const bool untied = EXT && p.w != nullptr;
    const uint32_t tq = tbase + ((uint32_t)(qd * 32) << 16);
    uint8_t* PMS = base + WK_PMS;
    float* Af = reinterpret_cast<float*>(base + WK_AF);
    float* Tf = reinterpret_cast<float*>(base + WK_TF);
    uint8_t* TB = base + WK_TB;
    uint8_t* TW = base + WK_TW;
    const uint32_t ID_MK = idesc_bf16(128, 64, 1, 0, 0);
    const int gid = lane >> 2, tig = lane & 3;
    bool wm_pending = false;
    int n_wm = 0;
    for (int it = 0;; ++it) {
        const int pb = it & 1;
        if (stid == 0 && !mbar_wait_bounded(b_mma1 + pb, (uint32_t)((it >> 1) & 1), lim)) atomicExch(abort_f, 1);
        named_bar(2, 128);
        if (*abort_f) break;
        // No task for iteration it: the elementwise group stored a value >= total and arrived on the
        // barrier itself (a release).  Otherwise the value is re-read below, after the barrier on
        // which the elementwise group published this task's data.
        if (tk_ring[it & 3] >= total) {
            if (stid == 0) mbar_arrive(b_solved + pb);     // tells the publisher there is no task it
            break;
        }
        if (stid == 0) {
            if (!mbar_wait_bounded(b_ewdone + pb, (uint32_t)((it >> 1) & 1), lim)) atomicExch(abort_f, 1);
            // the publisher has read the tiles staged for task it - 1
            if (it >= 1 && !mbar_wait_bounded(b_pubread + (pb ^ 1), (uint32_t)(((it - 1) >> 1) & 1), lim))
                atomicExch(abort_f, 1);
        }
        named_bar(2, 128);
        if (*abort_f) break;
        GDR_TL(stid == 0, it, 4);
        tc_fence_after();
        const float* vsm = reinterpret_cast<const float*>(base + WK_VEC) + pb * 128;   // beta[64], w[64]
        // ---- read back [A' ; Pm]: rows 0-63 -> A = diag(beta) strict_lower(A') (fp32, shared);
        //      rows 64-127 -> masked Pm (fp32), staged in its ring layout --------------------------
        {
            float v[64];
            tmem_ld32(tq + COL_ACC + pb * 64, *reinterpret_cast<float(*)[32]>(v));
            tmem_ld32(tq + COL_ACC + pb * 64 + 32, *reinterpret_cast<float(*)[32]>(v + 32));
            if (qd < 2) {
                const int r = qd * 32 + lane;
                const float br = vsm[r];
#pragma unroll
                for (int i = 0; i < 64; i += 4) {
                    float4 w4;
                    w4.x = (i < r) ? br * v[i] : 0.f;
                    w4.y = (i + 1 < r) ? br * v[i + 1] : 0.f;
                    w4.z = (i + 2 < r) ? br * v[i + 2] : 0.f;
                    w4.w = (i + 3 < r) ? br * v[i + 3] : 0.f;
                    *reinterpret_cast<float4*>(Af + r * AS + i) = w4;
                }
            } else {
                const int r = (qd - 2) * 32 + lane;
#pragma unroll
                for (int i = 0; i < 64; i += 4) {
                    float4 w4;
                    w4.x = (i <= r) ? v[i] : 0.f;
                    w4.y = (i + 1 <= r) ? v[i + 1] : 0.f;
                    w4.z = (i + 2 <= r) ? v[i + 2] : 0.f;
                    w4.w = (i + 3 <= r) ? v[i + 3] : 0.f;
                    *reinterpret_cast<float4*>(PMS + (uint32_t)(i >> 5) * 8192u +
                                               sw128_off((uint32_t)r, (uint32_t)((i & 31) >> 2))) = w4;
                }
            }
        }
        {   // Tb (and Tw) start from zero: the blocks above the diagonal stay so
            uint4* z = reinterpret_cast<uint4*>(TB);
#pragma unroll
            for (int e = 0; e < 4; ++e) z[stid + 128 * e] = make_uint4(0u, 0u, 0u, 0u);
            if (untied) {
                uint4* zw = reinterpret_cast<uint4*>(TW);
#pragma unroll
                for (int e = 0; e < 4; ++e) zw[stid + 128 * e] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        tc_fence_before();
        named_bar(2, 128);
        if (stid == 0) mbar_arrive(b_accfree + pb);
        GDR_TL(stid == 0, it, 5);
        // Tb / Tw elements (row r, columns i and i + 1) from T
        auto tb_put2 = [&](int r, int i, float x0, float x1) {
            const uint32_t off = sw128_off((uint32_t)r, (uint32_t)(i >> 3)) + (uint32_t)(i & 7) * 2u;
            *reinterpret_cast<uint32_t*>(TB + off) = pack_bf16x2(x0 * vsm[i], x1 * vsm[i + 1]);
            if (untied) *reinterpret_cast<uint32_t*>(TW + off) = pack_bf16x2(x0 * vsm[64 + i], x1 * vsm[64 + i + 1]);
        };
        // ---- the four 16x16 diagonal blocks: forward substitution, one column per thread ----------
        if (stid < 64) {
            const int bb = (stid >> 4) * 16, jj = stid & 15;
            float s[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) s[i] = (i == jj) ? 1.f : 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const float tr = s[r];
#pragma unroll
                for (int i = r + 1; i < 16; ++i) s[i] = fmaf(-Af[(bb + i) * AS + bb + r], tr, s[i]);
            }
            const int ic = bb + jj;
            const float bj = vsm[ic], wj = vsm[64 + ic];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                Tf[(bb + i) * AS + ic] = s[i];
                const uint32_t off = sw128_off((uint32_t)(bb + i), (uint32_t)(ic >> 3)) + (uint32_t)(ic & 7) * 2u;
                *reinterpret_cast<__nv_bfloat16*>(TB + off) = __float2bfloat16_rn(s[i] * bj);
                if (untied) *reinterpret_cast<__nv_bfloat16*>(TW + off) = __float2bfloat16_rn(s[i] * wj);
            }
        }
        named_bar(2, 128);
        GDR_TL(stid == 0, it, 6);
        // ---- blocks below the diagonal (T_IJ = -D_I sum_{K=J}^{I-1} A_IK T_KJ), tf32 warp MMAs ---------
        //   phase 1: T10 = -D1 (A10 D0), T32 = -D3 (A32 D2), X21 = A21 D1, X31 = A31 D1
        //   phase 2: X20 = A20 D0 + A21 T10, X30 = A30 D0 + A31 T10, T21 = -D2 X21, T31 = -(T32 X21 + D3 X31)
        //   phase 3: T20 = -D2 X20, T30 = -(T32 X20 + D3 X30)
        // The X blocks live in the unused blocks above the diagonal of T.
        {
            auto Ab = [&](int I, int J) -> const float* { return Af + 16 * I * AS + 16 * J; };
            auto Tb_ = [&](int I, int J) -> float* { return Tf + 16 * I * AS + 16 * J; };
            auto mm = [&](float (&acc)[2][4], const float* L, const float* R) {   // acc += L R (16x16)
#pragma unroll
                for (int k8 = 0; k8 < 16; k8 += 8) {
                    const uint32_t a[4] = {to_tf32(L[gid * AS + k8 + tig]), to_tf32(L[(gid + 8) * AS + k8 + tig]),
                                           to_tf32(L[gid * AS + k8 + tig + 4]), to_tf32(L[(gid + 8) * AS + k8 + tig + 4])};
                    const uint32_t b0[2] = {to_tf32(R[(k8 + tig) * AS + gid]), to_tf32(R[(k8 + tig + 4) * AS + gid])};
                    const uint32_t b1[2] = {to_tf32(R[(k8 + tig) * AS + 8 + gid]), to_tf32(R[(k8 + tig + 4) * AS + 8 + gid])};
                    mma_tf32_16x8x8(acc[0], a, b0);
                    mma_tf32_16x8x8(acc[1], a, b1);
                }
            };
            auto zero = [&](float (&acc)[2][4]) {
#pragma unroll
                for (int h = 0; h < 2; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
            };
            auto put = [&](float* Dst, const float (&acc)[2][4], float sgn) {     // Dst = sgn * acc
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    *reinterpret_cast<float2*>(Dst + gid * AS + 8 * h + 2 * tig) = make_float2(sgn * acc[h][0], sgn * acc[h][1]);
                    *reinterpret_cast<float2*>(Dst + (gid + 8) * AS + 8 * h + 2 * tig) =
                        make_float2(sgn * acc[h][2], sgn * acc[h][3]);
                }
                __syncwarp();
            };
            auto out = [&](int I, int J, const float (&acc)[2][4]) {      // Tb / Tw block (I, J) = -acc
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int i = 16 * J + 8 * h + 2 * tig;
                    tb_put2(16 * I + gid, i, -acc[h][0], -acc[h][1]);
                    tb_put2(16 * I + gid + 8, i, -acc[h][2], -acc[h][3]);
                }
            };
            float x[2][4], y[2][4];
            if (sw == 0) {
                zero(x); mm(x, Ab(1, 0), Tb_(0, 0)); put(Tb_(0, 1), x, 1.f);
                zero(y); mm(y, Tb_(1, 1), Tb_(0, 1)); put(Tb_(1, 0), y, -1.f); out(1, 0, y);
            } else if (sw == 1) {
                zero(x); mm(x, Ab(3, 2), Tb_(2, 2)); put(Tb_(2, 3), x, 1.f);
                zero(y); mm(y, Tb_(3, 3), Tb_(2, 3)); put(Tb_(3, 2), y, -1.f); out(3, 2, y);
            } else if (sw == 2) {
                zero(x); mm(x, Ab(2, 1), Tb_(1, 1)); put(Tb_(0, 2), x, 1.f);          // X21
            } else {
                zero(x); mm(x, Ab(3, 1), Tb_(1, 1)); put(Tb_(0, 3), x, 1.f);          // X31
            }
            named_bar(2, 128);
            if (sw == 0) {
                zero(x); mm(x, Ab(2, 0), Tb_(0, 0)); mm(x, Ab(2, 1), Tb_(1, 0)); put(Tb_(1, 2), x, 1.f);   // X20
            } else if (sw == 1) {
                zero(x); mm(x, Ab(3, 0), Tb_(0, 0)); mm(x, Ab(3, 1), Tb_(1, 0)); put(Tb_(1, 3), x, 1.f);   // X30
            } else if (sw == 2) {
                zero(y); mm(y, Tb_(2, 2), Tb_(0, 2)); out(2, 1, y);                                      // T21
            } else {
                zero(y); mm(y, Tb_(3, 2), Tb_(0, 2)); mm(y, Tb_(3, 3), Tb_(0, 3)); out(3, 1, y);          // T31
            }
            named_bar(2, 128);
            if (sw == 0) {
                zero(y); mm(y, Tb_(2, 2), Tb_(1, 2)); out(2, 0, y);                                      // T20
            } else if (sw == 1) {
                zero(y); mm(y, Tb_(3, 2), Tb_(1, 2)); mm(y, Tb_(3, 3), Tb_(1, 3)); out(3, 0, y);          // T30
            }
        }
        fence_proxy_async_smem();
        named_bar(2, 128);
        GDR_TL(stid == 0, it, 7);
        // ---- Wm^T = Ktil^T Tb^T (128 x 64 x 64) -> TMEM ------------------------------------------------
        if (stid == 0) {
            tc_fence_after();
            const uint32_t kq_s = sb + WK_KQ + pb * 32768;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tbase + COL_WM, sdesc_sw128(kq_s + ks * 2048, 16384, 1024),
                            sdesc_sw128(sb + WK_TB + ks * 32, 16, 1024), ID_MK, ks > 0);
            mma_commit(b_wm + pb);
            wm_pending = true;
            ++n_wm;
        }
        if (stid == 0) {
            if (!mbar_wait_bounded(b_wm + pb, (uint32_t)((it >> 1) & 1), lim)) atomicExch(abort_f, 1);
            else wm_pending = false;
        }
        named_bar(2, 128);
        if (*abort_f) break;
        GDR_TL(stid == 0, it, 8);
        tc_fence_after();
        {   // Wm^T (lane = dk row, 64 tokens) -> bf16 MN-major tile, staged (over T) in its ring layout
            float v[64];
            tmem_ld32(tq + COL_WM, *reinterpret_cast<float(*)[32]>(v));
            tmem_ld32(tq + COL_WM + 32, *reinterpret_cast<float(*)[32]>(v + 32));
            const uint32_t d = (uint32_t)(qd * 32 + lane);
            uint8_t* WS = base + WK_TF;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                *reinterpret_cast<uint4*>(WS + sw128_off(d, (uint32_t)cc)) = pack8(v + cc * 8);
        }
        tc_fence_before();
        fence_proxy_async_smem();     // the staged tiles are read by the publisher's bulk copies
        named_bar(2, 128);
        if (stid == 0) mbar_arrive(b_solved + pb);
    }
    if (stid == 0 && wm_pending) {   // gave up with the Wm^T MMA in flight
        mma_commit(b_dummy2);
        (void)mbar_wait_bounded(b_dummy2, 0u, lim);
    }
    (void)n_wm;
}

// ======================================================================= state chain ====

template <bool ROT, typename OT, bool EXT>
__device__ __forceinline__ void chain_role(const FwdParams& p, const Cfg& cf, const Maps& tm, uint8_t* base, uint32_t sb,
                                           uint32_t tbase, uint64_t* bars, int* ab) {
    using namespace tc;
    uint64_t* bar_full = bars;        // [2] slot buffer landed
    uint64_t* bar_v = bars + 2;       // V tile landed
    uint64_t* bar_u = bars + 3;       // U^T MMA done (V buffer free)
    uint64_t* bar_e = bars + 4;       // E^T MMA done
    uint64_t* bar_s = bars + 5;       // state MMA done
    uint64_t* bar_o = bars + 6;       // [2] O^T MMAs done
    uint64_t* bar_sbr = bars + 8;     // prescaled state of the next chunk written (bf16 copy)
    uint64_t* bar_ofree = bars + 9;   // [2] O^T read out of TMEM
    uint64_t* bar_empty = bars + 11;  // [2] slot buffer released (every MMA that read it done)
    uint64_t* bar_dummy = bars + 13;
    uint64_t* bar_sf = bars + 14;     // prescaled state of the next chunk written (fp32 accumulator)
    uint64_t* bar_vec = bars + 15;    // [4] decay vectors of a chunk landed
    uint64_t* bar_vfree = bars + 19;  // [4] decay vectors of a chunk no longer needed
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = (int)blockIdx.x;
    const Geo geo = geometry(p);
    const int nchunks = geo.nchunks, NV = geo.nv, NC = cf.nc;
    const int nwaves = (NV - j + NC - 1) / NC;       // virtual heads j, j + NC, ...
    const int nseq = nwaves * nchunks;
    const unsigned long long lim = cf.wait_limit_ns;
    const bool cmean = EXT && p.chunk_mean != nullptr;
    const bool vzero = p.v == nullptr;               // zero values: no V tile, U^T = 0
    auto vh_of = [&](int s) -> int { return j + (s / nchunks) * NC; };               // virtual head
    auto head_of = [&](int s) -> int { return vh_head(p, geo, vh_of(s)); };          // global head
    auto tok0_of = [&](int s) -> int { return vh_t0(p, geo, vh_of(s)) + (s % nchunks) * C; };   // chunk's first token

    if (warp == 0) {
        // ---------------- loader ----------------------------------------------------------------
        int* abort_f = ab + 0;
        int v_issued = 0;
        for (int s = 0; s < nseq; ++s) {
            const int b = s & 1;
            const uint8_t* src = cf.ring + ((size_t)j * RING + s % RING) * SLOT_BYTES;
            bool ok = true;
            if (lane == 0) {
                if (s >= 2) ok = mbar_wait_bounded(bar_empty + b, (uint32_t)(((s - 2) >> 1) & 1), lim);
                if (ok) ok = spin_until_ge(cf.ready + (size_t)j * RING + s % RING, (unsigned)(s + 1), lim);
                GDR_TL(true, s, 0);
                if (ok) {
                    fence_proxy_async_global();
                    mbar_arrive_expect_tx(bar_full + b, SLOT_BYTES);
                    for (uint32_t off = 0; off < SLOT_BYTES; off += 16384u) {
                        const uint32_t n = SLOT_BYTES - off < 16384u ? SLOT_BYTES - off : 16384u;
                        bulk_g2s(sb + (uint32_t)b * SLOT_BYTES + off, src + off, n, bar_full + b);
                    }
                    // V of this chunk, once the previous chunk's U^T MMA has read the V buffer
                    bool vok = vzero || s == 0 || mbar_wait_bounded(bar_u, (uint32_t)((s - 1) & 1), lim);
                    if (vok && !vzero) {
                        const int gx = head_of(s), t0 = tok0_of(s);
                        mbar_arrive_expect_tx(bar_v, 16384u);
                        tma_load_4d(sb + CH_V, &tm.v, 0, gx % p.H, t0, gx / p.H, bar_v);
                        tma_load_4d(sb + CH_V + 8192u, &tm.v, 64, gx % p.H, t0, gx / p.H, bar_v);
                        ++v_issued;
                    }
                    // the slot copy always lands before anything else happens
                    ok = mbar_wait_bounded(bar_full + b, (uint32_t)((s >> 1) & 1), lim) && vok;
                    GDR_TL(true, s, 1);
                }
                if (!ok) atomicExch(abort_f, 1);
            }
            // the decay vectors of the slot have been copied too (by the vector loader)
            if (lane == 0 && ok && !mbar_wait_bounded(bar_vec + (s & 3), (uint32_t)((s >> 2) & 1), lim)) {
                ok = false;
                atomicExch(abort_f, 1);
            }
            if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) break;
            // the slot's bytes are here: its L2 lines are dead, drop them without write-back
            if (cf.discard)
                for (uint32_t off = (uint32_t)lane * 128u; off < SLOT_BYTES; off += 32u * 128u) discard_l2_line(src + off);
            __syncwarp();
            if (lane == 0) st_release_gpu(cf.consumed + j, (unsigned)(s + 1));
        }
        // the last V copy lands before the CTA ends (its MMA may never have run)
        if (lane == 0 && v_issued > 0) (void)mbar_wait_bounded(bar_v, (uint32_t)((v_issued - 1) & 1), lim);
    } else if (warp == 2) {
        // ---------------- decay-vector loader: each chunk's P_m and P_m^{-1} P_C, as soon as its
        // slot is published, into a ring of 4 (the state pass of chunk s needs those of s + 1) --
        int* abort_f = ab + 4;
        if (lane == 0) {
            int issued = 0;
            for (int s = 0; s < nseq; ++s) {
                const int e = s & 3;
                if (s >= 4 && !mbar_wait_bounded(bar_vfree + e, (uint32_t)(((s - 4) >> 2) & 1), lim)) {
                    atomicExch(abort_f, 1);
                    break;
                }
                if (!spin_until_ge(cf.ready + (size_t)j * RING + s % RING, (unsigned)(s + 1), lim)) {
                    atomicExch(abort_f, 1);
                    break;
                }
                fence_proxy_async_global();
                mbar_arrive_expect_tx(bar_vec + e, 1024u);
                bulk_g2s(sb + CH_VEC + (uint32_t)e * 1024u,
                         cf.ring + ((size_t)j * RING + s % RING) * SLOT_BYTES + SL_VEC, 1024u, bar_vec + e);
                issued = s + 1;
            }
            // the last copies land before the CTA ends
            for (int s = issued > 4 ? issued - 4 : 0; s < issued; ++s)
                (void)mbar_wait_bounded(bar_vec + (s & 3), (uint32_t)((s >> 2) & 1), lim);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ------------------------------------------------------------
        if (lane == 0) {
            int* abort_f = ab + 1;
            auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
                if (mbar_wait_bounded(bar, parity, lim)) return true;
                atomicExch(abort_f, 1);
                return false;
            };
            const uint32_t ID_MK = idesc_bf16(128, 64, 1, 0, 0), ID_NEG = idesc_bf16(128, 64, 0, 1, 1);
            const uint32_t ID_KK = idesc_bf16(128, 64, 0, 0, 0);
            const uint32_t ID_T128 = idesc_tf32(128, 128), ID_T64 = idesc_tf32(128, 64);
            auto issue_u = [&](int s) {     // U^T = V^T Tw^T -> E^T buffer of chunk s
                const uint32_t sl = sb + (uint32_t)(s & 1) * SLOT_BYTES;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tbase + COL_E + (s & 1) * 64, sdesc_sw128(sb + CH_V + ks * 2048, 8192, 1024),
                                sdesc_sw128(sl + SL_T + ks * 32, 16, 1024), ID_MK, ks > 0);
                mma_commit(bar_u);
            };
            int u_issued = 0;
            for (int s = 0; s < nseq; ++s) {
                const int b = s & 1;
                const uint32_t sl = sb + (uint32_t)b * SLOT_BYTES;
                if (!vzero && u_issued <= s) {
                    if (!wait(bar_full + b, (uint32_t)((s >> 1) & 1)) || !wait(bar_v, (uint32_t)(s & 1))) break;
                    tc_fence_after();
                    issue_u(s);
                    u_issued = s + 1;
                }
                if (vzero && !wait(bar_full + b, (uint32_t)((s >> 1) & 1))) break;
                if (!wait(bar_sbr, (uint32_t)(s & 1))) break;
                GDR_TL(true, s, 2);
                tc_fence_after();
                const uint32_t a0 = tbase + COL_SB + b * 64;
                {   // E^T = U^T - Stil Wm^T (bf16, K = dk; E^T = -Stil Wm^T with zero values)
                    const uint64_t dW = sdesc_sw128(sl + SL_W, 8192, 1024);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16_ts(tbase + COL_E + b * 64, a0 + ks * 8, dW + (uint64_t)(ks * 2048 / 16), ID_NEG,
                                    (vzero && ks == 0) ? 0u : 1u);
                    mma_commit(bar_e);
                }
                if (!wait(bar_e, (uint32_t)(s & 1)) || !wait(bar_sf, (uint32_t)(s & 1))) break;
                GDR_TL(true, s, 3);
                tc_fence_after();
                {   // S_acc += E^T Khat (tf32: E^T read from TMEM as fp32, K = 64 tokens)
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_tf32_ts(tbase + COL_S, tbase + COL_E + b * 64 + ks * 8,
                                    sdesc_sw128(sl + SL_H + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024), ID_T128, 1);
                    mma_commit(bar_s);
                }
                // O^T = Stil Qtil^T (bf16) + E^T Pm^T (tf32)
                if (s >= 2 && !wait(bar_ofree + b, (uint32_t)(((s - 2) >> 1) & 1))) break;
                tc_fence_after();
                {
                    const uint64_t dQ = sdesc_sw128(sl + SL_Q, 16, 1024);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16_ts(tbase + COL_O + b * 64, a0 + ks * 8,
                                    dQ + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) / 16), ID_KK, ks > 0);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_tf32_ts(tbase + COL_O + b * 64, tbase + COL_E + b * 64 + ks * 8,
                                    sdesc_sw128(sl + SL_P + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), ID_T64, 1);
                    mma_commit(bar_o + b);
                }
                GDR_TL(true, s, 4);
                // the next chunk's U^T, if its slot and V are here
                if (!vzero && s + 1 < nseq && u_issued <= s + 1 &&
                    mbar_test_wait(bar_full + (b ^ 1), (uint32_t)(((s + 1) >> 1) & 1)) &&
                    mbar_test_wait(bar_v, (uint32_t)((s + 1) & 1))) {
                    tc_fence_after();
                    issue_u(s + 1);
                    u_issued = s + 2;
                }
            }
            // every MMA issued has completed before the CTA ends
            mma_commit(bar_dummy);
            (void)mbar_wait_bounded(bar_dummy, 0u, lim);
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------- o: O^T (TMEM) -> global ---------------------------------------------------
        // O^T sits in TMEM with lane = value row, column = token.  Each 8x8 block (8 value rows of
        // this warp x 8 tokens) is transposed across 8 lanes, so that every lane stores 8
        // consecutive value columns of one token (16 bytes in bf16, 32 in fp32).
        const int qd = warp & 3, row = qd * 32 + lane, et = tid - 128;
        const int j8 = lane & 7, grp = lane >> 3;
        const uint32_t tq = tbase + ((uint32_t)(qd * 32) << 16);
        int* abort_f = ab + 2;
        OT* __restrict__ o = static_cast<OT*>(p.o);
        const size_t tstride = (size_t)p.H * D;
        for (int s = 0; s < nseq; ++s) {
            const int b = s & 1, c = s % nchunks, gx = head_of(s), t0 = tok0_of(s);
            const int Lc = vh_chunk_len(p, geo, vh_of(s), c);
            if (et == 0 && !mbar_wait_bounded(bar_o + b, (uint32_t)((s >> 1) & 1), lim)) atomicExch(abort_f, 1);
            named_bar(4, 128);
            if (*abort_f) break;
            tc_fence_after();
            // every MMA that read slot buffer b has completed: it may be refilled
            if (et == 0) mbar_arrive(bar_empty + b);
            GDR_TL(et == 0, s, 7);
            OT* obase = o + tok_row(p, gx, t0) * D + qd * 32 + grp * 8;
            float msum = 0.f;
#pragma unroll 1
            for (int g = 0; g < 2; ++g) {
                float vals[32];
                tmem_ld32(tq + COL_O + b * 64 + g * 32, vals);
                if (cmean) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) msum += (g * 32 + u < Lc) ? vals[u] : 0.f;
                }
#pragma unroll
                for (int blk8 = 0; blk8 < 4; ++blk8) {
                    float v8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v8[e] = vals[blk8 * 8 + e];
                    transpose8(v8, j8);
                    const int r = g * 32 + blk8 * 8 + j8;
                    if (r < Lc && GDR_INB(gx < p.B * p.H && t0 + r < p.T, 109)) {
                        OT* dst = obase + (size_t)r * tstride;
                        if constexpr (sizeof(OT) == 2) {
                            *reinterpret_cast<uint4*>(dst) = pack8(v8);
                        } else {
                            reinterpret_cast<float4*>(dst)[0] = make_float4(v8[0], v8[1], v8[2], v8[3]);
                            reinterpret_cast<float4*>(dst)[1] = make_float4(v8[4], v8[5], v8[6], v8[7]);
                        }
                    }
                }
            }
            if (cmean && Lc > 0 && GDR_INB(gx < p.B * p.H && t0 < p.T, 110)) {    // the chunk index within the whole sequence
                const int nct = (p.T + C - 1) / C, cg = t0 / C;
                p.chunk_mean[(((size_t)(gx / p.H) * nct + cg) * p.H + gx % p.H) * D + row] = msum / (float)Lc;
            }
            tc_fence_before();
            named_bar(4, 128);
            if (et == 0) mbar_arrive(bar_ofree + b);    // O^T buffer b may be overwritten
            GDR_TL(et == 0, s, 8);
        }
    } else if (warp >= 8) {
        // ---------------- state: S_acc -> S_next -> the next chunk's prescaled state ------------------
        // Stil(s+1) = S_acc(s) (P_m^{-1} P_C)(s) P_m(s+1): its bf16 copy (the A operand of the next
        // chunk's first MMAs) is written and announced first, the fp32 accumulator after it.
        const int qd = warp & 3, hf = (warp - 8) >> 2, row = qd * 32 + lane;
        const bool lead = (tid == 256);
        int* abort_f = ab + 3;
        const int c0 = hf * 64;          // this thread's 64 key columns
        const uint32_t tq = tbase + ((uint32_t)(qd * 32) << 16);
        auto vecs = [&](int s) -> const float* {
            return reinterpret_cast<const float*>(base + CH_VEC + (uint32_t)(s & 3) * 1024u);
        };
        auto sbar = [&]() { named_bar(3, 256); };
        auto store_bf16 = [&](int s, const float (&v)[64]) {      // Stil_b of chunk s, columns c0..c0+63
            const uint32_t cb = tq + COL_SB + (s & 1) * 64 + (c0 >> 1);
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
                uint32_t w8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) w8[u] = pack_bf16x2(v[16 * q8 + 2 * u], v[16 * q8 + 2 * u + 1]);
                tmem_st8u(cb + 8 * q8, w8);
            }
        };
        auto store_f32 = [&](const float (&v)[64]) {
#pragma unroll
            for (int q16 = 0; q16 < 4; ++q16)
                tmem_st16(tq + COL_S + c0 + 16 * q16, *reinterpret_cast<const float(*)[16]>(v + 16 * q16));
        };
        auto announce = [&](uint64_t* bar) {     // TMEM stores of every state thread done -> bar
            tmem_wait_st();
            tc_fence_before();
            sbar();
            if (lead) mbar_arrive(bar);
        };
        // Stil of the first chunk of a (virtual) head: S0, zero or the identity, times P_m
        auto init_head = [&](int s, float (&v)[64]) {
            const float* pm = vecs(s);
            const int gx = head_of(s);
            const bool from_s0 = p.S0 != nullptr && !p.s0_identity && vh_seg(p, geo, vh_of(s)) == 0;
            if (p.s0_identity) {
#pragma unroll
                for (int u = 0; u < 64; ++u) v[u] = (c0 + u == row) ? 1.f : 0.f;
            } else if (from_s0 && GDR_INB(gx < p.B * p.H, 112)) {
                const float4* src = reinterpret_cast<const float4*>(p.S0 + ((size_t)gx * D + row) * D + c0);
#pragma unroll
                for (int u4 = 0; u4 < 16; ++u4) {
                    const float4 t4 = src[u4];
                    v[4 * u4] = t4.x; v[4 * u4 + 1] = t4.y; v[4 * u4 + 2] = t4.z; v[4 * u4 + 3] = t4.w;
                }
            } else {
#pragma unroll
                for (int u = 0; u < 64; ++u) v[u] = 0.f;
            }
            scale_cols<ROT, 64>(v, c0, pm);
        };
        bool alive = true;
        if (nseq > 0) {
            if (lead && !mbar_wait_bounded(bar_vec + 0, 0u, lim)) atomicExch(abort_f, 1);
            sbar();
            alive = *abort_f == 0;
            if (alive) {
                float v[64];
                init_head(0, v);
                store_bf16(0, v);
                announce(bar_sbr);
                store_f32(v);
                announce(bar_sf);
            }
        }
        for (int s = 0; s < nseq && alive; ++s) {
            const int c = s % nchunks;
            const bool last = (c == nchunks - 1);
            const bool more = s + 1 < nseq;
            if (lead) {
                if (!mbar_wait_bounded(bar_s, (uint32_t)(s & 1), lim)) atomicExch(abort_f, 1);
                if (more && !mbar_wait_bounded(bar_vec + ((s + 1) & 3), (uint32_t)(((s + 1) >> 2) & 1), lim))
                    atomicExch(abort_f, 1);
            }
            sbar();
            if (*abort_f) break;
            GDR_TL(lead, s, 5);
            tc_fence_after();
            const float* rc = vecs(s) + 128;        // P_m^{-1} P_C of chunk s
            float v[64];
            tmem_ld32x2(tq + COL_S + c0, tq + COL_S + c0 + 32, v);
            scale_cols<ROT, 64>(v, c0, rc);         // S(s+1), the plain state at the next chunk's start
            if (!last) {
                scale_cols<ROT, 64>(v, c0, vecs(s + 1));     // times P_m of chunk s + 1
                store_bf16(s + 1, v);
                announce(bar_sbr);
                store_f32(v);
                announce(bar_sf);
            } else {
                // S_T: one per head, or one per virtual head when segments run separately
                const int sx = p.nseg > 1 ? vh_of(s) : head_of(s);
                if (p.S_T && GDR_INB(sx < (p.nseg > 1 ? geo.nv : p.B * p.H), 111)) {
                    float4* dst = reinterpret_cast<float4*>(p.S_T + ((size_t)sx * D + row) * D + c0);
#pragma unroll
                    for (int u4 = 0; u4 < 16; ++u4)
                        dst[u4] = make_float4(v[4 * u4], v[4 * u4 + 1], v[4 * u4 + 2], v[4 * u4 + 3]);
                }
                if (more) {                           // the next (virtual) head of this chain
                    init_head(s + 1, v);
                    store_bf16(s + 1, v);
                    announce(bar_sbr);
                    store_f32(v);
                    announce(bar_sf);
                } else {
                    tc_fence_before();
                    sbar();
                }
            }
            if (lead) mbar_arrive(bar_vfree + (s & 3));     // the vectors of chunk s have been read
            GDR_TL(lead, s, 6);
        }
    }
}

// ======================================================================= kernel ====

template <bool ROT, typename OT, bool EXT>
__global__ void __launch_bounds__(NT, 1) split_fwd_kernel(FwdParams p, Cfg cf, const __grid_constant__ Maps tm) {
    using namespace tc;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (sb - raw_u32);
    const bool chain = (int)blockIdx.x < cf.nc;
    uint8_t* bar_base = base + (chain ? CH_BAR : WK_BAR);
    uint64_t* bars = reinterpret_cast<uint64_t*>(bar_base);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_base + 192);
    // Abort flags, one per role group, each set only by that group's leader before one of the
    // group's barriers (so that all of its warps leave at the same point): chain loader,
    // issuer, o, state; worker elementwise, solve.
    int* ab = reinterpret_cast<int*>(bar_base + 196);            // [6]
    int* range_f = reinterpret_cast<int*>(bar_base + 220);
    int* tk_ring = reinterpret_cast<int*>(bar_base + 224);       // [4] task of worker iteration it & 3
    static_assert(23 * 8 <= 192 && WB_COUNT * 8 <= 192, "barriers overlap the control words");
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t ncols = chain ? 512u : 256u;

    if (warp == 0) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    if (tid == 0) {
        // chain: full[2], v, u, e, s, o[2], sbr, ofree[2], empty[2], dummy, sf, vec[4], vfree[4];
        // worker: the WB_* barriers.  One arrival each.
        const int nb = chain ? 23 : WB_COUNT;
        for (int i = 0; i < nb; ++i) mbar_init(bars + i, 1u);
        fence_mbar_init();
        for (int i = 0; i < 6; ++i) ab[i] = 0;
        *range_f = 0;
        for (int i = 0; i < 4; ++i) tk_ring[i] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (p.T > 0) {
        if (chain) {
            chain_role<ROT, OT, EXT>(p, cf, tm, base, sb, tbase, bars, ab);
        } else if (tid < 256) {
            worker_elementwise<ROT, EXT>(p, cf, base, sb, tbase, bars, ab, range_f, tk_ring);
        } else if (tid == 256) {
            worker_producer<ROT>(p, cf, tm, sb, bars, ab + 2, tk_ring);
        } else if (tid == 288) {
            worker_publisher<EXT>(p, cf, sb, bars, ab + 3, tk_ring);
        } else if (tid >= 384) {
            worker_solve<EXT>(p, cf, base, sb, tbase, bars, ab + 1, tk_ring);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        unsigned bits = 0;
        if (ab[0] | ab[1] | ab[2] | ab[3] | ab[4] | ab[5]) bits |= STATUS_TIMEOUT;
        if (*range_f) bits |= STATUS_RANGE;
        if (bits) atomicOr(&g_device_status, bits);
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, ncols);
    }
}

}  // namespace spl
}  // namespace gdr
