// gdr.cu -- the C ABI declared in include/gdr.h: argument checks and kernel dispatch.
//
// All kernels are compiled into this one translation unit so that the device
// status word below is a single symbol per loaded module.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "gdr.h"
#include "common.cuh"
#include "simt_fwd.cuh"
#include "decode.cuh"
#include "tc_fwd.cuh"
#include "split_fwd.cuh"
#include "seg_combine.cuh"
#include "bwd.cuh"
#include "raven.cuh"

namespace gdr {

// Test hook state (gdr_debug_set_tc_fault): bound of every mbarrier wait in the
// tensor-core kernel, and whether its first MMA completion is never signalled.
static unsigned long long s_wait_limit_ns = 2000000000ull;
static int s_fault_skip_commit = 0;

static thread_local char t_detail[256] = "";

static gdr_status fail(gdr_status s, const char* fmt, const char* what = "") {
    snprintf(t_detail, sizeof(t_detail), fmt, what);
    return s;
}

static gdr_status cuda_fail(cudaError_t e, const char* where) {
    snprintf(t_detail, sizeof(t_detail), "%s: %s", where, cudaGetErrorString(e));
    return GDR_ERR_CUDA;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }
static bool dtype_ok(gdr_dtype t) { return t == GDR_F32 || t == GDR_BF16; }

// ---------------------------------------------------------------- forward ----

template <int DK, bool ROT, typename QT, typename OT>
static gdr_status launch_simt(const FwdParams& p, cudaStream_t st) {
    using L = simt::Smem<DK, ROT>;
    auto kern = simt::chunk_fwd_kernel<DK, ROT, QT, OT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(simt chunk kernel)");
    dim3 grid(p.B * p.H, p.dv / simt::DVT);
    kern<<<grid, simt::NT, L::bytes, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch(simt chunk kernel)");
    return GDR_OK;
}

template <int DK, bool ROT>
static gdr_status dispatch_simt_types(const gdr_fwd_desc* d, const FwdParams& p, cudaStream_t st) {
    const bool qb = d->qkv_dtype == GDR_BF16, ob = d->out_dtype == GDR_BF16;
    if (qb && ob) return launch_simt<DK, ROT, __nv_bfloat16, __nv_bfloat16>(p, st);
    if (qb && !ob) return launch_simt<DK, ROT, __nv_bfloat16, float>(p, st);
    if (!qb && ob) return launch_simt<DK, ROT, float, __nv_bfloat16>(p, st);
    return launch_simt<DK, ROT, float, float>(p, st);
}

template <bool ROT>
static gdr_status dispatch_simt_dk(const gdr_fwd_desc* d, const FwdParams& p, cudaStream_t st) {
    switch (d->dk) {
        case 32: return dispatch_simt_types<32, ROT>(d, p, st);
        case 64: return dispatch_simt_types<64, ROT>(d, p, st);
        default: return dispatch_simt_types<128, ROT>(d, p, st);
    }
}

static bool tc_supported(const gdr_fwd_desc* d) {
    return d->qkv_dtype == GDR_BF16 && d->dk == 128 && d->dv == 128 && d->chunk == 64;
}

static int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) { cudaGetLastError(); return 148; }
    return n;
}

// The split kernel runs the state chains on `nc` SMs and prepares chunks on the others; with
// more heads than chains, each chain runs its heads one after another (waves of nc heads).
// nc balances the two sides with a cost model measured on B200: a chain needs about
// CHAIN_CYCLES per chunk, a worker SM about WORKER_CYCLES per chunk of one head.
constexpr double CHAIN_CYCLES = 1500.0, WORKER_CYCLES = 2600.0;
static double split_cost(long long nv, long long nchunks, int nc, int sms) {
    const long long waves = (nv + nc - 1) / nc;
    const double t_chain = (double)waves * nchunks * CHAIN_CYCLES;
    const double t_work = (double)nv * nchunks * WORKER_CYCLES / (double)(sms - nc);
    return t_chain > t_work ? t_chain : t_work;
}
static int plan_chains(long long nv, long long nchunks, int sms) {
    if (nv <= 0 || nchunks <= 0) return 1;
    int best = 1;
    double best_t = 1e300;
    const int max_nc = (int)(nv < sms / 2 ? nv : sms / 2);
    for (int nc = 1; nc <= max_nc; ++nc) {
        const double t = split_cost(nv, nchunks, nc, sms);
        if (t < best_t * 0.999) { best_t = t; best = nc; }
    }
    return best;
}
// Virtual heads (chains) and chunks per virtual head of one split-kernel launch.
static void split_geometry(const FwdParams& p, long long* nv, long long* nchunks) {
    const long long ns = p.nseg > 1 ? p.nseg - p.seg0 : 1;
    *nv = (long long)p.nheads * ns;
    *nchunks = p.nseg > 1 ? p.seg_len / 64 : (p.T + 63) / 64;
}
// The split kernel (tcf, one chain CTA per head) shares the SMs without a chain among prep
// workers; with more than half of the SMs taken by chains, too few workers are left and the
// fused kernel (prep and chain of a head in one CTA) is faster.
static bool split_fits_heads(long long nh, int sms, int T) { return nh >= 1 && 2 * nh <= (long long)sms && T > 64; }
static bool split_fits(const gdr_fwd_desc* d, int sms) {
    return split_fits_heads((long long)d->B * d->H, sms, d->T);
}
// More heads than SMs: the fused kernel runs whole waves of SM-count heads; a last partial
// wave that would leave more than half of the SMs idle goes to the split kernel instead.
static long long waves_remainder(const gdr_fwd_desc* d, int sms) {
    const long long nh = (long long)d->B * d->H;
    return nh > sms ? nh % sms : 0;
}
static bool waves_fit(const gdr_fwd_desc* d, int sms) {
    const long long rem = waves_remainder(d, sms);
    return rem > 0 && split_fits_heads(rem, sms, d->T);
}
static bool segments_pay(long long nh, long long T, int sms);

// The algorithm a descriptor runs with.  AUTO: the CUDA-core kernel for shapes and dtypes the
// tensor-core kernels do not take; the fused kernel for a single chunk; the sequence-parallel
// form when its model puts it well ahead (few heads, long sequences); else the split kernel when
// the heads leave room for prep workers, the waves mix when a partial last wave would leave
// most SMs idle, the fused kernel otherwise.
static gdr_algo resolve_algo(const gdr_fwd_desc* d) {
    if (d->algo == GDR_ALGO_AUTO) {
        if (!tc_supported(d)) return GDR_ALGO_SIMT;
        const int sms = device_sm_count();
        if (d->T <= 64) return GDR_ALGO_TCGEN05;
        if (segments_pay((long long)d->B * d->H, d->T, sms)) return GDR_ALGO_TCGEN05_SEGMENTS;
        if (split_fits(d, sms)) return GDR_ALGO_TCGEN05_SPLIT;
        return waves_fit(d, sms) ? GDR_ALGO_TCGEN05_WAVES : GDR_ALGO_TCGEN05;
    }
    return d->algo;
}

static size_t split_workspace_heads(size_t nh) {
    return nh * tcf::RING * tcf::SLOT_BYTES + tcf::split_flag_words(nh) * sizeof(unsigned int);
}
static size_t split_workspace_bytes(const gdr_fwd_desc* d) { return split_workspace_heads((size_t)d->B * d->H); }
static size_t chains_workspace_bytes(const gdr_fwd_desc* d) {
    const long long nh = (long long)d->B * d->H;
    return spl::workspace_bytes((size_t)plan_chains(nh, (d->T + 63) / 64, device_sm_count()));
}

// ---- scratch for gdr_chunk_fwd_noalloc ---------------------------------------------------
// The split kernel's ring and flags for at most NOALLOC_MAX_HEADS heads, as a file-scope
// device array: every GPU that loads this library holds these bytes until the process exits.
constexpr int NOALLOC_MAX_HEADS = GDR_NOALLOC_MAX_HEADS;
constexpr size_t NOALLOC_BYTES =
    (size_t)NOALLOC_MAX_HEADS * tcf::RING * tcf::SLOT_BYTES +
    tcf::split_flag_words(NOALLOC_MAX_HEADS) * sizeof(unsigned int);
static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_BYTES];

// The current context's unique id (the driver's cuCtxGetId), so that per-device caches can
// tell a context that was destroyed and created again (cudaDeviceReset, a released primary
// context) from the one they were filled in: module globals and streams of the old context are
// gone with it.  The driver calls are looked up through the runtime so that the library does
// not link libcuda itself.  *id is 0 when no context is current on this thread.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static gdr_status current_ctx_id(unsigned long long* id) {
    static std::mutex mu;
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!get_current || !get_id) {
            void* p1 = nullptr;
            void* p2 = nullptr;
            cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
            cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1);
            if (e == cudaSuccess) e = cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetDriverEntryPoint(cuCtxGetCurrent / cuCtxGetId)");
            if (q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !p1 || !p2)
                return fail(GDR_ERR_CUDA, "the driver has no cuCtxGetCurrent / cuCtxGetId%s");
            get_current = reinterpret_cast<CtxGetCurrentFn>(p1);
            get_id = reinterpret_cast<CtxGetIdFn>(p2);
        }
    }
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return fail(GDR_ERR_CUDA, "cuCtxGetCurrent failed%s");
    *id = 0;
    if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return fail(GDR_ERR_CUDA, "cuCtxGetId failed%s");
    return GDR_OK;
}

// In host code g_noalloc_scratch names a host-side stand-in, not device memory.  Its device
// address is looked up with the device current (cudaGetSymbolAddress), once per device and
// context, and cached; a context that has been destroyed and created again is seen by its new
// id, and the address is looked up again.  The first call on a device (or in a new context)
// does the lookup, so it should come before any stream capture.
constexpr int NOALLOC_MAX_DEVICES = 64;
static void* s_noalloc_ptr[NOALLOC_MAX_DEVICES] = {};
static unsigned long long s_noalloc_ctx[NOALLOC_MAX_DEVICES] = {};
static std::mutex s_noalloc_mu;

static gdr_status noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return fail(GDR_ERR_UNSUPPORTED, "device index too large%s");
    unsigned long long ctx = 0;
    gdr_status s = current_ctx_id(&ctx);
    if (s != GDR_OK) return s;
    std::lock_guard<std::mutex> lock(s_noalloc_mu);
    if (!s_noalloc_ptr[dev] || ctx == 0 || s_noalloc_ctx[dev] != ctx) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
        // the lookup makes the device's primary context current if none was
        if (ctx == 0 && (s = current_ctx_id(&ctx)) != GDR_OK) return s;
        s_noalloc_ptr[dev] = ptr;
        s_noalloc_ctx[dev] = ctx;
    }
    *out = s_noalloc_ptr[dev];
    return GDR_OK;
}

static gdr_status check_fwd_desc(const gdr_fwd_desc* d) {
    if (!d) return fail(GDR_ERR_INVALID_ARG, "desc is NULL%s");
    if (d->B < 0 || d->H < 0 || d->T < 0) return fail(GDR_ERR_INVALID_ARG, "B, H, T must be >= 0%s");
    if (!head_dim_ok(d->dk) || !head_dim_ok(d->dv))
        return fail(GDR_ERR_UNSUPPORTED, "dk and dv must each be 32, 64 or 128%s");
    if (d->chunk != 64) return fail(GDR_ERR_UNSUPPORTED, "chunk must be 64%s");
    if (!dtype_ok(d->qkv_dtype) || !dtype_ok(d->out_dtype)) return fail(GDR_ERR_INVALID_ARG, "bad dtype%s");
    if (d->gate_mode != GDR_GATE_LOGDECAY && d->gate_mode != GDR_GATE_NEG_SOFTPLUS)
        return fail(GDR_ERR_INVALID_ARG, "bad gate_mode%s");
    if (d->rotation != 0 && d->rotation != 1) return fail(GDR_ERR_INVALID_ARG, "rotation must be 0 or 1%s");
    if (d->qk_l2norm != 0 && d->qk_l2norm != 1) return fail(GDR_ERR_INVALID_ARG, "qk_l2norm must be 0 or 1%s");
    if (d->algo != GDR_ALGO_AUTO && d->algo != GDR_ALGO_SIMT && d->algo != GDR_ALGO_TCGEN05 &&
        d->algo != GDR_ALGO_TCGEN05_SPLIT && d->algo != GDR_ALGO_TCGEN05_WAVES && d->algo != GDR_ALGO_TCGEN05_SEGMENTS &&
        d->algo != GDR_ALGO_TCGEN05_CHAINS)
        return fail(GDR_ERR_INVALID_ARG, "bad algo%s");
    if (d->segments < 0 || d->segments == 1 || d->segments > 4096)
        return fail(GDR_ERR_INVALID_ARG, "segments must be 0 (library's choice) or 2 .. 4096%s");
    if ((long long)d->B * d->H > 0x7fffffffLL) return fail(GDR_ERR_INVALID_ARG, "B*H too large%s");
    if ((d->algo == GDR_ALGO_TCGEN05 || d->algo == GDR_ALGO_TCGEN05_SPLIT || d->algo == GDR_ALGO_TCGEN05_WAVES ||
         d->algo == GDR_ALGO_TCGEN05_SEGMENTS || d->algo == GDR_ALGO_TCGEN05_CHAINS) &&
        !tc_supported(d))
        return fail(GDR_ERR_UNSUPPORTED, "the tcgen05 kernels need bf16 q/k/v and dk = dv = 128%s");
    return GDR_OK;
}

// ---- tensor maps of the split kernel ---------------------------------------------------
// cuTensorMapEncodeTiled is a driver call; it is looked up through the runtime so that the
// library does not link libcuda itself.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static gdr_status encode_fn(EncodeTiledFn* out) {
    static std::mutex mu;
    static EncodeTiledFn fn = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
        if (q != cudaDriverEntryPointSuccess || !ptr)
            return fail(GDR_ERR_CUDA, "the driver has no cuTensorMapEncodeTiled%s");
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    *out = fn;
    return GDR_OK;
}

// A [B][T][H][inner] row-major tensor as the 4-D map {inner, H, T, B}; boxes cover `box_inner`
// elements of one head for 64 consecutive tokens.  Out-of-range tokens read as zero and are
// not written by stores.
static gdr_status encode_bthd(EncodeTiledFn fn, CUtensorMap* m, const void* base, CUtensorMapDataType dt,
                              size_t esize, const FwdParams& p, int inner, int box_inner, bool swizzle128) {
    const cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)p.H, (cuuint64_t)p.T, (cuuint64_t)p.B};
    const cuuint64_t strides[3] = {(cuuint64_t)inner * esize, (cuuint64_t)p.H * inner * esize,
                                   (cuuint64_t)p.T * p.H * inner * esize};
    const cuuint32_t box[4] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)tcf::C, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(t_detail, sizeof(t_detail), "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return GDR_ERR_CUDA;
    }
    return GDR_OK;
}

template <bool ROT>
static gdr_status encode_split_maps(const FwdParams& p, spl::Maps* tm) {
    EncodeTiledFn fn = nullptr;
    gdr_status s = encode_fn(&fn);
    if (s != GDR_OK) return s;
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const int D = spl::D, NG = ROT ? spl::D / 2 : spl::D;
    if ((s = encode_bthd(fn, &tm->q, p.q, bf, 2, p, D, D, false)) != GDR_OK) return s;
    if ((s = encode_bthd(fn, &tm->k, p.k, bf, 2, p, D, D, false)) != GDR_OK) return s;
    if ((s = encode_bthd(fn, &tm->g, p.g, f32, 4, p, NG, NG, false)) != GDR_OK) return s;
    if (ROT && (s = encode_bthd(fn, &tm->th, p.theta, f32, 4, p, NG, NG, false)) != GDR_OK) return s;
    if (p.v && (s = encode_bthd(fn, &tm->v, p.v, bf, 2, p, D, 64, true)) != GDR_OK) return s;   // NULL: zero values
    return GDR_OK;
}

template <bool ROT, typename OT>
static gdr_status encode_tc_maps(const FwdParams& p, tcf::TmaMaps* tm) {
    EncodeTiledFn fn = nullptr;
    gdr_status s = encode_fn(&fn);
    if (s != GDR_OK) return s;
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const int D = tcf::D, NG = ROT ? tcf::D / 2 : tcf::D;
    if ((s = encode_bthd(fn, &tm->q, p.q, bf, 2, p, D, D, false)) != GDR_OK) return s;
    if ((s = encode_bthd(fn, &tm->k, p.k, bf, 2, p, D, D, false)) != GDR_OK) return s;
    if ((s = encode_bthd(fn, &tm->g, p.g, f32, 4, p, NG, NG, false)) != GDR_OK) return s;
    if (ROT && (s = encode_bthd(fn, &tm->th, p.theta, f32, 4, p, NG, NG, false)) != GDR_OK) return s;
    if ((s = encode_bthd(fn, &tm->v, p.v, bf, 2, p, D, 64, true)) != GDR_OK) return s;
    const bool ob = sizeof(OT) == 2;
    return encode_bthd(fn, &tm->o, p.o, ob ? bf : f32, sizeof(OT), p, D, D, false);
}

template <int MODE, bool ROT, typename OT, bool EXT>
static gdr_status launch_tc(const FwdParams& p, cudaStream_t st, void* ws) {
    auto kern = tcf::chunk_fwd_tc_kernel<MODE, ROT, OT, EXT>;
    constexpr int nt = tcf::nthreads<MODE>();
    constexpr uint32_t smem = tcf::smem_bytes<MODE>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tcgen05 chunk kernel)");
    tcf::TcExtra x;
    x.wait_limit_ns = s_wait_limit_ns;
    x.fault_skip_commit = s_fault_skip_commit;
    tcf::SplitArgs sa{nullptr, nullptr, nullptr};
    tcf::TmaMaps tm;
    memset(&tm, 0, sizeof(tm));
    if (MODE == 0) {
        kern<<<p.nheads, nt, smem, st>>>(p, x, sa, tm);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "launch(tcgen05 chunk kernel)");
        return GDR_OK;
    }
    // Split: the whole grid must be resident at once (one CTA per SM), which a cooperative
    // launch guarantees or refuses.
    const int nh = p.nheads;
    const int sms = device_sm_count();
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, nt, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    const int grid = sms * (per_sm < 1 ? 1 : per_sm > 1 ? 1 : per_sm);
    if (per_sm < 1 || grid <= nh) return fail(GDR_ERR_UNSUPPORTED, "split kernel: B*H must be below the SM count%s");
    gdr_status s = encode_tc_maps<ROT, OT>(p, &tm);
    if (s != GDR_OK) return s;
    const size_t nring = (size_t)nh * tcf::RING * tcf::SLOT_BYTES;
    sa.ring = static_cast<uint8_t*>(ws);
    sa.ready = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + nring);
    sa.consumed = sa.ready + (size_t)nh * tcf::RING;
    sa.next_task = sa.consumed + nh;
    // Worker order: from the counter while the worker groups fill at most half the ring's
    // slots (the workers are then the bound and the counter evens out their load); at a
    // fixed stride otherwise (measured faster there: it paces each group to the chains).
    sa.dynamic = (2 * (grid - nh) <= nh * tcf::RING / 2) ? 1 : 0;
    sa.discard = (reinterpret_cast<uintptr_t>(ws) & 127u) == 0 ? 1 : 0;
    e = cudaMemsetAsync(sa.ready, 0, tcf::split_flag_words(nh) * sizeof(unsigned int), st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(split flags)");
    void* args[] = {const_cast<FwdParams*>(&p), &x, &sa, &tm};
    e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(nt), args, smem, st);
    if (e != cudaSuccess) return cuda_fail(e, "cooperative launch(tcgen05 split kernel)");
    return GDR_OK;
}

template <int MODE>
static gdr_status dispatch_tc_mode(const gdr_fwd_desc* d, const FwdParams& p, cudaStream_t st, void* ws) {
    const bool ob = d->out_dtype == GDR_BF16;
    if (p.w || p.qk_norm || p.chunk_mean) {      // the kernel with the optional features
        if (d->rotation)
            return ob ? launch_tc<MODE, true, __nv_bfloat16, true>(p, st, ws) : launch_tc<MODE, true, float, true>(p, st, ws);
        return ob ? launch_tc<MODE, false, __nv_bfloat16, true>(p, st, ws) : launch_tc<MODE, false, float, true>(p, st, ws);
    }
    if (d->rotation)
        return ob ? launch_tc<MODE, true, __nv_bfloat16, false>(p, st, ws) : launch_tc<MODE, true, float, false>(p, st, ws);
    return ob ? launch_tc<MODE, false, __nv_bfloat16, false>(p, st, ws) : launch_tc<MODE, false, float, false>(p, st, ws);
}

template <bool ROT, typename OT, bool EXT>
static gdr_status launch_chains(const FwdParams& p, cudaStream_t st, void* ws) {
    auto kern = spl::split_fwd_kernel<ROT, OT, EXT>;
    constexpr uint32_t smem = spl::SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(split chunk kernel)");
    // The whole grid must be resident at once (one CTA per SM), which a cooperative launch
    // guarantees or refuses.
    long long nv = 0, nchunks = 0;
    split_geometry(p, &nv, &nchunks);
    const int sms = device_sm_count();
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, spl::NT, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (per_sm < 1) return fail(GDR_ERR_UNSUPPORTED, "split kernel: does not fit on an SM%s");
    const int grid = sms;
    const int nc = plan_chains(nv, nchunks, sms);
    if (nc < 1 || nc >= grid) return fail(GDR_ERR_UNSUPPORTED, "split kernel: no SM left for prep workers%s");
    spl::Maps tm;
    memset(&tm, 0, sizeof(tm));
    gdr_status s = encode_split_maps<ROT>(p, &tm);
    if (s != GDR_OK) return s;
    spl::Cfg cf;
    cf.ring = static_cast<uint8_t*>(ws);
    cf.ready = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + (size_t)nc * spl::RING * spl::SLOT_BYTES);
    cf.consumed = cf.ready + (size_t)nc * spl::RING;
    cf.next_task = cf.consumed + nc;
    cf.nc = nc;
    // Task order: from the counter while the prep workers are the bound (few chains, so a worker
    // that ran fast takes the next task); at a fixed stride otherwise, which paces each worker
    // to the chains.
    const long long waves = (nv + nc - 1) / nc;
    const double t_chain = (double)waves * nchunks * CHAIN_CYCLES;
    const double t_work = (double)nv * nchunks * WORKER_CYCLES / (double)(grid - nc);
    cf.dynamic = t_work >= t_chain ? 1 : 0;
    cf.wait_limit_ns = s_wait_limit_ns;
    cf.fault_skip_commit = s_fault_skip_commit;
    cf.discard = (reinterpret_cast<uintptr_t>(ws) & 127u) == 0 ? 1 : 0;
    e = cudaMemsetAsync(cf.ready, 0, spl::flag_words((size_t)nc) * sizeof(unsigned int), st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(split flags)");
    void* args[] = {const_cast<FwdParams*>(&p), &cf, &tm};
    e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(spl::NT), args, smem, st);
    if (e != cudaSuccess) return cuda_fail(e, "cooperative launch(split chunk kernel)");
    return GDR_OK;
}

static gdr_status dispatch_fused(const gdr_fwd_desc* d, const FwdParams& p, cudaStream_t st) {
    return dispatch_tc_mode<0>(d, p, st, nullptr);
}
static gdr_status dispatch_split(const gdr_fwd_desc* d, const FwdParams& p, cudaStream_t st, void* ws) {
    return dispatch_tc_mode<1>(d, p, st, ws);
}

// The chains kernel; f32_out writes o in fp32 whatever the descriptor's output dtype (the
// segments' second pass).  The instantiation with the optional features runs only when one of
// them is asked for.
static gdr_status dispatch_chains(const gdr_fwd_desc* d, const FwdParams& p, cudaStream_t st, void* ws,
                                  bool f32_out = false) {
    const bool ob = d->out_dtype == GDR_BF16 && !f32_out;
    if (p.w || p.qk_norm || p.chunk_mean) {
        if (d->rotation) return ob ? launch_chains<true, __nv_bfloat16, true>(p, st, ws) : launch_chains<true, float, true>(p, st, ws);
        return ob ? launch_chains<false, __nv_bfloat16, true>(p, st, ws) : launch_chains<false, float, true>(p, st, ws);
    }
    if (d->rotation) return ob ? launch_chains<true, __nv_bfloat16, false>(p, st, ws) : launch_chains<true, float, false>(p, st, ws);
    return ob ? launch_chains<false, __nv_bfloat16, false>(p, st, ws) : launch_chains<false, float, false>(p, st, ws);
}

// ---- sequence-parallel forward (segments) ---------------------------------------------------
// Each head's sequence is cut into nseg segments of seg_len tokens (a multiple of 64; the last
// one may be shorter).  Pass 1 runs every segment from the zero state (segment 0 from S0): o0
// into o, chunk means of o0, end states Bz.  Pass 2 runs segments 1.. from the identity with
// zero values: y_t = A_{start->t} q_t (fp32) and the transitions A.  The scan kernel forms the
// start states St of segments 1.. and S_T; the correction kernel adds St y to o (and to the
// chunk means).
struct SegPlan {
    int nseg = 1, seg_len = 0;
    size_t off_bz = 0, off_a = 0, off_st = 0, off_y = 0, total = 0;
};
constexpr double HBM_BYTES_PER_CYCLE = 3300.0;   // about 6.5 TB/s at 1.965 GHz
static double seg_cost(long long nh, long long T, int nseg, int sms) {
    const long long seg_len = ((T + nseg - 1) / nseg + 63) / 64 * 64;
    const long long ns = (T + seg_len - 1) / seg_len, sc = seg_len / 64;
    double t = split_cost(nh * ns, sc, plan_chains(nh * ns, sc, sms), sms);
    if (ns > 1) {
        t += split_cost(nh * (ns - 1), sc, plan_chains(nh * (ns - 1), sc, sms), sms);
        t += (double)(ns - 1) * 3000.0;                                                // scan steps
        t += (double)nh * T * (ns - 1) / ns * 1024.0 / HBM_BYTES_PER_CYCLE;           // y, o traffic
    }
    return t;
}
static int choose_segments(long long nh, long long T, int sms) {
    double best = 1e300;
    int bn = 2;
    for (int n = 2; n <= 64; n *= 2) {
        if (T < 128LL * n) break;
        const double t = seg_cost(nh, T, n, sms);
        if (t < best) { best = t; bn = n; }
    }
    return bn;
}
// AUTO takes the segments when the model puts them well ahead of one chain per head.
static bool segments_pay(long long nh, long long T, int sms) {
    if (T < 256) return false;
    const long long nchunks = (T + 63) / 64;
    const double t_plain = split_cost(nh, nchunks, plan_chains(nh, nchunks, sms), sms);
    return seg_cost(nh, T, choose_segments(nh, T, sms), sms) < 0.75 * t_plain;
}
static size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
static void seg_plan(const gdr_fwd_desc* d, int sms, SegPlan* P) {
    const long long nh = (long long)d->B * d->H, T = d->T;
    const int want = d->segments > 0 ? d->segments : choose_segments(nh, T, sms);
    const long long seg_len = ((T + want - 1) / want + 63) / 64 * 64;
    const long long ns = seg_len > 0 ? (T + seg_len - 1) / seg_len : 1, sc = seg_len / 64;
    P->nseg = (int)ns;
    P->seg_len = (int)seg_len;
    int nc = plan_chains(nh * ns, sc, sms);
    if (ns > 1) {
        const int nc2 = plan_chains(nh * (ns - 1), sc, sms);
        if (nc2 > nc) nc = nc2;
    }
    const size_t DD4 = (size_t)spl::D * spl::D * 4;
    size_t o = round256(spl::workspace_bytes((size_t)nc));
    P->off_bz = o;  o += round256((size_t)nh * ns * DD4);
    P->off_a = o;   o += round256((size_t)nh * (ns - 1) * DD4);
    P->off_st = o;  o += round256((size_t)nh * (ns - 1) * DD4);
    P->off_y = o;   o += round256(ns > 1 ? (size_t)d->B * T * d->H * spl::D * 4 : 0);
    P->total = o;
}

template <typename OT>
static gdr_status launch_correct(const seg::CorrParams& cp, const CUtensorMap& ymap, int nblocks, cudaStream_t st) {
    auto kern = seg::seg_correct_kernel<OT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)seg::CORR_SMEM);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(segment correction kernel)");
    kern<<<nblocks, seg::CORR_NT, seg::CORR_SMEM, st>>>(cp, ymap, s_wait_limit_ns);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch(segment correction kernel)");
    return GDR_OK;
}

static gdr_status run_segments(const gdr_fwd_desc* d, const FwdParams& p, cudaStream_t st, void* ws) {
    SegPlan P;
    seg_plan(d, device_sm_count(), &P);
    uint8_t* w = static_cast<uint8_t*>(ws);
    FwdParams p1 = p;
    if (P.nseg <= 1) return dispatch_chains(d, p1, st, ws);
    float* Bz = reinterpret_cast<float*>(w + P.off_bz);
    float* A = reinterpret_cast<float*>(w + P.off_a);
    float* St = reinterpret_cast<float*>(w + P.off_st);
    float* y = reinterpret_cast<float*>(w + P.off_y);
    p1.nseg = P.nseg; p1.seg_len = P.seg_len; p1.seg0 = 0; p1.s0_identity = 0;
    p1.S_T = Bz;
    gdr_status s = dispatch_chains(d, p1, st, w);                  // o0, chunk means of o0, Bz
    if (s != GDR_OK) return s;
    FwdParams p2 = p1;
    p2.seg0 = 1; p2.s0_identity = 1;
    p2.v = nullptr; p2.w = nullptr; p2.S0 = nullptr; p2.chunk_mean = nullptr;
    p2.o = y; p2.S_T = A;
    s = dispatch_chains(d, p2, st, w, true);                       // y (fp32), A
    if (s != GDR_OK) return s;
    seg::ScanParams sp{p.nheads, P.nseg, Bz, A, St, p.S_T};
    cudaError_t e = cudaFuncSetAttribute(seg::seg_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)seg::SCAN_SMEM);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(segment scan kernel)");
    seg::seg_scan_kernel<<<dim3(p.nheads, seg::D / seg::RB), seg::SCAN_NT, seg::SCAN_SMEM, st>>>(sp);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "launch(segment scan kernel)");
    EncodeTiledFn fn = nullptr;
    if ((s = encode_fn(&fn)) != GDR_OK) return s;
    CUtensorMap ymap;
    memset(&ymap, 0, sizeof(ymap));
    if ((s = encode_bthd(fn, &ymap, y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p, spl::D, 32, true)) != GDR_OK) return s;
    seg::CorrParams cp{p.B, p.H, p.T, P.nseg, P.seg_len, p.head0, St, p.o, p.chunk_mean};
    const int nblocks = p.nheads * (P.nseg - 1) * (P.seg_len / seg::TOK);
    return d->out_dtype == GDR_BF16 ? launch_correct<__nv_bfloat16>(cp, ymap, nblocks, st)
                                    : launch_correct<float>(cp, ymap, nblocks, st);
}

// ----------------------------------------------------------------- decode ----

template <int DK, bool ROT, typename QT, typename OT>
static gdr_status launch_decode(const dec::DecParams& p, cudaStream_t st) {
    // persistent: at most CTAS_PER_SM CTAs per SM, each warp walking 16-row work items
    const long long items = (long long)p.N * p.H * (p.dv / dec::RI);
    if (items > 0x7fffffffLL) return fail(GDR_ERR_INVALID_ARG, "N*H too large%s");
    const long long need = (items + dec::WARPS - 1) / dec::WARPS;
    const long long cap = (long long)device_sm_count() * dec::CTAS_PER_SM;
    const long long grid = need < cap ? need : cap;
    if (grid <= 0) return GDR_OK;
    dec::decode_kernel<DK, ROT, QT, OT><<<(unsigned)grid, dec::WARPS * 32, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch(decode kernel)");
    return GDR_OK;
}

template <int DK, bool ROT>
static gdr_status decode_types(const gdr_dec_desc* d, const dec::DecParams& p, cudaStream_t st) {
    const bool qb = d->qkv_dtype == GDR_BF16, ob = d->out_dtype == GDR_BF16;
    if (qb && ob) return launch_decode<DK, ROT, __nv_bfloat16, __nv_bfloat16>(p, st);
    if (qb && !ob) return launch_decode<DK, ROT, __nv_bfloat16, float>(p, st);
    if (!qb && ob) return launch_decode<DK, ROT, float, __nv_bfloat16>(p, st);
    return launch_decode<DK, ROT, float, float>(p, st);
}

// ---- host-buffer forward: batch slices through two device slots ----------------------------
// gdr_chunk_fwd_host copies slice i's inputs into slot i % 2 on one copy stream, runs the
// forward of that slice on the caller's stream and copies its outputs back on a second copy
// stream, so the copies of neighbouring slices overlap each other and the compute.  The
// streams and events are created once per device and kept for the life of the process.
constexpr int HOST_MAX_DEVICES = 64;
constexpr int HOST_MAX_SLICES = 8;
struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr;
    cudaEvent_t loaded[2] = {}, computed[2] = {}, stored[2] = {};
    bool ready = false;
    unsigned long long ctx = 0;     // the context they were created in
};
static HostPipe s_pipe[HOST_MAX_DEVICES];
static std::mutex s_pipe_mu;     // held while a call enqueues: the events are shared

static gdr_status host_pipe(HostPipe** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= HOST_MAX_DEVICES) return fail(GDR_ERR_UNSUPPORTED, "device index out of range%s");
    HostPipe& P = s_pipe[dev];
    unsigned long long ctx = 0;
    gdr_status s = current_ctx_id(&ctx);
    if (s != GDR_OK) return s;
    // Streams and events of a context that has since been destroyed are gone with it (and
    // cannot be destroyed again); a new context gets new ones.
    if (P.ready && ctx != 0 && P.ctx != ctx) P = HostPipe();
    if (!P.ready) {
        if ((e = cudaStreamCreateWithFlags(&P.h2d, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaStreamCreateWithFlags(&P.d2h, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaEventCreateWithFlags(&P.start, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "host pipeline streams");
        for (int i = 0; i < 2; ++i) {
            if ((e = cudaEventCreateWithFlags(&P.loaded[i], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&P.computed[i], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&P.stored[i], cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(e, "host pipeline events");
        }
        if (ctx == 0 && (s = current_ctx_id(&ctx)) != GDR_OK) return s;
        P.ctx = ctx;
        P.ready = true;
    }
    *out = &P;
    return GDR_OK;
}

// Bytes per batch entry of each tensor of the forward, in the order of HostTensor.
enum HostTensor { HT_Q, HT_K, HT_V, HT_G, HT_BETA, HT_W, HT_THETA, HT_S0, HT_O, HT_ST, HT_CM, HT_COUNT };
struct HostPlan {
    size_t per_b[HT_COUNT];   // bytes of one batch entry (0: tensor absent)
    size_t off[HT_COUNT];     // offset in a slot (256-byte aligned)
    size_t slot_bytes;
    size_t ring_bytes;        // split-kernel workspace at the start, rounded to 256
    int bs, nslices;          // batch entries per slice, number of slices
};

static void host_plan(const gdr_fwd_desc* d, bool w, bool S0, bool S_T, bool cm, HostPlan* P) {
    const size_t T = (size_t)d->T, H = (size_t)d->H, dk = (size_t)d->dk, dv = (size_t)d->dv;
    const size_t si = d->qkv_dtype == GDR_BF16 ? 2 : 4, so = d->out_dtype == GDR_BF16 ? 2 : 4;
    const size_t ng = d->rotation ? dk / 2 : dk, nc = (T + 63) / 64;
    P->per_b[HT_Q] = T * H * dk * si;
    P->per_b[HT_K] = T * H * dk * si;
    P->per_b[HT_V] = T * H * dv * si;
    P->per_b[HT_G] = T * H * ng * 4;
    P->per_b[HT_BETA] = T * H * 4;
    P->per_b[HT_W] = w ? T * H * 4 : 0;
    P->per_b[HT_THETA] = d->rotation ? T * H * (dk / 2) * 4 : 0;
    P->per_b[HT_S0] = S0 ? H * dv * dk * 4 : 0;
    P->per_b[HT_O] = T * H * dv * so;
    P->per_b[HT_ST] = S_T ? H * dv * dk * 4 : 0;
    P->per_b[HT_CM] = cm ? nc * H * dv * 4 : 0;
    const int B = d->B > 0 ? d->B : 1;
    const int ns = B < HOST_MAX_SLICES ? B : HOST_MAX_SLICES;
    P->bs = (B + ns - 1) / ns;
    P->nslices = (B + P->bs - 1) / P->bs;
    size_t o = 0;
    for (int t = 0; t < HT_COUNT; ++t) {
        P->off[t] = o;
        o += round256(P->per_b[t] * (size_t)P->bs);
    }
    P->slot_bytes = o;
    // the slices have bs entries, the last one possibly fewer: the larger workspace of the two
    gdr_fwd_desc sd = *d;
    sd.B = P->bs;
    size_t ring = gdr_chunk_fwd_workspace_bytes(&sd);
    sd.B = B - (P->nslices - 1) * P->bs;
    const size_t ring_last = gdr_chunk_fwd_workspace_bytes(&sd);
    P->ring_bytes = round256(ring > ring_last ? ring : ring_last);
}

// ---- backward ------------------------------------------------------------------------------
static gdr_status check_bwd_desc(const gdr_fwd_desc* d) {
    gdr_status s = check_fwd_desc(d);
    if (s != GDR_OK) return s;
    if (d->dk != d->dv) return fail(GDR_ERR_UNSUPPORTED, "the backward needs dk = dv%s");
    return GDR_OK;
}

// Backward workspace (floats): the chunk coefficients (3 per chunk), the chunk start states and
// end-state gradients (1 each per chunk), and one scratch region per CTA of the two parallel
// passes (one CTA per SM).
static size_t bwd_scratch_floats(int d) {
    switch (d) {
        case 32: return bwd::Lay<32, 32>::floats();
        case 64: return bwd::Lay<64, 64>::floats();
        default: return bwd::Lay<128, 128>::floats();
    }
}
static int bwd_grid(long long nh, int T) {
    const long long tasks = nh * ((T + 63) / 64), sms = device_sm_count();
    return (int)(tasks < sms ? tasks : sms);
}
static size_t bwd_workspace_floats(const gdr_fwd_desc* d) {
    const size_t nh = (size_t)d->B * d->H, nc = (size_t)(d->T + 63) / 64, dd = (size_t)d->dk * d->dv;
    return nh * nc * 5 * dd + (size_t)bwd_grid((long long)nh, d->T) * bwd_scratch_floats(d->dk);
}

template <typename K>
static gdr_status launch_bwd_kernel(K kern, int grid, size_t smem, const bwd::BwdParams& p, cudaStream_t st,
                                   const char* what) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(backward kernel)");
    kern<<<(unsigned)grid, bwd::NT, smem, st>>>(p);
    e = cudaGetLastError();
    return e == cudaSuccess ? GDR_OK : cuda_fail(e, what);
}

template <int D, typename QT, typename OT>
static gdr_status launch_bwd(const bwd::BwdParams& p, int nh, cudaStream_t st) {
    const int grid = bwd_grid(nh, p.T);
    gdr_status s = launch_bwd_kernel(bwd::bwd_coef_kernel<D, D, QT, OT>, grid, bwd::SMEM_BYTES, p, st,
                                     "launch(backward coefficients)");
    if (s != GDR_OK) return s;
    if constexpr (D == 128)    // the chains on tcgen05 (tf32, three-way split)
        s = launch_bwd_kernel(bwd::bwd_chain_tc_kernel, nh, bwd::TC_SMEM_BYTES, p, st, "launch(backward chains)");
    else
        s = launch_bwd_kernel(bwd::bwd_chain_kernel<D>, nh, bwd::chain_smem_bytes<D>(), p, st, "launch(backward chains)");
    if (s != GDR_OK) return s;
    return launch_bwd_kernel(bwd::bwd_grad_kernel<D, D, QT, OT>, grid, bwd::SMEM_BYTES, p, st,
                             "launch(backward gradients)");
}

template <int D>
static gdr_status dispatch_bwd_d(const gdr_fwd_desc* d, const bwd::BwdParams& p, cudaStream_t st) {
    const int nh = d->B * d->H;
    const bool qb = d->qkv_dtype == GDR_BF16, ob = d->out_dtype == GDR_BF16;
    if (qb && ob) return launch_bwd<D, __nv_bfloat16, __nv_bfloat16>(p, nh, st);
    if (qb) return launch_bwd<D, __nv_bfloat16, float>(p, nh, st);
    if (ob) return launch_bwd<D, float, __nv_bfloat16>(p, nh, st);
    return launch_bwd<D, float, float>(p, nh, st);
}

// ---- Raven (routed slot memory) ------------------------------------------------------------
static gdr_status check_raven_desc(const gdr_raven_desc* d) {
    if (!d) return fail(GDR_ERR_INVALID_ARG, "descriptor is NULL%s");
    if (d->B < 0 || d->H < 0 || d->T < 0) return fail(GDR_ERR_INVALID_ARG, "B, H, T must be >= 0%s");
    if (d->d != 64 && d->d != 128) return fail(GDR_ERR_UNSUPPORTED, "Raven head dim must be 64 or 128%s");
    if (d->slots != rvn::M) return fail(GDR_ERR_UNSUPPORTED, "Raven needs 64 slots%s");
    if (d->topk < 1 || d->topk > rvn::KMAX) return fail(GDR_ERR_INVALID_ARG, "topk must be in 1..16%s");
    if (d->qkv_dtype != GDR_BF16) return fail(GDR_ERR_UNSUPPORTED, "Raven takes bf16 q, k, v%s");
    if (!dtype_ok(d->out_dtype)) return fail(GDR_ERR_INVALID_ARG, "bad out dtype%s");
    if (d->gate_mode != GDR_GATE_LOGDECAY && d->gate_mode != GDR_GATE_NEG_SOFTPLUS)
        return fail(GDR_ERR_INVALID_ARG, "bad gate mode%s");
    if (d->segments < 0) return fail(GDR_ERR_INVALID_ARG, "segments must be >= 0%s");
    return GDR_OK;
}

// Segments per sequence: enough CTAs to cover the SMs, at least 8 chunks per segment, unless
// the caller fixes the number.
static void raven_plan(const gdr_raven_desc* d, int* nseg, int* seg_chunks) {
    const int nc = (d->T + rvn::C - 1) / rvn::C;
    const long long nh = (long long)d->B * d->H;
    long long want = d->segments;
    if (want <= 0) {
        want = nh > 0 ? device_sm_count() / nh : 1;
        if (want > nc / 8) want = nc / 8;
    }
    if (want < 1) want = 1;
    if (want > nc) want = nc > 0 ? nc : 1;
    const int per = nc > 0 ? (int)((nc + want - 1) / want) : 1;
    *seg_chunks = per;
    *nseg = nc > 0 ? (nc + per - 1) / per : 1;
}

// State units of the state pass: the chunks before the last segment, in units of a divisor of
// the segment length, halved while a unit keeps at least the length that gives about two waves
// of state CTAs (and at least 4 chunks).
static void raven_units(const gdr_raven_desc* d, int nseg, int seg_chunks, int* nsub, int* sub_chunks) {
    if (nseg <= 1) {
        *nsub = 0;
        *sub_chunks = seg_chunks;
        return;
    }
    const long long nh = (long long)d->B * d->H;
    long long want = (2LL * device_sm_count() + nh - 1) / nh;          // units per sequence
    if (want < nseg - 1) want = nseg - 1;
    const long long target = ((long long)(nseg - 1) * seg_chunks + want - 1) / want;
    int sub = seg_chunks;
    while (sub % 2 == 0 && sub / 2 >= target && sub / 2 >= 4) sub /= 2;
    *sub_chunks = sub;
    *nsub = (nseg - 1) * (seg_chunks / sub);
}

// Workspace: every token's routing record (rounded up to 256 bytes), then the state units.
static size_t raven_route_bytes(const gdr_raven_desc* d) {
    return ((size_t)d->B * d->T * d->H * rvn::ROUTE_BYTES + 255) / 256 * 256;
}
static size_t raven_workspace_bytes_(const gdr_raven_desc* d) {
    int nseg, per, nsub, sub;
    raven_plan(d, &nseg, &per);
    raven_units(d, nseg, per, &nsub, &sub);
    const size_t nh = (size_t)d->B * d->H;
    return raven_route_bytes(d) + nh * (size_t)nsub * (2 * (size_t)rvn::M * d->d + rvn::M) * sizeof(float);
}

template <int D, bool FULL, typename OT>
static gdr_status launch_raven_kernel(const rvn::RavenParams& p, int grid, cudaStream_t st) {
    auto kern = rvn::raven_fwd_kernel<D, FULL, OT>;
    const size_t smem = rvn::Sm<D>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(raven kernel)");
    kern<<<(unsigned)grid, rvn::NT, smem, st>>>(p);
    e = cudaGetLastError();
    return e == cudaSuccess ? GDR_OK : cuda_fail(e, FULL ? "launch(raven outputs)" : "launch(raven segment states)");
}

template <int D, typename OT>
static gdr_status launch_raven(const rvn::RavenParams& p, cudaStream_t st) {
    const int nh = p.B * p.H;
    {   // the router, one warp per (token, head)
        const long long n_tok = (long long)p.B * p.T * p.H;
        const long long blocks = (n_tok + 7) / 8, cap = (long long)device_sm_count() * 8;
        rvn::raven_route_kernel<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, st>>>(p);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "launch(raven router)");
    }
    if (p.nsub > 0) {
        const gdr_status s = launch_raven_kernel<D, false, OT>(p, nh * p.nsub, st);
        if (s != GDR_OK) return s;
    }
    return launch_raven_kernel<D, true, OT>(p, nh * p.nseg, st);
}

}  // namespace gdr

using namespace gdr;

extern "C" {

int gdr_abi_version(void) { return GDR_ABI_VERSION; }

const char* gdr_status_string(gdr_status s) {
    switch (s) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT";
        case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE";
        case GDR_ERR_RANGE: return "GDR_ERR_RANGE";
        case GDR_ERR_BOUNDS: return "GDR_ERR_BOUNDS";
    }
    return "GDR_ERR_UNKNOWN";
}

const char* gdr_last_error_detail(void) { return t_detail; }

size_t gdr_chunk_fwd_workspace_bytes(const gdr_fwd_desc* desc) {
    if (check_fwd_desc(desc) != GDR_OK) return 0;
    const gdr_algo a = resolve_algo(desc);
    if (a == GDR_ALGO_TCGEN05_SPLIT) return split_workspace_bytes(desc);
    if (a == GDR_ALGO_TCGEN05_CHAINS) return desc->T > 64 ? chains_workspace_bytes(desc) : 0;
    if (a == GDR_ALGO_TCGEN05_SEGMENTS) {
        if (desc->T <= 0) return 0;
        SegPlan P;
        seg_plan(desc, device_sm_count(), &P);
        return P.total;
    }
    if (a == GDR_ALGO_TCGEN05_WAVES) {
        // only a last partial wave that the split kernel runs needs the ring
        const int sms = device_sm_count();
        const long long rem = waves_remainder(desc, sms);
        return (rem > 0 && split_fits_heads(rem, sms, desc->T)) ? split_workspace_heads((size_t)rem) : 0;
    }
    return 0;
}

gdr_status gdr_chunk_fwd(const gdr_fwd_desc* d, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const float* theta, const float* S0,
                         void* o, float* S_T, void* workspace, size_t workspace_bytes,
                         gdr_stream_t stream) {
    return gdr_chunk_fwd_untied(d, q, k, v, g, beta, nullptr, theta, S0, o, S_T, workspace, workspace_bytes,
                                stream);
}

gdr_status gdr_chunk_fwd_untied(const gdr_fwd_desc* d, const void* q, const void* k, const void* v,
                                const float* g, const float* beta, const float* w, const float* theta,
                                const float* S0, void* o, float* S_T, void* workspace,
                                size_t workspace_bytes, gdr_stream_t stream) {
    return gdr_chunk_fwd_ex(d, q, k, v, g, beta, w, theta, S0, o, S_T, nullptr, workspace, workspace_bytes,
                            stream);
}

gdr_status gdr_chunk_fwd_ex(const gdr_fwd_desc* d, const void* q, const void* k, const void* v,
                            const float* g, const float* beta, const float* w, const float* theta,
                            const float* S0, void* o, float* S_T, float* chunk_mean, void* workspace,
                            size_t workspace_bytes, gdr_stream_t stream) {
    t_detail[0] = 0;
    gdr_status s = check_fwd_desc(d);
    if (s != GDR_OK) return s;
    if (d->B == 0 || d->H == 0) return GDR_OK;
    if (d->T > 0) {
        if (!q || !k || !v || !g || !beta || !o) return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta and o are required%s");
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) || !aligned16(o))
            return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned%s");
        if (d->rotation && !theta) return fail(GDR_ERR_INVALID_ARG, "theta is required with rotation%s");
    }
    if (!d->rotation && theta) return fail(GDR_ERR_INVALID_ARG, "theta must be NULL without rotation%s");
    if ((theta && !aligned16(theta)) || (S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)) ||
        (w && !aligned16(w)) || (chunk_mean && !aligned16(chunk_mean)))
        return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned%s");
    const size_t need = gdr_chunk_fwd_workspace_bytes(d);
    if (need > 0 && (!workspace || workspace_bytes < need)) return fail(GDR_ERR_WORKSPACE, "workspace too small%s");

    FwdParams p;
    p.B = d->B; p.H = d->H; p.T = d->T; p.dv = d->dv;
    p.head0 = 0; p.nheads = d->B * d->H;
    p.qk_norm = d->qk_l2norm;
    p.gate_mode = (int)d->gate_mode;
    p.scale = d->scale;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.w = w; p.theta = theta;
    p.S0 = S0; p.o = o; p.S_T = S_T; p.chunk_mean = chunk_mean;
    p.nseg = 1; p.seg_len = 0; p.seg0 = 0; p.s0_identity = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (d->T == 0 && !S_T) return GDR_OK;
    const gdr_algo algo = resolve_algo(d);
    if (algo == GDR_ALGO_TCGEN05_SPLIT && d->T > 0) {
        if (!aligned16(workspace)) return fail(GDR_ERR_INVALID_ARG, "workspace must be 16-byte aligned%s");
        return dispatch_split(d, p, st, workspace);
    }
    if (algo == GDR_ALGO_TCGEN05_CHAINS && d->T > 64) {
        if (!aligned16(workspace)) return fail(GDR_ERR_INVALID_ARG, "workspace must be 16-byte aligned%s");
        return dispatch_chains(d, p, st, workspace);
    }
    if (algo == GDR_ALGO_TCGEN05_SEGMENTS && d->T > 0) {
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return fail(GDR_ERR_INVALID_ARG, "workspace must be 256-byte aligned for GDR_ALGO_TCGEN05_SEGMENTS%s");
        return run_segments(d, p, st, workspace);
    }
    if (algo == GDR_ALGO_TCGEN05_WAVES && d->T > 0) {
        const long long rem = waves_remainder(d, device_sm_count());
        if (rem > 0 && split_fits_heads(rem, device_sm_count(), d->T)) {
            if (!aligned16(workspace)) return fail(GDR_ERR_INVALID_ARG, "workspace must be 16-byte aligned%s");
            FwdParams pf = p, ps = p;
            pf.nheads = (int)(p.nheads - rem);
            ps.head0 = pf.nheads;
            ps.nheads = (int)rem;
            s = dispatch_fused(d, pf, st);                    // whole waves, fused
            if (s != GDR_OK) return s;
            return dispatch_split(d, ps, st, workspace);      // the last partial wave, split
        }
        return dispatch_fused(d, p, st);
    }
    if (algo == GDR_ALGO_TCGEN05 || algo == GDR_ALGO_TCGEN05_SPLIT || algo == GDR_ALGO_TCGEN05_WAVES ||
        algo == GDR_ALGO_TCGEN05_SEGMENTS || algo == GDR_ALGO_TCGEN05_CHAINS)
        return dispatch_fused(d, p, st);
    return d->rotation ? dispatch_simt_dk<true>(d, p, st) : dispatch_simt_dk<false>(d, p, st);
}

gdr_status gdr_decode_step(const gdr_dec_desc* d, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, const float* theta, float* S,
                           void* o, gdr_stream_t stream) {
    return gdr_decode_step_untied(d, q, k, v, g, beta, nullptr, theta, S, o, stream);
}

gdr_status gdr_decode_step_untied(const gdr_dec_desc* d, const void* q, const void* k, const void* v,
                                  const float* g, const float* beta, const float* w, const float* theta,
                                  float* S, void* o, gdr_stream_t stream) {
    t_detail[0] = 0;
    if (!d) return fail(GDR_ERR_INVALID_ARG, "desc is NULL%s");
    if (d->N < 0 || d->H < 0) return fail(GDR_ERR_INVALID_ARG, "N, H must be >= 0%s");
    if (!head_dim_ok(d->dk) || !head_dim_ok(d->dv))
        return fail(GDR_ERR_UNSUPPORTED, "dk and dv must each be 32, 64 or 128%s");
    if (!dtype_ok(d->qkv_dtype) || !dtype_ok(d->out_dtype)) return fail(GDR_ERR_INVALID_ARG, "bad dtype%s");
    if (d->gate_mode != GDR_GATE_LOGDECAY && d->gate_mode != GDR_GATE_NEG_SOFTPLUS)
        return fail(GDR_ERR_INVALID_ARG, "bad gate_mode%s");
    if (d->rotation != 0 && d->rotation != 1) return fail(GDR_ERR_INVALID_ARG, "rotation must be 0 or 1%s");
    if (d->qk_l2norm != 0 && d->qk_l2norm != 1) return fail(GDR_ERR_INVALID_ARG, "qk_l2norm must be 0 or 1%s");
    if (d->N == 0 || d->H == 0) return GDR_OK;
    if (!q || !k || !v || !g || !beta || !S || !o) return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta, S and o are required%s");
    if (d->rotation && !theta) return fail(GDR_ERR_INVALID_ARG, "theta is required with rotation%s");
    if (!d->rotation && theta) return fail(GDR_ERR_INVALID_ARG, "theta must be NULL without rotation%s");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) ||
        !aligned16(S) || !aligned16(o) || (theta && !aligned16(theta)) || (w && !aligned16(w)))
        return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned%s");
    dec::DecParams p;
    p.N = d->N; p.H = d->H; p.dv = d->dv;
    p.gate_mode = (int)d->gate_mode;
    p.scale = d->scale;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.w = w; p.theta = theta; p.S = S; p.o = o;
    p.qk_norm = d->qk_l2norm;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (d->rotation) {
        switch (d->dk) {
            case 32: return decode_types<32, true>(d, p, st);
            case 64: return decode_types<64, true>(d, p, st);
            default: return decode_types<128, true>(d, p, st);
        }
    }
    switch (d->dk) {
        case 32: return decode_types<32, false>(d, p, st);
        case 64: return decode_types<64, false>(d, p, st);
        default: return decode_types<128, false>(d, p, st);
    }
}

gdr_status gdr_query_device_status(gdr_stream_t stream) {
    t_detail[0] = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int word = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&word, g_device_status, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(status)");
    if (word != 0) {
        e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol(status)");
        snprintf(t_detail, sizeof(t_detail), "device status word 0x%08x", word);
        if (word & tcf::STATUS_TIMEOUT) return GDR_ERR_TIMEOUT;
        return (word & STATUS_BOUNDS) ? GDR_ERR_BOUNDS : GDR_ERR_RANGE;
    }
    return GDR_OK;
}

int gdr_debug_bounds_site(void) {
#ifdef GDR_BOUNDS_CHECK
    unsigned int site = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&site, g_bounds_site, sizeof(site)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_bounds_site, &zero, sizeof(zero)) != cudaSuccess) {
        cudaGetLastError();
        return -2;
    }
    return (int)site;
#else
    return -1;
#endif
}

int gdr_chunk_fwd_algo(const gdr_fwd_desc* desc) {
    if (check_fwd_desc(desc) != GDR_OK) return -1;
    return (int)resolve_algo(desc);
}

int gdr_chunk_fwd_kernel_launches(const gdr_fwd_desc* d) {
    if (check_fwd_desc(d) != GDR_OK) return -1;
    if (d->B == 0 || d->H == 0) return 0;
    const gdr_algo a = resolve_algo(d);
    if (d->T == 0) return 1;
    if (a == GDR_ALGO_TCGEN05_SEGMENTS) {
        SegPlan P;
        seg_plan(d, device_sm_count(), &P);
        return P.nseg <= 1 ? 1 : 4;         // two split passes, the scan, the correction
    }
    if (a == GDR_ALGO_TCGEN05_WAVES) {
        const int sms = device_sm_count();
        const long long rem = waves_remainder(d, sms);
        return (rem > 0 && split_fits_heads(rem, sms, d->T)) ? 2 : 1;
    }
    return 1;
}

size_t gdr_chunk_bwd_workspace_bytes(const gdr_fwd_desc* d) {
    if (check_bwd_desc(d) != GDR_OK) return 0;
    if (d->B == 0 || d->H == 0 || d->T == 0) return 0;
    return bwd_workspace_floats(d) * sizeof(float);
}

gdr_status gdr_chunk_bwd(const gdr_fwd_desc* d, const void* q, const void* k, const void* v, const float* g,
                         const float* beta, const float* w, const float* theta, const float* S0, const void* dO,
                         const float* dS_T, float* dq, float* dk, float* dv, float* dg, float* dbeta, float* dw,
                         float* dtheta, float* dS0, void* workspace, size_t workspace_bytes, gdr_stream_t stream) {
    t_detail[0] = 0;
    gdr_status s = check_bwd_desc(d);
    if (s != GDR_OK) return s;
    if (d->B == 0 || d->H == 0) return GDR_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t sbytes = (size_t)d->B * d->H * d->dv * d->dk * sizeof(float);
    if (d->T == 0) {    // no tokens: the gradient of S0 is that of S_T
        if (!dS0) return GDR_OK;
        if (!aligned16(dS0) || (dS_T && !aligned16(dS_T))) return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned%s");
        const cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, sbytes, cudaMemcpyDeviceToDevice, st)
                                   : cudaMemsetAsync(dS0, 0, sbytes, st);
        return e == cudaSuccess ? GDR_OK : cuda_fail(e, "copy(dS0)");
    }
    if (!q || !k || !v || !g || !beta || !dq || !dk || !dv || !dg || !dbeta)
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta, dq, dk, dv, dg and dbeta are required%s");
    if ((w == nullptr) != (dw == nullptr)) return fail(GDR_ERR_INVALID_ARG, "dw is required exactly when w is given%s");
    if (d->rotation ? (!theta || !dtheta) : (theta || dtheta))
        return fail(GDR_ERR_INVALID_ARG, "theta and dtheta are required exactly with rotation%s");
    const void* ptrs[] = {q, k, v, g, beta, w, theta, S0, dO, dS_T, dq, dk, dv, dg, dbeta, dw, dtheta, dS0, workspace};
    for (const void* x : ptrs)
        if (x && !aligned16(x)) return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned%s");
    const size_t need = gdr_chunk_bwd_workspace_bytes(d);
    if (!workspace || workspace_bytes < need) return fail(GDR_ERR_WORKSPACE, "workspace too small%s");
    bwd::BwdParams p;
    p.B = d->B; p.H = d->H; p.T = d->T; p.gate_mode = (int)d->gate_mode; p.scale = d->scale;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.w = w; p.theta = theta; p.S0 = S0; p.dO = dO; p.dS_T = dS_T;
    p.dq = dq; p.dk = dk; p.dv = dv; p.dg = dg; p.dbeta = dbeta; p.dw = dw; p.dS0 = dS0; p.dtheta = dtheta;
    p.rot = d->rotation ? 1 : 0;
    p.norm = d->qk_l2norm ? 1 : 0;
    {
        const size_t nh = (size_t)d->B * d->H, nc = (size_t)(d->T + 63) / 64, dd = (size_t)d->dk * d->dv;
        float* w = static_cast<float*>(workspace);
        p.coef = w;
        p.ckpt = p.coef + nh * nc * 3 * dd;
        p.dsl = p.ckpt + nh * nc * dd;
        p.scratch = p.dsl + nh * nc * dd;
        p.scratch_floats = bwd_scratch_floats(d->dk);
    }
    switch (d->dk) {
        case 32: return dispatch_bwd_d<32>(d, p, st);
        case 64: return dispatch_bwd_d<64>(d, p, st);
        default: return dispatch_bwd_d<128>(d, p, st);
    }
}

int gdr_raven_fwd_segments(const gdr_raven_desc* d) {
    if (check_raven_desc(d) != GDR_OK) return -1;
    int nseg, per;
    raven_plan(d, &nseg, &per);
    return nseg;
}

size_t gdr_raven_fwd_workspace_bytes(const gdr_raven_desc* d) {
    if (check_raven_desc(d) != GDR_OK) return 0;
    if (d->B == 0 || d->H == 0 || d->T == 0) return 0;
    return raven_workspace_bytes_(d);
}

gdr_status gdr_raven_fwd(const gdr_raven_desc* d, const void* q, const void* k, const void* v, const float* z,
                         const float* g, const float* S0k, const float* S0v, void* o, float* Sk_T, float* Sv_T,
                         void* workspace, size_t workspace_bytes, gdr_stream_t stream) {
    t_detail[0] = 0;
    gdr_status s = check_raven_desc(d);
    if (s != GDR_OK) return s;
    if (d->B == 0 || d->H == 0) return GDR_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const void* ptrs[] = {q, k, v, z, g, S0k, S0v, o, Sk_T, Sv_T, workspace};
    for (const void* x : ptrs)
        if (x && !aligned16(x)) return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned%s");
    const size_t sbytes = (size_t)d->B * d->H * rvn::M * d->d * sizeof(float);
    if (d->T == 0) {    // no tokens: the final states are the initial ones
        float* outs[2] = {Sk_T, Sv_T};
        const float* ins[2] = {S0k, S0v};
        for (int j = 0; j < 2; ++j) {
            if (!outs[j]) continue;
            const cudaError_t e = ins[j] ? cudaMemcpyAsync(outs[j], ins[j], sbytes, cudaMemcpyDeviceToDevice, st)
                                         : cudaMemsetAsync(outs[j], 0, sbytes, st);
            if (e != cudaSuccess) return cuda_fail(e, "copy(S_T)");
        }
        return GDR_OK;
    }
    if (!q || !k || !v || !z || !g || !o) return fail(GDR_ERR_INVALID_ARG, "q, k, v, z, g and o are required%s");
    const size_t need = gdr_raven_fwd_workspace_bytes(d);
    if (!workspace || workspace_bytes < need) return fail(GDR_ERR_WORKSPACE, "workspace too small%s");
    rvn::RavenParams p;
    p.B = d->B; p.H = d->H; p.T = d->T; p.K = d->topk; p.gate_mode = (int)d->gate_mode; p.scale = d->scale;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.z = z; p.g = g; p.S0k = S0k; p.S0v = S0v; p.o = o; p.SkT = Sk_T; p.SvT = Sv_T;
    raven_plan(d, &p.nseg, &p.seg_chunks);
    raven_units(d, p.nseg, p.seg_chunks, &p.nsub, &p.sub_chunks);
    p.route = static_cast<unsigned char*>(workspace);
    p.segW = reinterpret_cast<float*>(p.route + raven_route_bytes(d));
    p.segL = p.nsub > 0 ? p.segW + (size_t)d->B * d->H * p.nsub * 2 * rvn::M * d->d : nullptr;
    const bool ob = d->out_dtype == GDR_BF16;
    if (d->d == 64) return ob ? launch_raven<64, __nv_bfloat16>(p, st) : launch_raven<64, float>(p, st);
    return ob ? launch_raven<128, __nv_bfloat16>(p, st) : launch_raven<128, float>(p, st);
}

gdr_status gdr_chunk_fwd_noalloc(const gdr_fwd_desc* d, const void* q, const void* k, const void* v,
                                 const float* g, const float* beta, const float* theta, const float* S0,
                                 void* o, float* S_T, gdr_stream_t stream) {
    t_detail[0] = 0;
    gdr_status s = check_fwd_desc(d);
    if (s != GDR_OK) return s;
    if (d->algo != GDR_ALGO_AUTO && d->algo != GDR_ALGO_TCGEN05_SPLIT)
        return fail(GDR_ERR_INVALID_ARG, "gdr_chunk_fwd_noalloc runs the split tensor-core kernel: algo must be AUTO or TCGEN05_SPLIT%s");
    if (!tc_supported(d))
        return fail(GDR_ERR_UNSUPPORTED, "gdr_chunk_fwd_noalloc needs bf16 q/k/v and dk = dv = 128%s");
    if ((long long)d->B * d->H > NOALLOC_MAX_HEADS) {
        snprintf(t_detail, sizeof(t_detail),
                 "gdr_chunk_fwd_noalloc: B*H = %lld exceeds the built-in scratch limit of %d heads; "
                 "use gdr_chunk_fwd with a caller workspace", (long long)d->B * d->H, NOALLOC_MAX_HEADS);
        return GDR_ERR_UNSUPPORTED;
    }
    if (d->B == 0 || d->H == 0) return GDR_OK;
    if (d->T > 0) {
        if (!q || !k || !v || !g || !beta || !o) return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta and o are required%s");
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) || !aligned16(o))
            return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned%s");
        if (d->rotation && !theta) return fail(GDR_ERR_INVALID_ARG, "theta is required with rotation%s");
    }
    if (!d->rotation && theta) return fail(GDR_ERR_INVALID_ARG, "theta must be NULL without rotation%s");
    if ((theta && !aligned16(theta)) || (S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)))
        return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned%s");
    FwdParams p;
    p.B = d->B; p.H = d->H; p.T = d->T; p.dv = d->dv;
    p.head0 = 0; p.nheads = d->B * d->H;
    p.qk_norm = d->qk_l2norm;
    p.gate_mode = (int)d->gate_mode;
    p.scale = d->scale;
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.w = nullptr; p.theta = theta;
    p.S0 = S0; p.o = o; p.S_T = S_T; p.chunk_mean = nullptr;
    p.nseg = 1; p.seg_len = 0; p.seg0 = 0; p.s0_identity = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (d->T == 0) return S_T ? dispatch_fused(d, p, st) : GDR_OK;
    void* scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != GDR_OK) return s;
    return dispatch_split(d, p, st, scratch);
}

size_t gdr_chunk_fwd_host_workspace_bytes(const gdr_fwd_desc* d, int with_w, int with_S0, int with_S_T,
                                          int with_chunk_mean) {
    if (check_fwd_desc(d) != GDR_OK || d->B == 0 || d->H == 0) return 0;
    HostPlan P;
    host_plan(d, with_w != 0, with_S0 != 0, with_S_T != 0, with_chunk_mean != 0, &P);
    return P.ring_bytes + 2 * P.slot_bytes;
}

gdr_status gdr_chunk_fwd_host(const gdr_fwd_desc* d, const void* q, const void* k, const void* v,
                              const float* g, const float* beta, const float* w, const float* theta,
                              const float* S0, void* o, float* S_T, float* chunk_mean, void* workspace,
                              size_t workspace_bytes, gdr_stream_t stream) {
    t_detail[0] = 0;
    gdr_status s = check_fwd_desc(d);
    if (s != GDR_OK) return s;
    if (d->B == 0 || d->H == 0) return GDR_OK;
    if (d->T > 0 && (!q || !k || !v || !g || !beta || !o))
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta and o are required%s");
    if (d->T > 0 && d->rotation && !theta) return fail(GDR_ERR_INVALID_ARG, "theta is required with rotation%s");
    if (!d->rotation && theta) return fail(GDR_ERR_INVALID_ARG, "theta must be NULL without rotation%s");
    HostPlan P;
    host_plan(d, w != nullptr, S0 != nullptr, S_T != nullptr, chunk_mean != nullptr, &P);
    if (!workspace || workspace_bytes < P.ring_bytes + 2 * P.slot_bytes)
        return fail(GDR_ERR_WORKSPACE, "workspace too small (gdr_chunk_fwd_host_workspace_bytes)%s");
    if (!aligned16(workspace)) return fail(GDR_ERR_INVALID_ARG, "workspace must be 16-byte aligned%s");
    const void* host_in[HT_COUNT] = {q, k, v, g, beta, w, theta, S0, nullptr, nullptr, nullptr};
    void* host_out[HT_COUNT] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                o, S_T, chunk_mean};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);

    std::lock_guard<std::mutex> lock(s_pipe_mu);
    HostPipe* pp = nullptr;
    s = host_pipe(&pp);
    if (s != GDR_OK) return s;
    HostPipe& H = *pp;
    cudaError_t e;
    // On an error after copies were queued, the caller's stream still waits for the copy
    // streams, so that host buffers are not released while a copy may still read or write them.
    auto bail = [&](gdr_status err) -> gdr_status {
        if (cudaEventRecord(H.loaded[0], H.h2d) == cudaSuccess) (void)cudaStreamWaitEvent(st, H.loaded[0], 0);
        if (cudaEventRecord(H.stored[0], H.d2h) == cudaSuccess) (void)cudaStreamWaitEvent(st, H.stored[0], 0);
        return err;
    };
    // the copy streams start after the work already on the caller's stream
    if ((e = cudaEventRecord(H.start, st)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = cudaStreamWaitEvent(H.h2d, H.start, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(H.d2h, H.start, 0)) != cudaSuccess)
        return cuda_fail(e, "cudaStreamWaitEvent");
    for (int i = 0; i < P.nslices; ++i) {
        const int j = i & 1;
        const size_t b0 = (size_t)i * P.bs;
        const int nb = (int)((size_t)d->B - b0 < (size_t)P.bs ? (size_t)d->B - b0 : (size_t)P.bs);
        uint8_t* slot = ws + P.ring_bytes + (size_t)j * P.slot_bytes;
        void* dptr[HT_COUNT];
        for (int t = 0; t < HT_COUNT; ++t) dptr[t] = P.per_b[t] ? slot + P.off[t] : nullptr;
        // inputs of slice i into slot j, once the slice two back has finished reading them
        if (i >= 2 && (e = cudaStreamWaitEvent(H.h2d, H.computed[j], 0)) != cudaSuccess)
            return bail(cuda_fail(e, "cudaStreamWaitEvent"));
        for (int t = HT_Q; t <= HT_S0; ++t) {
            const size_t n = P.per_b[t] * (size_t)nb;
            if (n == 0 || !host_in[t]) continue;
            e = cudaMemcpyAsync(dptr[t], static_cast<const uint8_t*>(host_in[t]) + P.per_b[t] * b0, n,
                                cudaMemcpyHostToDevice, H.h2d);
            if (e != cudaSuccess) return bail(cuda_fail(e, "cudaMemcpyAsync (host to device)"));
        }
        if ((e = cudaEventRecord(H.loaded[j], H.h2d)) != cudaSuccess) return bail(cuda_fail(e, "cudaEventRecord"));
        // the forward of slice i on the caller's stream; its outputs overwrite slot j's, so it
        // also waits for the slice two back to have been copied out
        if ((e = cudaStreamWaitEvent(st, H.loaded[j], 0)) != cudaSuccess)
            return bail(cuda_fail(e, "cudaStreamWaitEvent"));
        if (i >= 2 && (e = cudaStreamWaitEvent(st, H.stored[j], 0)) != cudaSuccess)
            return bail(cuda_fail(e, "cudaStreamWaitEvent"));
        gdr_fwd_desc sd = *d;
        sd.B = nb;
        s = gdr_chunk_fwd_ex(&sd, dptr[HT_Q], dptr[HT_K], dptr[HT_V], static_cast<const float*>(dptr[HT_G]),
                             static_cast<const float*>(dptr[HT_BETA]), static_cast<const float*>(dptr[HT_W]),
                             static_cast<const float*>(dptr[HT_THETA]), static_cast<const float*>(dptr[HT_S0]),
                             dptr[HT_O], static_cast<float*>(dptr[HT_ST]), static_cast<float*>(dptr[HT_CM]),
                             P.ring_bytes ? ws : nullptr, P.ring_bytes, stream);
        if (s != GDR_OK) return bail(s);
        if ((e = cudaEventRecord(H.computed[j], st)) != cudaSuccess) return bail(cuda_fail(e, "cudaEventRecord"));
        // outputs of slice i back to the host
        if ((e = cudaStreamWaitEvent(H.d2h, H.computed[j], 0)) != cudaSuccess)
            return bail(cuda_fail(e, "cudaStreamWaitEvent"));
        for (int t = HT_O; t <= HT_CM; ++t) {
            const size_t n = P.per_b[t] * (size_t)nb;
            if (n == 0 || !host_out[t]) continue;
            e = cudaMemcpyAsync(static_cast<uint8_t*>(host_out[t]) + P.per_b[t] * b0, dptr[t], n,
                                cudaMemcpyDeviceToHost, H.d2h);
            if (e != cudaSuccess) return bail(cuda_fail(e, "cudaMemcpyAsync (device to host)"));
        }
        if ((e = cudaEventRecord(H.stored[j], H.d2h)) != cudaSuccess) return bail(cuda_fail(e, "cudaEventRecord"));
    }
    // the caller's stream completes once every output is in host memory
    if ((e = cudaStreamWaitEvent(st, H.stored[(P.nslices - 1) & 1], 0)) != cudaSuccess)
        return bail(cuda_fail(e, "cudaStreamWaitEvent"));
    return GDR_OK;
}

#ifdef GDR_TIMELINE
// Profiling builds only: copy the split kernel's event timeline to host memory (see split_fwd.cuh).
GDR_API int gdr_debug_timeline(unsigned long long* host, size_t n) {
    return cudaMemcpyFromSymbol(host, g_timeline, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : -1;
}
GDR_API int gdr_debug_timeline_clear(void) {
    static unsigned long long zero[148 * TL_ITERS * TL_EVENTS];
    return cudaMemcpyToSymbol(g_timeline, zero, sizeof(zero)) == cudaSuccess ? 0 : -1;
}
#endif

void gdr_debug_set_tc_fault(int skip_first_commit, unsigned long long wait_limit_ns) {
    s_fault_skip_commit = skip_first_commit ? 1 : 0;
    s_wait_limit_ns = wait_limit_ns ? wait_limit_ns : 2000000000ull;
}

}  // extern "C"
