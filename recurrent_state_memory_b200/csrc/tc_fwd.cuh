// tc_fwd.cuh -- chunk-WY forward on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// The WY/UT-transform triangular chunk solver ("CARVE" page, section 1 item 3 and
// section 3 item 1; "Semidirect Fourier Delta Attention" page, "Constructive Chunk-WY
// Theorem" and the exact affine chunk transfer), bf16 operands, fp32 accumulation,
// dk = dv = 128, chunk C = 64.  One CTA owns the state chain of one (batch, head); the state
// S (dv x dk, fp32) stays resident in tensor memory for the whole sequence.
//
// Per chunk, with P_r = D_1 ... D_r and the reference token m = 31 (the middle of the
// chunk), every decay factor is split around P_m so that no factor exceeds the decay
// of half a chunk:
//   Ktil_r = (P_m^{-1} P_r) k_r,  Qtil_r = (P_m^{-1} P_r) q_r,  Khat_i = (P_i^{-1} P_m)^T k_i
//   [A' ; Pmat] = [Ktil ; Qtil] Khat^T                              (MMA1, 128 x 64 x 128)
//   Tm = (I + diag(beta) strict_lower(A'))^{-1},  Tb = Tm diag(beta) (fp32 blocked solve)
//   U^T = V^T Tb^T,   Wm^T = Ktil^T Tb^T                            (MMA, 128 x 64 x 64)
//   Stil = S P_m                                                    (prescaled state)
//   E^T = U^T - Stil Wm^T,   O^T = Stil Qtil^T                      (MMA, 128 x 64 x 128)
//   O^T += E^T Pm^T,   S_acc = Stil + E^T Khat                      (MMA, K = 64)
//   S <- S_acc (P_m^{-1} P_C)
// A tail chunk is padded with identity tokens (g = 0, beta = 0, k = q = v = 0).
// The split kernel (MODE 1) evaluates the same chunk with the reference decay folded into the
// operands its chain reads (Qtil2 = Qtil P_m^T, Ktil2 = Ktil P_m^T, Khat2 = Khat P_m^{-1} P_C),
// so its chain keeps the plain state:
//   Wm2^T = Ktil2^T Tb^T,  E^T = U^T - S Wm2^T,  O^T = S Qtil2^T + E^T Pm^T,  S <- S P_C + E^T Khat2.
//
// Warp roles of the fused kernel (384 threads):
//   warps 0-7  "prep": gate activation and decay factors (register-prefetched inputs),
//              the operand tiles, MMA1, the triangular solve, U^T / Wm^T.  They run up
//              to two chunks ahead of the chain, through double-buffered tiles.
//   warps 8-11 "chain": one thread per TMEM lane (value row of S); issue the state MMAs,
//              convert E^T to bf16 in TMEM, rescale S, write o and S_T.
// Hand-offs use mbarriers in pairs indexed by chunk parity (full: prep -> chain,
// empty: chain -> prep), so no barrier ever runs two phases ahead of its waiter.
// Every mbarrier wait is bounded; a group that gives up stops at a point where all of
// its warps agree, and the other group then gives up on its own bounded waits.
//
// Tensor memory (512 columns, lane = row):
//   [0,128) S fp32 | [128,192) Stil bf16 (A operand) | [192,320) O^T x 2 |
//   [320,448) U^T -> E^T x 2 (fp32, then bf16 in the first 32 columns) | [448,512) A'/Wm^T
// Shared-memory tiles use the 128-byte swizzle; K-major tiles have rows of 128 B along K,
// MN-major tiles rows of 128 B along M/N; the K-major Khat tile doubles as the MN-major
// B operand of the state update.
#pragma once

#include <cuda.h>   // CUtensorMap

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdr {
namespace tcf {

constexpr int C = 64;
constexpr int D = 128;           // dk = dv
constexpr int NT = 384;
constexpr int NPREP = 256;       // threads of a prep group
constexpr int CHAIN_THREADS = 128;   // threads of the chain group (one per TMEM lane)
constexpr uint32_t COL_S = 0, COL_SB = 128, COL_O = 192, COL_E = 320, COL_AW = 448;
constexpr uint32_t TMEM_COLS = 512;

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_KQ = 0;                       // [Ktil ; Qtil] K-major, x2: 2 kblocks x 128 rows x 128 B
constexpr uint32_t OFF_KH = OFF_KQ + 2 * 32768;      // Khat K-major, x2: 2 kblocks x 64 rows x 128 B
constexpr uint32_t OFF_W = OFF_KH + 2 * 16384;       // Wm^T bf16 MN-major, x2: 128 dk rows x 128 B
constexpr uint32_t OFF_PM = OFF_W + 2 * 16384;       // Pm K-major, x2: 64 rows x 128 B
constexpr uint32_t OFF_V = OFF_PM + 2 * 8192;        // V, MN-major for V^T: 2 groups x 64 tokens x 128 B
constexpr uint32_t OFF_TB = OFF_V + 16384;           // Tb K-major: 64 rows x 128 B
constexpr int AS = 68;                               // row stride (floats) of the fp32 solve matrices
constexpr uint32_t OFF_AF = OFF_TB + 8192;           // fp32 A [64][68]
constexpr uint32_t OFF_TF = OFF_AF + 64 * AS * 4;    // fp32 Tm [64][68]
constexpr uint32_t OFF_QT = OFF_TF + 64 * AS * 4;    // segment products [8 segments][32 dim groups][8]
constexpr uint32_t VEC_FLOATS = 64 + 4 * 128 + 64;   // beta[64], rho_ref[2][128], rho_C[2][128], w[64]
constexpr uint32_t VEC_W = 64 + 4 * 128;             // offset of the write strengths in a vector block
constexpr uint32_t OFF_VEC = OFF_QT + 8 * 32 * 8 * 4;   // x2
constexpr uint32_t OFF_BAR = (OFF_VEC + 2 * VEC_FLOATS * 4 + 63) & ~63u;
constexpr uint32_t BAR_BYTES = 256;                  // mbarriers, TMEM address, flags
// Tw = Tm diag(w) K-major, for a write strength w separate from the erase strength beta
constexpr uint32_t OFF_TW = (OFF_BAR + BAR_BYTES + 1023) & ~1023u;
// per-token inverse L2 norms of k and q (fused L2-normalisation only): [64][2] fp32
constexpr uint32_t OFF_NRM = OFF_TW + 8192;

// Split mode: a per-head ring in global memory carries each chunk's operands from the prep
// workers to the chain CTA.  Slot layout (bytes), identical to the chain's shared-memory copy:
constexpr uint32_t SL_Q = 0;          // Qtil K-major: 2 kblocks x 64 rows x 128 B
constexpr uint32_t SL_KH = 16384;     // Khat K-major: 2 kblocks x 64 rows x 128 B
constexpr uint32_t SL_W = 32768;      // Ktil2 (2 kblocks x 64 rows x 128 B); in the chain CTA then
                                      // Wm2^T bf16 MN-major (128 dk rows x 128 B)
constexpr uint32_t SL_PM = 49152;     // Pm K-major: 64 rows x 128 B
constexpr uint32_t SL_TB = 57344;     // Tb K-major: 64 rows x 128 B
constexpr uint32_t SL_TW = 65536;     // Tw K-major (only with a separate write strength)
constexpr uint32_t SL_VEC = 73728;    // beta, P_C, ... (VEC_FLOATS floats)
constexpr uint32_t SLOT_BYTES = SL_VEC + VEC_FLOATS * 4;        // bytes of one ring slot
// The chain CTA's copy of a slot is followed by the chunk's V tile, which the chain loads
// itself from the input (MN-major: 2 groups x 64 tokens x 128 B).
constexpr uint32_t SL_V = (SLOT_BYTES + 1023) & ~1023u;
constexpr uint32_t SLOT_STRIDE = SL_V + 16384;                  // slot buffers in the chain CTA
constexpr int RING = 8;               // ring slots per head
// Split chain CTAs stage each chunk's o here ([64 tokens][128] in the output type) and
// store it with one tensor-map tile store.
constexpr uint32_t OFF_OSTG = 2 * SLOT_STRIDE;
// Split-mode prep workers run two independent groups of 8 warps, each with its own tiles
// (bytes from the group's base, group g at g * G_STRIDE).  A group stages the raw inputs of
// its next task into tiles that the current task no longer needs: q into G_KH and the gates
// (and angles) into G_KQ once MMA1 has read them, k into G_AF once the solve is done.
constexpr uint32_t G_KQ = 0;         // [Ktil ; Qtil] K-major: 2 kblocks x 128 rows x 128 B
constexpr uint32_t G_KH = 32768;     // Khat K-major: 2 kblocks x 64 rows x 128 B
constexpr uint32_t G_TB = 49152;     // Tb K-major: 64 rows x 128 B
constexpr uint32_t G_QT = 57344;     // segment products [8][32][8]
constexpr uint32_t G_TW = 65536;     // Tw K-major (separate write strength only)
constexpr uint32_t G_AF = 73728;     // fp32 A [64][68]
constexpr uint32_t G_TF = G_AF + 64 * AS * 4;   // fp32 Tm [64][68]
constexpr uint32_t G_VEC = G_TF + 64 * AS * 4;  // beta, rho_ref, rho_C
constexpr uint32_t G_NRM = G_VEC + VEC_FLOATS * 4;   // inverse L2 norms [64][2] fp32
constexpr uint32_t G_STRIDE = (G_NRM + 512 + 1023) & ~1023u;
constexpr int NT_SPLIT = 2 * NPREP;             // two prep groups (16 warps: 128 registers a thread)
constexpr uint32_t OFF_BAR_SPLIT = 2 * G_STRIDE;
static_assert(2 * SLOT_STRIDE + 64 * 128 * 4 <= OFF_BAR_SPLIT, "chain slot buffers overlap the barriers");
static_assert(G_KH - G_KQ >= 32768 && 64 * AS * 4 >= 16384, "staging does not fit");

template <int MODE> __host__ __device__ constexpr int nthreads() { return MODE == 0 ? NT : NT_SPLIT; }
template <int MODE> __host__ __device__ constexpr uint32_t off_bar() { return MODE == 0 ? OFF_BAR : OFF_BAR_SPLIT; }
// dynamic shared memory, with slack for the 1024-byte alignment of the base
template <int MODE> __host__ __device__ constexpr uint32_t smem_bytes() {
    return (MODE == 0 ? OFF_NRM + 512 : OFF_BAR_SPLIT + BAR_BYTES) + 1024;
}
static_assert(OFF_NRM + 512 + 1024 <= 232448 && OFF_BAR_SPLIT + BAR_BYTES + 1024 <= 232448,
              "shared memory exceeds 227 KB");

// 4-D tensor maps {inner dim, H, T, B} with boxes of 64 tokens (split mode only).
// q, k: bf16 box {128,1,64,1}; g: fp32 box {128,...} ({64,...} with rotation); th: fp32
// {64,...} (rotation); v: bf16 box {64,1,64,1}, 128-byte swizzle (the MN-major V tile);
// o: output type, box {128,1,64,1}.
struct TmaMaps {
    CUtensorMap q, k, g, th, v, o;
};

struct SplitArgs {
    uint8_t* ring;            // [B*H][RING][SLOT_BYTES]
    unsigned int* ready;      // [B*H][RING]: index + 1 of the chunk a slot holds
    unsigned int* consumed;   // [B*H]: chunks the chain has copied out of the ring
    unsigned int* next_task;  // [1]: the next worker task to hand out (dynamic order)
    int dynamic;              // 1: tasks from the counter; 0: group i takes tasks i, i + G, ...
                              //    (G worker groups)
    int discard;              // 1: the ring is 128-byte aligned, so consumed slots are dropped from
                              //    L2 (no write-back of lines that nothing reads again)
};

// Flag words of the split workspace after the ring: ready, consumed, next_task (zeroed
// before every launch).
__host__ __device__ constexpr size_t split_flag_words(size_t nh) { return nh * RING + nh + 1; }

// Device status bits (gdr_query_device_status).
constexpr unsigned STATUS_TIMEOUT = 1u;
constexpr unsigned STATUS_RANGE = 2u;

struct TcExtra {
    unsigned long long wait_limit_ns;   // bound on every mbarrier wait
    int fault_skip_commit;              // test hook: 1 = never signal the first MMA barrier
};

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

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

// fp32 -> tf32 bits, rounded to nearest with ties away from zero, with two integer
// operations (the conversion instruction issues at a fraction of the ALU rate).  Finite
// inputs only: a NaN payload may round into another encoding.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u;
}

// D (16x8, fp32) += A (16x8, tf32, row-major fragment) * B (8x8, tf32, column fragment),
// one warp (mma.sync m16n8k8).
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint4 pack8(const float* m8) {
    using tc::pack_bf16x2;
    return make_uint4(pack_bf16x2(m8[0], m8[1]), pack_bf16x2(m8[2], m8[3]),
                      pack_bf16x2(m8[4], m8[5]), pack_bf16x2(m8[6], m8[7]));
}

// MODE 0 (fused): one CTA per (batch, head) runs both groups (384 threads).
// MODE 1 (split, 512 threads): CTAs [0, B*H) run the chain of head blockIdx.x: warp 0 copies
// ring slots into shared memory, warp 12 lane 0 issues the MMAs, warps 8-11 run the state and
// warps 4-7 convert the Wm tiles and write o.  Every other CTA is a prep worker with two
// independent 8-warp groups that compute chunks in chunk-major task order and write their
// operand tiles into the ring.  The grid must be co-resident (cooperative launch).
// EXT: the kernel with the optional features (a write strength w separate from beta when
// p.w is set; the fused L2 normalisation of q and k when p.qk_norm is set), switched on at
// run time; the plain kernel carries none of their cost.
template <int MODE, bool ROT, typename OT, bool EXT>
__global__ void __launch_bounds__(nthreads<MODE>(), 1) chunk_fwd_tc_kernel(FwdParams p, TcExtra x, SplitArgs sa,
                                                              const __grid_constant__ TmaMaps tm) {
    using namespace tc;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;          // shared-window base address
    uint8_t* base = smem_raw + (sb - raw_u32);               // generic pointer to the same byte
    uint8_t* bar_base = base + off_bar<MODE>();
    uint64_t* bar_pmma = reinterpret_cast<uint64_t*>(bar_base);   // [2] prep MMAs done (per group)
    uint64_t* bar_cmma = bar_pmma + 2;       // chain MMAs done
    uint64_t* bar_full = bar_pmma + 3;       // [2] prep -> chain: tiles of a chunk ready;
                                             //     split workers: group g's task done
    uint64_t* bar_empty = bar_pmma + 5;      // [2] chain -> prep: buffers of a chunk free
    uint64_t* bar_rho = bar_pmma + 7;        // [2] prep -> chain: decay vectors of a chunk ready;
                                             //     split workers: group g's staged inputs landed
    uint64_t* bar_o = bar_pmma + 9;          // split chain: O^T of a chunk complete
    uint64_t* bar_wready = bar_pmma + 11;    // split chain: P_m Wm^T of a chunk converted into its slot
    uint64_t* bar_sbr = bar_pmma + 10;       // split chain: bf16 state of the next chunk written
    uint64_t* bar_ecv = bar_pmma + 12;       // split chain: E^T converted and S decayed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_base + 112);
    int* abort_p = reinterpret_cast<int*>(bar_base + 116);
    int* abort_c = reinterpret_cast<int*>(bar_base + 120);
    int* range_flag = reinterpret_cast<int*>(bar_base + 124);
    auto vecs = [&](int c) -> float* { return reinterpret_cast<float*>(base + OFF_VEC) + (c & 1) * VEC_FLOATS; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;
    // Heads [p.head0, p.head0 + p.nheads) of the flattened b*H + h; indices below are local
    // (ring slots, task numbers) unless named global.
    const int NH = p.nheads;
    const bool chain_cta = (MODE == 0) || ((int)blockIdx.x < NH);
    const int bh = chain_cta ? (int)blockIdx.x : 0;
    const int gbh = p.head0 + bh;           // this chain's global head
    const __nv_bfloat16* __restrict__ q = static_cast<const __nv_bfloat16*>(p.q);
    const __nv_bfloat16* __restrict__ k = static_cast<const __nv_bfloat16*>(p.k);
    const __nv_bfloat16* __restrict__ v = static_cast<const __nv_bfloat16*>(p.v);
    OT* __restrict__ o = static_cast<OT*>(p.o);
    const int nchunks = (p.T + C - 1) / C;
    const bool untied = EXT && p.w != nullptr;    // a write strength w separate from beta
    const bool qkn = EXT && p.qk_norm != 0;       // fused L2 normalisation of q and k
    const bool cmean = EXT && p.chunk_mean != nullptr;   // per-chunk mean of o as a second output
    // chunk_mean [B, nchunks, H, dv] fp32: element of (global head gx, chunk c, value row r)
    auto cmean_at = [&](int gx, int c, int r) -> float* {
        return p.chunk_mean + (((size_t)(gx / p.H) * nchunks + c) * p.H + gx % p.H) * D + r;
    };
    auto chunk_len = [&](int c) -> int { return min(C, p.T - c * C); };
    auto tokh = [&](int bhx, int c, int r) -> size_t {      // bhx: local head
        const int gx = p.head0 + bhx;
        return ((size_t)(gx / p.H) * p.T + (c * C + r)) * p.H + (gx % p.H);
    };
    auto tok = [&](int c, int r) -> size_t { return tokh(bh, c, r); };
    // Split chain CTAs: the shared-memory buffer that holds chunk c's ring slot.
    auto slot_base = [&](int c) -> uint32_t { return (uint32_t)(c & 1) * SLOT_STRIDE; };

    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_cmma, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_pmma + i, 1);
            mbar_init(bar_o + i, 1);
            if (i == 0) {
                mbar_init(bar_wready, 1);
                mbar_init(bar_ecv, 1);
            }
            // split chain CTAs: the loader's expect_tx arrival (plus the slot's and V's bytes)
            mbar_init(bar_full + i, (MODE == 1 && chain_cta) ? 1 : NPREP);
            mbar_init(bar_empty + i, (MODE == 1) ? 1 : CHAIN_THREADS);
            // split workers: one expect_tx arrival plus the staged bytes
            mbar_init(bar_rho + i, (MODE == 1) ? 1 : NPREP);
        }
        fence_mbar_init();
        *abort_p = 0;
        *abort_c = 0;
        *range_flag = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tq = tbase + ((uint32_t)(quad * 32) << 16);   // this warp's lane quadrant

    if (nchunks > 0 && (MODE == 0 ? tid < NPREP : (!chain_cta && tid < 2 * NPREP))) {
        // =========================== prep group ===================================
        // Tasks: fused mode, the chunks of this CTA's head in order; split mode, tasks in
        // chunk-major order (chunk = task / NH, head = task % NH), either handed out one at a
        // time by a global counter (a group that ran fast takes the next task) or at a fixed
        // stride of the number of groups (which paces each group to the chains once the
        // stride nears the ring's depth in tasks).  A group claims its next task while it
        // works on the current one.
        const int grp = (MODE == 1) ? (int)threadIdx.x / NPREP : 0;
        const int tid = (int)threadIdx.x - grp * NPREP;      // thread within the group
        const int warp = tid >> 5;
        const int gbar = 1 + 2 * grp;                        // the group's named barrier
        uint8_t* gb = base + (uint32_t)grp * G_STRIDE;      // split: the group's tiles
        const uint32_t gsb = sb + (uint32_t)grp * G_STRIDE;
        uint64_t* g_pmma = bar_pmma + grp;
        uint64_t* g_stage = bar_rho + grp;
        const uint32_t col_aw = (MODE == 0) ? COL_AW : (uint32_t)grp * 64u;
        float* Af = reinterpret_cast<float*>(MODE == 0 ? base + OFF_AF : gb + G_AF);
        float* Tf = reinterpret_cast<float*>(MODE == 0 ? base + OFF_TF : gb + G_TF);
        float* QT = reinterpret_cast<float*>(MODE == 0 ? base + OFF_QT : gb + G_QT);
        const int total = (MODE == 0) ? nchunks : NH * nchunks;
        int* s_task = reinterpret_cast<int*>(bar_base + 128) + grp;   // split: the group's next task
        // Decay passes: each thread owns 4 key dims (two key pairs) of one 8-token segment;
        // warp w handles tokens 8w .. 8w+7.  The reference token 31 is the last token of
        // segment 3, so segments 0-3 run backward from it and segments 4-7 forward.
        const int dg = tid & 31;                 // dims 4dg .. 4dg+3 (pairs 2dg, 2dg+1)
        const int sg = tid >> 5;                 // token segment
        const int half = warp >> 2;              // TMEM column half for readbacks
        const int row = quad * 32 + lane;        // TMEM lane for readbacks
        const uint32_t kb = (uint32_t)(dg >> 4);             // K block of the 4 dims
        const uint32_t ch = (uint32_t)((dg & 15) >> 1);      // 16-byte chunk in the 128-byte row
        const uint32_t in_ch = (uint32_t)(dg & 1) * 8u;      // byte offset in the chunk
        const size_t tstride = (size_t)p.H * D;              // elements between consecutive tokens
        uint32_t mma_phase = 0;
        bool skip_commit = x.fault_skip_commit != 0;
        bool bad = false;

        // Register prefetch of this thread's raw inputs for one chunk.
        uint2 rk[8], rq[8];
        float4 ra[8];       // real: 4 gates; rotation: gates of the 2 pairs, then their 2 angles
        auto prefetch = [&](int bhx, int c) {
            const int Lc = chunk_len(c);
            const size_t t0 = tokh(bhx, c, 8 * sg);
            const __nv_bfloat16* kp = k + t0 * D + 4 * dg;
            const __nv_bfloat16* qp = q + t0 * D + 4 * dg;
#pragma unroll
            for (int s_ = 0; s_ < 8; ++s_) {
                rk[s_] = make_uint2(0u, 0u);
                rq[s_] = make_uint2(0u, 0u);
                ra[s_] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (8 * sg + s_ < Lc) {
                    rk[s_] = __ldg(reinterpret_cast<const uint2*>(kp + s_ * tstride));
                    rq[s_] = __ldg(reinterpret_cast<const uint2*>(qp + s_ * tstride));
                    if (!ROT) {
                        ra[s_] = __ldg(reinterpret_cast<const float4*>(p.g + (t0 + (size_t)s_ * p.H) * D + 4 * dg));
                    } else {
                        const size_t e = (t0 + (size_t)s_ * p.H) * (D / 2) + 2 * dg;
                        const float2 g2 = __ldg(reinterpret_cast<const float2*>(p.g + e));
                        const float2 t2 = __ldg(reinterpret_cast<const float2*>(p.theta + e));
                        ra[s_] = make_float4(g2.x, g2.y, t2.x, t2.y);
                    }
                }
            }
        };
        // One thread waits for the MMAs; the others wait at the named barrier (no issue slots)
        // and order their tensor-memory reads after it with the fence.
        auto mma_wait = [&]() -> bool {
            if (tid == 0 && !mbar_wait_bounded(g_pmma, mma_phase, x.wait_limit_ns)) atomicExch(abort_p, 1);
            mma_phase ^= 1u;
            named_bar(gbar, NPREP);
            tc_fence_after();
            return *abort_p == 0;
        };
        auto publish = [&]() {
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(gbar, NPREP);
            tc_fence_after();
        };
        // split: stage part `part` of task itx's raw inputs (tokens past the sequence end
        // arrive as zeros); part 0 also arms the barrier for all 64 KB
        int staged = 0, landed = 0;     // split: tasks whose staging was issued / has landed
        // Split: the ring slot of a finished task is published by the group's thread 32 once
        // the next task's inputs have been read (or after the last task), while the other warps
        // run pass 1; the named barriers order every thread's stores to the slot before its
        // gpu-scope release (cumulative over what the thread has observed).  Publishing before
        // the next task's ring-slot wait keeps the workers free of waits on one another.
        int pub_c = -1, pub_bh = 0;
        auto publish_slot = [&]() {
            st_release_gpu(sa.ready + (size_t)pub_bh * RING + pub_c % RING, (unsigned)(pub_c + 1));
            pub_c = -1;
        };
        auto stage_part = [&](int tk, int part) {
            const int c2 = tk / NH, b2 = p.head0 + tk % NH;     // global head
            const int bb = b2 / p.H, hh = b2 % p.H;
            if (part == 0) {
                ++staged;
                mbar_arrive_expect_tx(g_stage, 65536u);
                tma_load_4d(gsb + G_KH, &tm.q, 0, hh, c2 * C, bb, g_stage);
            } else if (part == 1) {
                tma_load_4d(gsb + G_KQ, &tm.g, 0, hh, c2 * C, bb, g_stage);
                if (ROT) tma_load_4d(gsb + G_KQ + 16384u, &tm.th, 0, hh, c2 * C, bb, g_stage);
            } else {
                tma_load_4d(gsb + G_AF, &tm.k, 0, hh, c2 * C, bb, g_stage);
            }
        };
        const uint32_t ID_KK = idesc_bf16(128, 64, 0, 0, 0), ID_MK = idesc_bf16(128, 64, 1, 0, 0);

        int task = 0, nxt = total;      // split: nxt, the claimed next task (thread 0)
        int fixed_next = (MODE == 0) ? 0 : 2 * ((int)blockIdx.x - NH) + grp;   // static order
        auto claim = [&]() -> int {
            if (sa.dynamic) return (int)atomicAdd(sa.next_task, 1u);
            const int t = fixed_next;
            fixed_next += 2 * ((int)gridDim.x - NH);
            return min(t, total);
        };
        if (MODE == 0 && total > 0) prefetch(bh, 0);
        if (MODE == 1) {
            if (tid == 0) {
                nxt = claim();
                *s_task = nxt;
                if (nxt < total) {
                    stage_part(nxt, 0);
                    stage_part(nxt, 1);
                    stage_part(nxt, 2);
                }
            }
            named_bar(gbar, NPREP);
            task = *s_task;
        }
        for (int it = 0; task < total; ++it) {
            const int c = (MODE == 0) ? task : task / NH, bhx = (MODE == 0) ? bh : task % NH;
            const int Lc = chunk_len(c);
            const int bufi = (MODE == 0) ? (it & 1) : 0;      // split workers: single tile buffers
            float* vec = (MODE == 0) ? vecs(bufi) : reinterpret_cast<float*>(gb + G_VEC);
            // split mode: this task's ring slot, written directly by the prep warps
            uint8_t* ring = (MODE == 1) ? sa.ring + ((size_t)bhx * RING + c % RING) * SLOT_BYTES : nullptr;
            // (debug build: a task outside the ring is reported and its writes go to slot 0,
            // inside the workspace, so that the group's barriers stay in step)
            if (MODE == 1 && !GDR_INB(bhx >= 0 && bhx < NH && c >= 0 && c < nchunks, 605)) ring = sa.ring;
            float* rvec = reinterpret_cast<float*>(ring + SL_VEC);
            // beta of this task, consumed after pass 1
            float beta_r = 0.f, w_r = 0.f;
            if (tid < 64 && tid < Lc) {
                beta_r = __ldg(p.beta + tokh(bhx, c, tid));
                w_r = untied ? __ldg(p.w + tokh(bhx, c, tid)) : beta_r;
            }
            if (MODE == 1) {
                // raw inputs of this task, staged by the transfer thread (tokens past the
                // sequence end arrive as zeros)
                const bool ok = mbar_wait_bounded(g_stage, it & 1, x.wait_limit_ns);
                if (!ok) atomicExch(abort_p, 1);
                landed = it + 1;
                named_bar(gbar, NPREP);
                if (*abort_p) break;
#pragma unroll
                for (int s_ = 0; s_ < 8; ++s_) {
                    const int r = 8 * sg + s_;
                    rk[s_] = *reinterpret_cast<const uint2*>(gb + G_AF + (uint32_t)(r * D + 4 * dg) * 2u);
                    rq[s_] = *reinterpret_cast<const uint2*>(gb + G_KH + (uint32_t)(r * D + 4 * dg) * 2u);
                    if (!ROT) {
                        ra[s_] = *reinterpret_cast<const float4*>(gb + G_KQ + (uint32_t)(r * D + 4 * dg) * 4u);
                    } else {
                        const float2 g2 = *reinterpret_cast<const float2*>(gb + G_KQ + (uint32_t)(r * 64 + 2 * dg) * 4u);
                        const float2 t2 = *reinterpret_cast<const float2*>(gb + G_KQ + 16384u + (uint32_t)(r * 64 + 2 * dg) * 4u);
                        ra[s_] = make_float4(g2.x, g2.y, t2.x, t2.y);
                    }
                }
                if (tid == 32 && pub_c >= 0) publish_slot();   // overlaps pass 1 of the other warps
            }
            float* sbeta = vec;
            float* rho_ref = vec + 64;
            float* rho_C = vec + 64 + 256;
            uint8_t* KQ = (MODE == 0) ? base + OFF_KQ + bufi * 32768 : gb + G_KQ;
            uint8_t* KH = (MODE == 0) ? base + OFF_KH + bufi * 16384 : gb + G_KH;
            const uint32_t kq_s = (MODE == 0) ? sb + OFF_KQ + bufi * 32768 : gsb + G_KQ;
            const uint32_t kh_s = (MODE == 0) ? sb + OFF_KH + bufi * 16384 : gsb + G_KH;

            // V tile of this chunk (MN-major for V^T), asynchronously; done before the U MMA.
            // (Split mode: the copy-out warps move V straight into the ring.)
            if (MODE == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int id = tid * 4 + j;
                const int i = id >> 4, c16 = id & 15;
                const bool ok = i < Lc;
                const void* src = ok ? (const void*)(v + tokh(bhx, c, i) * D + c16 * 8) : (const void*)v;
                cp_async16(sb + OFF_V + (uint32_t)(c16 >> 3) * 8192u + sw128_off(i, c16 & 7), src, ok ? 16u : 0u);
            }
            cp_async_commit();
            }

            // ---- fused L2 normalisation: inverse norms of this warp's 8 tokens' k and q ----
            float2* nrm = reinterpret_cast<float2*>((MODE == 0) ? base + OFF_NRM : gb + G_NRM);
            if (qkn) {
#pragma unroll
                for (int s_ = 0; s_ < 8; ++s_) {
                    const uint2 kr = rk[s_], qr = rq[s_];
                    const float k0 = __uint_as_float(kr.x << 16), k1 = __uint_as_float(kr.x & 0xFFFF0000u);
                    const float k2 = __uint_as_float(kr.y << 16), k3 = __uint_as_float(kr.y & 0xFFFF0000u);
                    const float q0 = __uint_as_float(qr.x << 16), q1 = __uint_as_float(qr.x & 0xFFFF0000u);
                    const float q2 = __uint_as_float(qr.y << 16), q3 = __uint_as_float(qr.y & 0xFFFF0000u);
                    float sk = k0 * k0 + k1 * k1 + k2 * k2 + k3 * k3;
                    float sq = q0 * q0 + q1 * q1 + q2 * q2 + q3 * q3;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {      // the warp holds all 128 dims
                        sk += __shfl_xor_sync(0xffffffffu, sk, off);
                        sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    }
                    if (lane == 0) nrm[8 * sg + s_] = make_float2(rsqrtf(sk + 1e-6f), rsqrtf(sq + 1e-6f));
                }
            }

            // ---- pass 1: per-token decays and segment products ---------------------------
            // real:     al[s][d] = alpha of dim 4dg+d;
            // rotation: al[s][j] = alpha of pair 2dg+j, al[s][2+j] = cos, sn[s][j] = sin.
            // (1/alpha is formed again where pass 2 needs it.)
            float al[8][4], sn[8][2];
            float PA[4] = {1.f, 1.f, 1.f, 1.f}, PI[4] = {1.f, 1.f, 1.f, 1.f};
            if (ROT) { PI[2] = 0.f; PI[3] = 0.f; }           // (PA[2+j], PI[2+j]) = prod e^{+i theta}, from 1 + 0i
            const float L2E = 1.4426950408889634f;
#pragma unroll
            for (int s_ = 0; s_ < 8; ++s_) {
                const bool ok = 8 * sg + s_ < Lc;
                const float ga[4] = {ra[s_].x, ra[s_].y, ra[s_].z, ra[s_].w};
#pragma unroll
                for (int d = 0; d < (ROT ? 2 : 4); ++d) {
                    float a_ = 1.f, i_ = 1.f;
                    if (ok) {
                        if (p.gate_mode == 1) {
                            i_ = 1.f + ex2_approx(ga[d] * L2E);
                            a_ = rcp_approx(i_);
                        } else {
                            a_ = ex2_approx(ga[d] * L2E);
                            i_ = ex2_approx(-ga[d] * L2E);
                        }
                    }
                    al[s_][d] = a_;
                    PA[d] *= a_; PI[d] *= i_;
                }
                if (ROT) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        float cs = 1.f, sn_ = 0.f;
                        if (ok) __sincosf(ga[2 + j], &sn_, &cs);
                        al[s_][2 + j] = cs; sn[s_][j] = sn_;
                        const float zr = PA[2 + j] * cs - PI[2 + j] * sn_, zi = PI[2 + j] * cs + PA[2 + j] * sn_;
                        PA[2 + j] = zr; PI[2 + j] = zi;
                    }
                }
            }
            {
                float4* qtp = reinterpret_cast<float4*>(QT + (sg * 32 + dg) * 8);
                qtp[0] = make_float4(PA[0], PA[1], PA[2], PA[3]);
                qtp[1] = make_float4(PI[0], PI[1], PI[2], PI[3]);
            }
            if (tid < 64) { sbeta[tid] = beta_r; vec[VEC_W + tid] = w_r; }
            named_bar(gbar, NPREP);
            // Buffers of task it - 2 must be released (by the chain, or by the copy-out warps)
            // before they are rewritten.
            if (MODE == 0 && it >= 2) {
                const bool ok = mbar_wait_bounded(bar_empty + bufi, ((it - 2) >> 1) & 1, x.wait_limit_ns);
                if (!ok) atomicExch(abort_p, 1);
            }
            if (MODE == 1 && tid == 0 && c >= RING) {
                // the chain must have copied chunk c - RING out of this ring slot
                const bool ok = spin_until_ge(sa.consumed + bhx, (unsigned)(c - RING + 1), x.wait_limit_ns);
                if (!ok) atomicExch(abort_p, 1);
            }
            named_bar(gbar, NPREP);
            if (*abort_p) break;
            if (MODE == 1 && tid < 64) rvec[tid] = beta_r;

            // ---- pass 2: factors around the reference token 31; operand tiles -----------
            {
                // P: products of alpha, Q: products of 1/alpha (per dim, or per pair magnitude);
                // R: phase of a pair, as a complex number.
                float P[4] = {1.f, 1.f, 1.f, 1.f}, Q[4] = {1.f, 1.f, 1.f, 1.f};
                float Rre[2] = {1.f, 1.f}, Rim[2] = {0.f, 0.f};
                const int lo = sg < 4 ? sg + 1 : 4, hi = sg < 4 ? 4 : sg;   // segments between me and token 31
                for (int s2 = lo; s2 < hi; ++s2) {
                    const float4* t = reinterpret_cast<const float4*>(QT + (s2 * 32 + dg) * 8);
                    const float4 a4 = t[0], i4 = t[1];
                    if (!ROT) {
                        P[0] *= a4.x; P[1] *= a4.y; P[2] *= a4.z; P[3] *= a4.w;
                        Q[0] *= i4.x; Q[1] *= i4.y; Q[2] *= i4.z; Q[3] *= i4.w;
                    } else {
                        P[0] *= a4.x; P[1] *= a4.y; Q[0] *= i4.x; Q[1] *= i4.y;
                        const float zr[2] = {a4.z, a4.w};
                        const float zi[2] = {sg < 4 ? i4.z : -i4.z, sg < 4 ? i4.w : -i4.w};   // forward: conjugate
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float nr = Rre[j] * zr[j] - Rim[j] * zi[j], ni = Rim[j] * zr[j] + Rre[j] * zi[j];
                            Rre[j] = nr; Rim[j] = ni;
                        }
                    }
                }
                const float sc = p.scale;
                // Split: the ring carries Qtil2 = Qtil P_m^T and Khat2 = Khat (P_m^{-1} P_C), the
                // reference decay folded in, so that the chain can keep the plain state.  rr / rc:
                // P_m and P_m^{-1} P_C of this thread's dims (rotation: [j] real, [2+j] imaginary
                // part of pair 2dg+j), from the segment products.
                float rr[4] = {1.f, 1.f, 1.f, 1.f}, rc[4] = {1.f, 1.f, 1.f, 1.f};
                if (MODE == 1) {
                    float mr[4] = {1.f, 1.f, 0.f, 0.f}, mc[4] = {1.f, 1.f, 0.f, 0.f};   // rotation: magnitudes, phases
                    float pr_re[2] = {1.f, 1.f}, pr_im[2] = {0.f, 0.f}, pc_re[2] = {1.f, 1.f}, pc_im[2] = {0.f, 0.f};
#pragma unroll
                    for (int s2 = 0; s2 < 8; ++s2) {
                        const float4* t = reinterpret_cast<const float4*>(QT + (s2 * 32 + dg) * 8);
                        const float4 a4 = t[0];
                        if (!ROT) {
                            float* f = s2 < 4 ? rr : rc;
                            f[0] *= a4.x; f[1] *= a4.y; f[2] *= a4.z; f[3] *= a4.w;
                        } else {
                            const float4 i4 = t[1];
                            float* m = s2 < 4 ? mr : mc;
                            float* zre = s2 < 4 ? pr_re : pc_re;
                            float* zim = s2 < 4 ? pr_im : pc_im;
                            m[0] *= a4.x; m[1] *= a4.y;
                            const float zr[2] = {a4.z, a4.w}, zi[2] = {i4.z, i4.w};
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const float nr = zre[j] * zr[j] - zim[j] * zi[j], ni = zim[j] * zr[j] + zre[j] * zi[j];
                                zre[j] = nr; zim[j] = ni;
                            }
                        }
                    }
                    if (ROT) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            rr[j] = mr[j] * pr_re[j]; rr[2 + j] = mr[j] * pr_im[j];
                            rc[j] = mc[j] * pc_re[j]; rc[2 + j] = mc[j] * pc_im[j];
                        }
                    }
                }
                auto emit = [&](int r, const float (&F)[4], const float (&G)[4], uint2 kraw, uint2 qraw) {
                    float kk[4] = {__uint_as_float(kraw.x << 16), __uint_as_float(kraw.x & 0xFFFF0000u),
                                   __uint_as_float(kraw.y << 16), __uint_as_float(kraw.y & 0xFFFF0000u)};
                    float qv[4] = {__uint_as_float(qraw.x << 16), __uint_as_float(qraw.x & 0xFFFF0000u),
                                   __uint_as_float(qraw.y << 16), __uint_as_float(qraw.y & 0xFFFF0000u)};
                    if (qkn) {
                        const float2 nn = nrm[r];
#pragma unroll
                        for (int d = 0; d < 4; ++d) { kk[d] *= nn.x; qv[d] *= nn.y; }
                    }
                    float kt[4], qt[4], kh[4];
                    if (!ROT) {
#pragma unroll
                        for (int d = 0; d < 4; ++d) {
                            kt[d] = kk[d] * F[d]; qt[d] = qv[d] * (sc * F[d]); kh[d] = kk[d] * G[d];
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            // F = |F| R, G = |G| R, applied to (x + i y) = (v[2j] + i v[2j+1])
                            const float fr = F[j] * Rre[j], fi = F[j] * Rim[j];
                            const float gr = G[j] * Rre[j], gi = G[j] * Rim[j];
                            const float k0 = kk[2 * j], k1 = kk[2 * j + 1], q0 = sc * qv[2 * j], q1 = sc * qv[2 * j + 1];
                            kt[2 * j] = fr * k0 - fi * k1; kt[2 * j + 1] = fr * k1 + fi * k0;
                            qt[2 * j] = fr * q0 - fi * q1; qt[2 * j + 1] = fr * q1 + fi * q0;
                            kh[2 * j] = gr * k0 - gi * k1; kh[2 * j + 1] = gr * k1 + gi * k0;
                        }
                    }
                    const uint32_t off = sw128_off(r, ch) + in_ch;
                    const uint2 qtv = make_uint2(pack_bf16x2(qt[0], qt[1]), pack_bf16x2(qt[2], qt[3]));
                    const uint2 khv = make_uint2(pack_bf16x2(kh[0], kh[1]), pack_bf16x2(kh[2], kh[3]));
                    *reinterpret_cast<uint2*>(KQ + kb * 16384u + off) = make_uint2(pack_bf16x2(kt[0], kt[1]), pack_bf16x2(kt[2], kt[3]));
                    *reinterpret_cast<uint2*>(KQ + kb * 16384u + 8192u + off) = qtv;
                    *reinterpret_cast<uint2*>(KH + kb * 8192u + off) = khv;
                    if (MODE == 1) {        // the ring slot has the tiles' shared-memory layout
                        float q2[4], k2[4];
                        if (!ROT) {
#pragma unroll
                            for (int d = 0; d < 4; ++d) { q2[d] = qt[d] * rr[d]; k2[d] = kh[d] * rc[d]; }
                        } else {
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const float a = qt[2 * j], b = qt[2 * j + 1], e = kh[2 * j], f = kh[2 * j + 1];
                                q2[2 * j] = a * rr[j] + b * rr[2 + j];        // times conj(P_m)
                                q2[2 * j + 1] = b * rr[j] - a * rr[2 + j];
                                k2[2 * j] = e * rc[j] - f * rc[2 + j];        // times P_m^{-1} P_C
                                k2[2 * j + 1] = e * rc[2 + j] + f * rc[j];
                            }
                        }
                        *reinterpret_cast<uint2*>(ring + SL_Q + kb * 8192u + off) =
                            make_uint2(pack_bf16x2(q2[0], q2[1]), pack_bf16x2(q2[2], q2[3]));
                        // Ktil2 = Ktil P_m^T, from which the chain CTA forms P_m Wm^T = Ktil2^T Tb^T
                        if (!ROT) {
#pragma unroll
                            for (int d = 0; d < 4; ++d) q2[d] = kt[d] * rr[d];
                        } else {
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const float a = kt[2 * j], b = kt[2 * j + 1];
                                q2[2 * j] = a * rr[j] + b * rr[2 + j];
                                q2[2 * j + 1] = b * rr[j] - a * rr[2 + j];
                            }
                        }
                        *reinterpret_cast<uint2*>(ring + SL_W + kb * 8192u + off) =
                            make_uint2(pack_bf16x2(q2[0], q2[1]), pack_bf16x2(q2[2], q2[3]));
                        *reinterpret_cast<uint2*>(ring + SL_KH + kb * 8192u + off) =
                            make_uint2(pack_bf16x2(k2[0], k2[1]), pack_bf16x2(k2[2], k2[3]));
                    }
                };
                auto include = [&](int s_, bool forward) {
#pragma unroll
                    for (int d = 0; d < (ROT ? 2 : 4); ++d) { P[d] *= al[s_][d]; Q[d] *= rcp_approx(al[s_][d]); }
                    if (ROT) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float cs = al[s_][2 + j], sv = forward ? -sn[s_][j] : sn[s_][j];
                            const float nr = Rre[j] * cs - Rim[j] * sv, ni = Rim[j] * cs + Rre[j] * sv;
                            Rre[j] = nr; Rim[j] = ni;
                        }
                    }
                };
                if (sg < 4) {
                    // backward from token 31: factors over tokens r+1..31, then include r
#pragma unroll
                    for (int s_ = 7; s_ >= 0; --s_) {
                        emit(8 * sg + s_, Q, P, rk[s_], rq[s_]);
                        include(s_, false);
                    }
                    if (sg == 0) {   // prod over tokens 0..31: e^{Gamma_m} (and e^{i Theta_m})
                        if (!ROT) {
                            *reinterpret_cast<float4*>(rho_ref + 4 * dg) = make_float4(P[0], P[1], P[2], P[3]);
                        } else {
                            rho_ref[2 * dg] = P[0] * Rre[0]; rho_ref[2 * dg + 1] = P[1] * Rre[1];
                            rho_ref[128 + 2 * dg] = P[0] * Rim[0]; rho_ref[128 + 2 * dg + 1] = P[1] * Rim[1];
                        }
                    }
                } else {
                    // forward from token 32: include r, then use
#pragma unroll
                    for (int s_ = 0; s_ < 8; ++s_) {
                        include(s_, true);
                        emit(8 * sg + s_, P, Q, rk[s_], rq[s_]);
                    }
                    if (sg == 7) {   // prod over tokens 32..63: e^{Gamma_C - Gamma_m}; R holds the conjugate phase
                        if (!ROT) {
                            *reinterpret_cast<float4*>(rho_C + 4 * dg) = make_float4(P[0], P[1], P[2], P[3]);
                        } else {
                            rho_C[2 * dg] = P[0] * Rre[0]; rho_C[2 * dg + 1] = P[1] * Rre[1];
                            rho_C[128 + 2 * dg] = -P[0] * Rim[0]; rho_C[128 + 2 * dg + 1] = -P[1] * Rim[1];
                        }
                    }
                }
                // The products grow monotonically away from token 31: checking the final ones
                // covers every factor this thread used.
#pragma unroll
                for (int d = 0; d < 4; ++d)
                    if (!(fabsf(Q[d]) < 3e38f && fabsf(P[d]) < 3e38f)) bad = true;
            }
            fence_proxy_async_smem();
            named_bar(gbar, NPREP);
            if (MODE == 1 && tid < 128) {   // P_C = P_m (P_m^{-1} P_C) -> ring
                if (!ROT) {
                    rvec[64 + tid] = vec[64 + tid] * vec[64 + 256 + tid];
                } else if (tid < 64) {
                    const float a = vec[64 + tid], b = vec[64 + 128 + tid], cc = vec[64 + 256 + tid], d = vec[64 + 384 + tid];
                    rvec[64 + tid] = a * cc - b * d;
                    rvec[64 + 128 + tid] = a * d + b * cc;
                }
            }
            if (MODE == 0) mbar_arrive(bar_rho + bufi);
            if (MODE == 0 && task + 1 < total) prefetch(bh, task + 1);

            // ---- MMA1: [Ktil ; Qtil] Khat^T -> TMEM ------------------------------------
            tc_fence_after();
            if (tid == 0) {
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t kbk = ks >> 2, kin = (ks & 3) * 32;
                    mma_bf16_ss(tbase + col_aw, sdesc_sw128(kq_s + kbk * 16384 + kin, 16, 1024),
                                sdesc_sw128(kh_s + kbk * 8192 + kin, 16, 1024), ID_KK, ks > 0);
                }
                if (!skip_commit) mma_commit(g_pmma);
                skip_commit = false;
            }
            if (!mma_wait()) break;
            if (MODE == 1 && tid == 0) {     // MMA1 has read the operand tiles
                // claim the next task; the group reads it after this task's last barrier
                nxt = claim();
                *s_task = nxt;
                if (nxt < total) {
                    stage_part(nxt, 0);
                    stage_part(nxt, 1);
                }
            }

            // ---- solve: Tm = (I + A)^{-1}; Pm masked -> bf16 ---------------------------
            {
                float vals[32];
                tmem_ld16(tq + col_aw + half * 32, *reinterpret_cast<float(*)[16]>(vals));
                tmem_ld16(tq + col_aw + half * 32 + 16, *reinterpret_cast<float(*)[16]>(vals + 16));
                if (row < 64) {
                    const int r = row;
                    const float br = sbeta[r];
#pragma unroll
                    for (int u = 0; u < 32; u += 4) {
                        float4 w;
                        const int i = half * 32 + u;
                        w.x = (i < r) ? br * vals[u] : 0.f;
                        w.y = (i + 1 < r) ? br * vals[u + 1] : 0.f;
                        w.z = (i + 2 < r) ? br * vals[u + 2] : 0.f;
                        w.w = (i + 3 < r) ? br * vals[u + 3] : 0.f;
                        *reinterpret_cast<float4*>(Af + r * AS + i) = w;
                    }
                } else {
                    const int r = row - 64;
                    uint8_t* PM = (MODE == 0) ? base + OFF_PM + bufi * 8192 : ring + SL_PM;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        float m8[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int i = half * 32 + cc * 8 + u;
                            m8[u] = (i <= r) ? vals[cc * 8 + u] : 0.f;
                        }
                        *reinterpret_cast<uint4*>(PM + sw128_off(r, half * 4 + cc)) = pack8(m8);
                    }
                }
            }
            uint8_t* TB = (MODE == 0) ? base + OFF_TB : gb + G_TB;
            uint8_t* TW = (MODE == 0) ? base + OFF_TW : gb + G_TW;
            const float* sw = vec + VEC_W;
            {   // Tb (and Tw): blocks above the diagonal stay zero
                uint4* tbz = reinterpret_cast<uint4*>(TB);
                tbz[tid] = make_uint4(0u, 0u, 0u, 0u);
                tbz[tid + NPREP] = make_uint4(0u, 0u, 0u, 0u);
                if (untied) {
                    uint4* twz = reinterpret_cast<uint4*>(TW);
                    twz[tid] = make_uint4(0u, 0u, 0u, 0u);
                    twz[tid + NPREP] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            named_bar(gbar, NPREP);
            // Tb = Tm diag(beta) as bf16 K-major [r][i] (blocks above the diagonal stay zero);
            // with a separate write strength also Tw = Tm diag(w), for U = Tw V.
            auto tb_put2 = [&](int r, int i, float x0, float x1) {      // columns i, i + 1
                const uint32_t off = sw128_off(r, i >> 3) + (i & 7) * 2;
                *reinterpret_cast<uint32_t*>(TB + off) = pack_bf16x2(x0 * sbeta[i], x1 * sbeta[i + 1]);
                if (untied) *reinterpret_cast<uint32_t*>(TW + off) = pack_bf16x2(x0 * sw[i], x1 * sw[i + 1]);
            };
            // 16x16 diagonal blocks by forward substitution (lane = column of one block).
            if (tid < 64) {
                const int bb = (tid >> 4) * 16, jj = tid & 15;
                float t[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float s_ = (r == jj) ? 1.f : 0.f;
#pragma unroll
                    for (int i = 0; i < r; ++i) s_ = fmaf(-Af[(bb + r) * AS + bb + i], t[i], s_);
                    t[r] = s_;
                }
                const float bj = sbeta[bb + jj], wj = sw[bb + jj];
                const int ib = bb + jj;
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    Tf[(bb + r) * AS + bb + jj] = t[r];
                    const uint32_t off = sw128_off(bb + r, ib >> 3) + (ib & 7) * 2;
                    *reinterpret_cast<__nv_bfloat16*>(TB + off) = __float2bfloat16_rn(t[r] * bj);
                    if (untied) *reinterpret_cast<__nv_bfloat16*>(TW + off) = __float2bfloat16_rn(t[r] * wj);
                }
            }
            named_bar(gbar, NPREP);
            // Blocks below the diagonal in one phase, one warp per block, with the 2x2 block
            // recursion T_lo,hi-split: T_hi,lo = -T_hi A_hi,lo T_lo for the halves {0,1}, {2,3}:
            //   T10 = -D1 A10 D0,  T21 = -D2 A21 D1,  T32 = -D3 A32 D2,
            //   T20 = -D2 X20,     T31 = -(T32 A21 + D3 A31) D1,   T30 = -(T32 X20 + D3 X30),
            //   X20 = A20 D0 + A21 T10,  X30 = A30 D0 + A31 T10   (D_I: diagonal blocks).
            // Each warp forms the blocks it depends on itself, in 16x16 scratch taken from the
            // unused upper triangles of A and Tm, on m16n8k8 tf32 tensor-core MMAs (the result
            // is rounded to bf16 for the UT transform anyway).
            if (warp < 6) {
                const int gid = lane >> 2, tig = lane & 3;
                auto Ab = [&](int I, int J) { return Af + 16 * I * AS + 16 * J; };
                auto Tb_ = [&](int I, int J) { return Tf + 16 * I * AS + 16 * J; };
                // acc += L R for 16x16 fp32 blocks (row stride AS)
                auto mm = [&](float (&acc)[2][4], const float* L, const float* R) {
#pragma unroll
                    for (int kb8 = 0; kb8 < 16; kb8 += 8) {
                        const uint32_t a[4] = {to_tf32(L[gid * AS + kb8 + tig]), to_tf32(L[(gid + 8) * AS + kb8 + tig]),
                                               to_tf32(L[gid * AS + kb8 + tig + 4]),
                                               to_tf32(L[(gid + 8) * AS + kb8 + tig + 4])};
                        const uint32_t b0[2] = {to_tf32(R[(kb8 + tig) * AS + gid]), to_tf32(R[(kb8 + tig + 4) * AS + gid])};
                        const uint32_t b1[2] = {to_tf32(R[(kb8 + tig) * AS + 8 + gid]),
                                                to_tf32(R[(kb8 + tig + 4) * AS + 8 + gid])};
                        mma_tf32_16x8x8(acc[0], a, b0);
                        mma_tf32_16x8x8(acc[1], a, b1);
                    }
                };
                auto zero = [&](float (&acc)[2][4]) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
                };
                auto put = [&](float* Dst, const float (&acc)[2][4], float sg) {   // Dst = sg * acc
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        *reinterpret_cast<float2*>(Dst + gid * AS + 8 * h + 2 * tig) = make_float2(sg * acc[h][0], sg * acc[h][1]);
                        *reinterpret_cast<float2*>(Dst + (gid + 8) * AS + 8 * h + 2 * tig) =
                            make_float2(sg * acc[h][2], sg * acc[h][3]);
                    }
                    __syncwarp();
                };
                auto out = [&](int I, int J, const float (&acc)[2][4]) {     // Tb block (I, J) = -acc
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int i = 16 * J + 8 * h + 2 * tig;
                        tb_put2(16 * I + gid, i, -acc[h][0], -acc[h][1]);
                        tb_put2(16 * I + gid + 8, i, -acc[h][2], -acc[h][3]);
                    }
                };
                float x[2][4], y[2][4];
                if (warp < 3) {                 // T(w+1, w) = -D(w+1) A(w+1, w) D(w)
                    const int J = warp, I = warp + 1;
                    float* S0 = Ab(0, warp + 1);
                    zero(x); mm(x, Ab(I, J), Tb_(J, J)); put(S0, x, 1.f);
                    zero(y); mm(y, Tb_(I, I), S0); out(I, J, y);
                } else if (warp == 3) {         // T20
                    float* S0 = Ab(1, 2); float* S1 = Ab(1, 3);
                    zero(x); mm(x, Ab(1, 0), Tb_(0, 0)); put(S0, x, 1.f);
                    zero(y); mm(y, Tb_(1, 1), S0); put(S1, y, -1.f);                       // T10
                    zero(x); mm(x, Ab(2, 0), Tb_(0, 0)); mm(x, Ab(2, 1), S1); put(S0, x, 1.f);   // X20
                    zero(y); mm(y, Tb_(2, 2), S0); out(2, 0, y);
                } else if (warp == 4) {         // T31
                    float* S0 = Ab(2, 3); float* S1 = Tb_(0, 1);
                    zero(x); mm(x, Ab(3, 2), Tb_(2, 2)); put(S0, x, 1.f);
                    zero(y); mm(y, Tb_(3, 3), S0); put(S1, y, -1.f);                       // T32
                    zero(x); mm(x, S1, Ab(2, 1)); mm(x, Tb_(3, 3), Ab(3, 1)); put(S0, x, 1.f);
                    zero(y); mm(y, S0, Tb_(1, 1)); out(3, 1, y);
                } else {                        // T30
                    float* S0 = Tb_(0, 2); float* S1 = Tb_(0, 3); float* S2 = Tb_(1, 2); float* S3 = Tb_(1, 3);
                    zero(x); mm(x, Ab(1, 0), Tb_(0, 0));
                    zero(y); mm(y, Ab(3, 2), Tb_(2, 2));
                    put(S0, x, 1.f); put(S1, y, 1.f);
                    zero(x); mm(x, Tb_(1, 1), S0);
                    zero(y); mm(y, Tb_(3, 3), S1);
                    put(S2, x, -1.f); put(S3, y, -1.f);                                   // T10, T32
                    zero(x); mm(x, Ab(2, 0), Tb_(0, 0)); mm(x, Ab(2, 1), S2);             // X20
                    zero(y); mm(y, Ab(3, 0), Tb_(0, 0)); mm(y, Ab(3, 1), S2);             // X30
                    put(S0, x, 1.f); put(S1, y, 1.f);
                    zero(x); mm(x, S3, S0); mm(x, Tb_(3, 3), S1); out(3, 0, x);
                }
            }
            if (MODE == 0) cp_async_wait_all();
            publish();
            if (MODE == 1) {                // Tb -> ring
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    reinterpret_cast<uint4*>(ring + SL_TB)[tid + e * NPREP] = reinterpret_cast<const uint4*>(TB)[tid + e * NPREP];
                    if (untied)
                        reinterpret_cast<uint4*>(ring + SL_TW)[tid + e * NPREP] = reinterpret_cast<const uint4*>(TW)[tid + e * NPREP];
                }
                if (tid == 0 && nxt < total) stage_part(nxt, 2);          // A and Tm done
            }

            if (MODE == 0) {
                // ---- U^T = V^T Tb^T -> E[c&1];  Wm^T = Ktil^T Tb^T -> A'/W columns ---------
                if (tid == 0) {
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t bdesc = sdesc_sw128(sb + OFF_TB + ks * 32, 16, 1024);
                        const uint64_t wdesc = sdesc_sw128(sb + (untied ? OFF_TW : OFF_TB) + ks * 32, 16, 1024);
                        mma_bf16_ss(tbase + COL_E + bufi * 64, sdesc_sw128(sb + OFF_V + ks * 2048, 8192, 1024), wdesc,
                                    ID_MK, ks > 0);
                        mma_bf16_ss(tbase + col_aw, sdesc_sw128(kq_s + ks * 2048, 16384, 1024), bdesc, ID_MK, ks > 0);
                    }
                    mma_commit(g_pmma);
                }
                if (!mma_wait()) break;
                // Wm^T -> bf16 MN-major tile (row = dk, 64 tokens per row).
                {
                    float vals[32];
                    tmem_ld16(tq + col_aw + half * 32, *reinterpret_cast<float(*)[16]>(vals));
                    tmem_ld16(tq + col_aw + half * 32 + 16, *reinterpret_cast<float(*)[16]>(vals + 16));
                    uint8_t* W = base + OFF_W + bufi * 16384;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        *reinterpret_cast<uint4*>(W + sw128_off(row, half * 4 + cc)) = pack8(vals + cc * 8);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(gbar, NPREP);
            }
            if (MODE == 0) mbar_arrive(bar_full + bufi);
            if (MODE == 1) { pub_c = c; pub_bh = bhx; }
            task = (MODE == 0) ? task + 1 : *s_task;
        }
        if (MODE == 1 && tid == 32 && pub_c >= 0) publish_slot();
        if (bad) atomicExch(range_flag, 1);
        // after an early exit, let staging copies still in flight land before the CTA ends
        if (MODE == 1 && tid == 0 && staged > landed) (void)mbar_wait_bounded(g_stage, landed & 1, x.wait_limit_ns);
    } else if (MODE == 1 && nchunks > 0 && chain_cta && tid >= NPREP - 128 && tid <= NPREP + CHAIN_THREADS) {
        // ============ split mode: chain (warps 8-11) and helper warps 4-7 ======================
        // The chain keeps the plain state S (fp32) in TMEM and its bf16 copy in one of two column
        // blocks (chunk parity); the workers fold the reference decay into the ring's tiles
        // (Qtil2 = Qtil P_m^T, Ktil2 = Ktil P_m^T, Khat2 = Khat P_m^{-1} P_C), so per chunk
        //   Wm2^T = Ktil2^T Tb^T,   E^T = U^T - S Wm2^T,   O^T = S Qtil2^T + E^T Pm^T,
        //   S <- S P_C + E^T Khat2,
        // and the decay S P_C runs while the E^T MMAs do, off the state's critical path.  The
        // helper warps turn each chunk's Wm2^T (TMEM) into the bf16 tile the E^T MMA reads (in
        // the slot, over Ktil2) and write o.
        // One thread (warp 12, lane 0) issues every MMA, so that the state warps never wait for
        // an issue queue.  MMA completions: bar_cmma (E^T), bar_pmma[0] (state), bar_o (O^T),
        // bar_rho[1] (Wm2^T); the state warps report the next bf16 state through bar_sbr and a
        // converted E^T (with S decayed) through bar_ecv; the helpers free O^T through
        // bar_rho[0], ring slot b through bar_empty[b], and report a converted Wm2^T tile
        // through bar_wready.
        const int row = quad * 32 + lane;
        constexpr uint32_t COL_WS = COL_O + 64;     // Wm2^T scratch (O^T is single-buffered here)
        uint64_t* bar_e = bar_cmma;
        uint64_t* bar_s = bar_pmma;
        uint64_t* bar_ofree = bar_rho;
        uint64_t* bar_w = bar_rho + 1;
        const uint32_t ID_KK = idesc_bf16(128, 64, 0, 0, 0), ID_NEG = idesc_bf16(128, 64, 0, 1, 1);
        const uint32_t ID_KM128 = idesc_bf16(128, 128, 0, 1, 0), ID_MK = idesc_bf16(128, 64, 1, 0, 0);
        auto sbcol = [](int c) -> uint32_t { return (c & 1) ? COL_AW : COL_SB; };
        auto scale_cols = [&](int col0, float (&s)[16], const float* rho) {
            if (!ROT) {
#pragma unroll
                for (int u4 = 0; u4 < 4; ++u4) {
                    const float4 f = *reinterpret_cast<const float4*>(rho + col0 + 4 * u4);
                    s[4 * u4] *= f.x; s[4 * u4 + 1] *= f.y; s[4 * u4 + 2] *= f.z; s[4 * u4 + 3] *= f.w;
                }
            } else {
#pragma unroll
                for (int u = 0; u < 16; u += 2) {
                    const int pr = (col0 + u) >> 1;
                    const float cr = rho[pr], ci = rho[128 + pr];
                    const float xr = s[u], xi = s[u + 1];
                    s[u] = xr * cr - xi * ci;
                    s[u + 1] = xr * ci + xi * cr;
                }
            }
        };
        // U^T = V^T Tb^T -> E^T buffer of chunk c;  Wm2^T = Ktil2^T Tb^T -> scratch (commit)
        auto issue_slot_mmas = [&](int c) {
            const uint32_t sl = sb + slot_base(c);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t dTb = sdesc_sw128(sl + SL_TB + ks * 32, 16, 1024);
                const uint64_t dTw = sdesc_sw128(sl + (untied ? SL_TW : SL_TB) + ks * 32, 16, 1024);
                mma_bf16_ss(tbase + COL_E + (c & 1) * 64, sdesc_sw128(sl + SL_V + ks * 2048, 8192, 1024), dTw,
                            ID_MK, ks > 0);
                mma_bf16_ss(tbase + COL_WS, sdesc_sw128(sl + SL_W + ks * 2048, 8192, 1024), dTb, ID_MK, ks > 0);
            }
            mma_commit(bar_w);
        };
        if (tid == NPREP + CHAIN_THREADS) {
            // ---------------- MMA issuer ------------------------------------------------------------
            auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
                if (mbar_wait_bounded(bar, parity, x.wait_limit_ns) && *abort_c == 0) return true;
                atomicExch(abort_c, 1);
                return false;
            };
            int u_issued = 0;                 // chunks whose U^T / Wm2^T MMAs have been issued
            for (int c = 0; c < nchunks; ++c) {
                const int b = c & 1;
                const bool last = (c == nchunks - 1);
                const uint32_t sl = sb + slot_base(c);
                if (u_issued <= c) {
                    if (!wait(bar_full + b, (c >> 1) & 1)) break;
                    tc_fence_after();
                    issue_slot_mmas(c);
                    u_issued = c + 1;
                }
                // the state's bf16 copy, this chunk's Wm2^T tile, and O^T read by the helpers
                if (!wait(bar_sbr, c & 1) || !wait(bar_wready, c & 1)) break;
                if (c >= 1 && !wait(bar_ofree, (c - 1) & 1)) break;
                tc_fence_after();
                {   // E^T = U^T - S Wm2^T (commit), O^T = S Qtil2^T
                    const uint32_t a0 = tbase + sbcol(c);
                    const uint64_t dW = sdesc_sw128(sl + SL_W, 8192, 1024), dQ = sdesc_sw128(sl + SL_Q, 16, 1024);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16_ts(tbase + COL_E + b * 64, a0 + ks * 8, dW + (uint64_t)(ks * 2048 / 16), ID_NEG, 1);
                    mma_commit(bar_e);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16_ts(tbase + COL_O, a0 + ks * 8, dQ + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) / 16),
                                    ID_KK, ks > 0);
                }
                if (!wait(bar_ecv, c & 1)) break;
                tc_fence_after();
                {   // S += E^T Khat2 (commit), O^T += E^T Pm^T (commit)
                    const uint64_t dH = sdesc_sw128(sl + SL_KH, 8192, 1024), dP = sdesc_sw128(sl + SL_PM, 16, 1024);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ts(tbase + COL_S, tbase + COL_E + b * 64 + ks * 8, dH + (uint64_t)(ks * 2048 / 16),
                                    ID_KM128, 1);
                    mma_commit(bar_s);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ts(tbase + COL_O, tbase + COL_E + b * 64 + ks * 8, dP + (uint64_t)(ks * 32 / 16), ID_KK, 1);
                    mma_commit(bar_o);
                }
                // the next chunk's U^T and Wm2^T, if its slot is already here
                if (!last && mbar_test_wait(bar_full + (b ^ 1), ((c + 1) >> 1) & 1)) {
                    tc_fence_after();
                    issue_slot_mmas(c + 1);
                    u_issued = c + 2;
                }
            }
        } else if (tid >= NPREP) {
            // ---------------- state warps: one thread per TMEM lane -----------------------------------
            const bool lead = (tid == NPREP);
            auto cbar = [&]() { named_bar(2, CHAIN_THREADS); };
            // MMA completions: one thread waits, the others at the named barrier
            auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
                if (lead && !mbar_wait_bounded(bar, parity, x.wait_limit_ns)) atomicExch(abort_c, 1);
                cbar();
                tc_fence_after();
                return *abort_c == 0;
            };
            if (lead && !mbar_wait_bounded(bar_full + 0, 0, x.wait_limit_ns)) atomicExch(abort_c, 1);
            cbar();
            bool alive = *abort_c == 0;
            if (alive) {
                // S_0 (fp32) and its bf16 copy
#pragma unroll 1
                for (int g = 0; g < 8; ++g) {
                    const int col0 = g * 16;
                    float s[16];
                    if (p.S0) {
                        const float4* src = reinterpret_cast<const float4*>(p.S0 + ((size_t)gbh * D + row) * D + col0);
#pragma unroll
                        for (int u4 = 0; u4 < 4; ++u4) {
                            const float4 t4 = src[u4];
                            s[4 * u4] = t4.x; s[4 * u4 + 1] = t4.y; s[4 * u4 + 2] = t4.z; s[4 * u4 + 3] = t4.w;
                        }
                    } else {
#pragma unroll
                        for (int u = 0; u < 16; ++u) s[u] = 0.f;
                    }
                    tmem_st16(tq + COL_S + col0, s);
                    uint32_t w[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) w[u] = pack_bf16x2(s[2 * u], s[2 * u + 1]);
                    tmem_st8u(tq + COL_SB + (col0 >> 1), w);
                }
                tmem_wait_st();
                tc_fence_before();
                cbar();
                if (lead) mbar_arrive(bar_sbr);
            }
            for (int c = 0; c < nchunks && alive; ++c) {
                const int b = c & 1;
                const bool last = (c == nchunks - 1);
                // ---- S <- S P_C while E^T is formed (no MMA reads or writes S now) ------------
                if (!mbar_wait_bounded(bar_full + b, (c >> 1) & 1, x.wait_limit_ns)) atomicExch(abort_c, 1);
                {
                    const float* rt = reinterpret_cast<const float*>(base + slot_base(c) + SL_VEC) + 64;
#pragma unroll 1
                    for (int g = 0; g < 4; ++g) {
                        float s32[32];
                        tmem_ld32(tq + COL_S + g * 32, s32);
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float s16[16];
#pragma unroll
                            for (int u = 0; u < 16; ++u) s16[u] = s32[hh * 16 + u];
                            scale_cols(g * 32 + hh * 16, s16, rt);
                            tmem_st16(tq + COL_S + g * 32 + hh * 16, s16);
                        }
                    }
                    tmem_wait_st();
                }
                if (!wait_all(bar_e, c & 1)) break;
                // ---- E^T (fp32) -> bf16 in place, as the A operand ----------------------------
                {
                    const uint32_t col = COL_E + b * 64;
                    uint32_t w[32];
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        float vals[32];
                        tmem_ld32(tq + col + g * 32, vals);
#pragma unroll
                        for (int u = 0; u < 16; ++u) w[g * 16 + u] = pack_bf16x2(vals[2 * u], vals[2 * u + 1]);
                    }
#pragma unroll
                    for (int g = 0; g < 4; ++g) tmem_st8u(tq + col + g * 8, *reinterpret_cast<uint32_t(*)[8]>(w + g * 8));
                    tmem_wait_st();
                }
                tc_fence_before();
                cbar();
                if (lead) mbar_arrive(bar_ecv);
                if (!wait_all(bar_s, c & 1)) break;
                // ---- S -> bf16 copy for the next chunk; the last chunk writes S_T --------------
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    float s32[32];
                    tmem_ld32(tq + COL_S + g * 32, s32);
                    if (last) {
                        if (p.S_T && GDR_INB(gbh < p.B * p.H, 601)) {
                            float4* dst = reinterpret_cast<float4*>(p.S_T + ((size_t)gbh * D + row) * D + g * 32);
#pragma unroll
                            for (int u4 = 0; u4 < 8; ++u4)
                                dst[u4] = make_float4(s32[4 * u4], s32[4 * u4 + 1], s32[4 * u4 + 2], s32[4 * u4 + 3]);
                        }
                    } else {
                        uint32_t w[16];
#pragma unroll
                        for (int u = 0; u < 16; ++u) w[u] = pack_bf16x2(s32[2 * u], s32[2 * u + 1]);
                        tmem_st8u(tq + sbcol(c + 1) + g * 16, *reinterpret_cast<uint32_t(*)[8]>(w));
                        tmem_st8u(tq + sbcol(c + 1) + g * 16 + 8, *reinterpret_cast<uint32_t(*)[8]>(w + 8));
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                cbar();
                if (lead && !last) mbar_arrive(bar_sbr);
            }
        } else {
            // ---------------- helpers: Wm2^T tiles and o --------------------------------------------
            const int et = tid - (NPREP - 128);
            auto ebar = [&]() { named_bar(4, 128); };
            OT* stg = reinterpret_cast<OT*>(base + OFF_OSTG);
            // Wm2^T of chunk c (lane = dk row, 64 token columns) -> bf16 MN-major tile over Ktil2
            auto convert_w = [&](int c) -> bool {
                if (et == 0 && !mbar_wait_bounded(bar_w, c & 1, x.wait_limit_ns)) atomicExch(abort_c, 1);
                ebar();
                if (*abort_c) return false;
                tc_fence_after();
                uint8_t* W = base + slot_base(c) + SL_W;
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float vals[32];
                    tmem_ld32(tq + COL_WS + g * 32, vals);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        *reinterpret_cast<uint4*>(W + sw128_off(row, g * 4 + cc)) = pack8(vals + cc * 8);
                }
                tc_fence_before();
                fence_proxy_async_smem();
                ebar();
                if (et == 0) mbar_arrive(bar_wready);
                return true;
            };
            bool ok = convert_w(0);
            for (int c = 0; c < nchunks && ok; ++c) {
                const int b = c & 1;
                if (et == 0 && !mbar_wait_bounded(bar_o, c & 1, x.wait_limit_ns)) atomicExch(abort_c, 1);
                ebar();
                if (*abort_c) break;
                tc_fence_after();
                if (et == 0) {
                    mbar_arrive(bar_empty + b);     // every MMA that read ring slot b is done
                    bulk_wait_read_all();           // the previous o store has read the staging
                }
                ebar();
                float msum = 0.f;       // this value row's sum over the chunk's tokens
#pragma unroll 1
                for (int g = 0; g < 2; ++g) {
                    float vals[32];
                    tmem_ld32(tq + COL_O + g * 32, vals);
#pragma unroll
                    for (int u = 0; u < 32; ++u) st_from_f32(stg + (g * 32 + u) * D + row, vals[u]);
                    if (cmean) {
                        const int Lg = chunk_len(c) - g * 32;    // tokens of this half inside T
#pragma unroll
                        for (int u = 0; u < 32; ++u) msum += (u < Lg) ? vals[u] : 0.f;
                    }
                }
                if (cmean) *cmean_at(gbh, c, row) = msum / (float)chunk_len(c);
                tc_fence_before();
                fence_proxy_async_smem();
                ebar();
                if (et == 0) {
                    mbar_arrive(bar_ofree);
                    tma_store_4d(&tm.o, 0, gbh % p.H, c * C, gbh / p.H, sb + OFF_OSTG);   // rows past T clipped
                    bulk_commit();
                }
                if (c + 1 < nchunks) ok = convert_w(c + 1);
            }
            if (et == 0) bulk_wait_all();
        }
    } else if (MODE == 0 && nchunks > 0 && tid >= NPREP && tid < NPREP + CHAIN_THREADS && chain_cta) {
        // =========================== chain group ==================================
        const int row = tid - NPREP;          // TMEM lane = value row of S (quad = warp & 3)
        uint32_t mma_phase = 0;
        const uint32_t ID_KK = idesc_bf16(128, 64, 0, 0, 0), ID_NEG = idesc_bf16(128, 64, 0, 1, 1);
        const uint32_t ID_KM128 = idesc_bf16(128, 128, 0, 1, 0);
        auto cbar = [&]() { named_bar(2, CHAIN_THREADS); };
        auto mma_wait = [&]() -> bool {      // one thread waits, the others at the barrier
            if (row == 0 && !mbar_wait_bounded(bar_cmma, mma_phase, x.wait_limit_ns)) atomicExch(abort_c, 1);
            mma_phase ^= 1u;
            cbar();
            tc_fence_after();
            return *abort_c == 0;
        };
        auto bounded = [&](uint64_t* bar, uint32_t parity) -> bool {
            const bool ok = mbar_wait_bounded(bar, parity, x.wait_limit_ns);
            if (!ok) atomicExch(abort_c, 1);
            cbar();
            return *abort_c == 0;
        };
        // Write 16 state columns as fp32 (S) and bf16 (Stil); s holds S * rho.
        auto store_state = [&](int col0, const float (&s)[16]) {
            tmem_st16(tq + COL_S + col0, s);
            uint32_t w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) w[u] = pack_bf16x2(s[2 * u], s[2 * u + 1]);
            tmem_st8u(tq + COL_SB + (col0 >> 1), w);
        };
        auto scale_cols = [&](int col0, float (&s)[16], const float* rho) {
            if (!ROT) {
#pragma unroll
                for (int u4 = 0; u4 < 4; ++u4) {
                    const float4 f = *reinterpret_cast<const float4*>(rho + col0 + 4 * u4);
                    s[4 * u4] *= f.x; s[4 * u4 + 1] *= f.y; s[4 * u4 + 2] *= f.z; s[4 * u4 + 3] *= f.w;
                }
            } else {
#pragma unroll
                for (int u = 0; u < 16; u += 2) {
                    const int pr = (col0 + u) >> 1;
                    const float cr = rho[pr], ci = rho[128 + pr];
                    const float xr = s[u], xi = s[u + 1];
                    s[u] = xr * cr - xi * ci;
                    s[u + 1] = xr * ci + xi * cr;
                }
            }
        };
        // o for one chunk: O^T sits in TMEM with lane = value row, column = token.  Each 8x8
        // block (8 value rows of this warp x 8 tokens) is transposed across 8 lanes so that
        // every lane stores 8 consecutive value columns of one token (16 bytes in bf16).
        auto o_epilogue = [&](int c) {
            const int Lc = chunk_len(c);
            const uint32_t col = COL_O + (c & 1) * 64;
            const int j8 = lane & 7, grp = lane >> 3;
            OT* obase = o + tok(c, 0) * D + quad * 32 + grp * 8;
            const size_t tstride = (size_t)p.H * D;
            float msum = 0.f;           // this value row's sum over the chunk's tokens
#pragma unroll 1
            for (int g = 0; g < 2; ++g) {
                float vals[32];
                tmem_ld32(tq + col + g * 32, vals);
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
                    if (r < Lc) {
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
            if (cmean) *cmean_at(gbh, c, row) = msum / (float)Lc;
        };

        // Initial state, prescaled by the first chunk's reference decay.
        bool alive = bounded(bar_rho + 0, 0);
        if (alive) {
            const float* rho_ref0 = vecs(0) + 64;
#pragma unroll 1
            for (int g = 0; g < 8; ++g) {
                const int col0 = g * 16;
                float s[16];
                if (p.S0) {
                    const float4* src = reinterpret_cast<const float4*>(p.S0 + ((size_t)gbh * D + row) * D + col0);
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4) {
                        const float4 t4 = src[u4];
                        s[4 * u4] = t4.x; s[4 * u4 + 1] = t4.y; s[4 * u4 + 2] = t4.z; s[4 * u4 + 3] = t4.w;
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 16; ++u) s[u] = 0.f;
                }
                scale_cols(col0, s, rho_ref0);
                store_state(col0, s);
            }
            tmem_wait_st();
            tc_fence_before();
        }
        for (int c = 0; c < nchunks && alive; ++c) {
            const int bufi = c & 1;
            const bool last = (c == nchunks - 1);
            if (!bounded(bar_full + bufi, (c >> 1) & 1)) break;
            tc_fence_after();
            // ---- E^T += -Stil Wm^T ;  O^T = Stil Qtil^T --------------------------------
            if (row == 0) {
                const uint64_t dW = sdesc_sw128(sb + OFF_W + bufi * 16384, 8192, 1024);
                const uint64_t dQ = sdesc_sw128(sb + OFF_KQ + bufi * 32768 + 8192, 16, 1024);
                const uint32_t qkb = 16384u;                         // K-block stride of the Qtil tile
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t a_t = tbase + COL_SB + ks * 8;
                    // descriptor start addresses advance in 16-byte units
                    mma_bf16_ts(tbase + COL_E + bufi * 64, a_t, dW + (uint64_t)(ks * 2048 / 16), ID_NEG, 1);
                    mma_bf16_ts(tbase + COL_O + bufi * 64, a_t,
                                dQ + (uint64_t)(((ks >> 2) * qkb + (ks & 3) * 32) / 16), ID_KK, ks > 0);
                }
                mma_commit(bar_cmma);
            }
            if (c > 0) o_epilogue(c - 1);          // overlaps the MMAs above
            if (!mma_wait()) break;

            // ---- E^T (fp32) -> bf16 in place, as the A operand ---------------------------
            {
                const uint32_t col = COL_E + bufi * 64;
                uint32_t w[32];
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float vals[32];
                    tmem_ld32(tq + col + g * 32, vals);
#pragma unroll
                    for (int u = 0; u < 16; ++u) w[g * 16 + u] = pack_bf16x2(vals[2 * u], vals[2 * u + 1]);
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) tmem_st8u(tq + col + g * 8, *reinterpret_cast<uint32_t(*)[8]>(w + g * 8));
                tmem_wait_st();
            }
            tc_fence_before();
            cbar();
            tc_fence_after();
            // ---- O^T += E^T Pm^T ;  S_acc += E^T Khat ---------------------------------------
            if (row == 0) {
                const uint64_t dP = sdesc_sw128(sb + OFF_PM + bufi * 8192, 16, 1024);
                const uint64_t dH = sdesc_sw128(sb + OFF_KH + bufi * 16384, 8192, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint32_t a_t = tbase + COL_E + bufi * 64 + ks * 8;
                    mma_bf16_ts(tbase + COL_O + bufi * 64, a_t, dP + (uint64_t)(ks * 32 / 16), ID_KK, 1);
                    mma_bf16_ts(tbase + COL_S, a_t, dH + (uint64_t)(ks * 2048 / 16), ID_KM128, 1);
                }
                mma_commit(bar_cmma);
            }
            if (!mma_wait()) break;

            // ---- S <- S_acc (P_m^{-1} P_C), then prescale by the next reference ----------
            if (!last && !bounded(bar_rho + ((c + 1) & 1), ((c + 1) >> 1) & 1)) break;
            {
                const float* rho_C = vecs(c) + 64 + 256;
                const float* rho_nx = vecs(c + 1) + 64;
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    const int col0 = g * 32;
                    float s32[32];
                    tmem_ld32(tq + COL_S + col0, s32);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float s[16];
#pragma unroll
                        for (int u = 0; u < 16; ++u) s[u] = s32[hh * 16 + u];
                        const int c16 = col0 + hh * 16;
                        scale_cols(c16, s, rho_C);
                        if (last) {
                            if (p.S_T && GDR_INB(gbh < p.B * p.H, 602)) {
                                float4* dst = reinterpret_cast<float4*>(p.S_T + ((size_t)gbh * D + row) * D + c16);
#pragma unroll
                                for (int u4 = 0; u4 < 4; ++u4)
                                    dst[u4] = make_float4(s[4 * u4], s[4 * u4 + 1], s[4 * u4 + 2], s[4 * u4 + 3]);
                            }
                        } else {
                            scale_cols(c16, s, rho_nx);
                            store_state(c16, s);
                        }
                    }
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_empty + bufi);
            if (last) o_epilogue(c);
        }
    }

    if (MODE == 1 && nchunks > 0 && chain_cta && warp == 0) {
        // ============ split mode: loader of the chain CTA (one warp, lane 0 issues) ============
        for (int c = 0; c < nchunks; ++c) {
            const int bufi = c & 1;
            bool ok = true;
            if (lane == 0) {
                // the chain must be done with chunk c - 2 before its buffer is refilled
                if (c >= 2) ok = mbar_wait_bounded(bar_empty + bufi, ((c - 2) >> 1) & 1, x.wait_limit_ns);
                const int slot = c % RING;
                if (ok) ok = spin_until_ge(sa.ready + (size_t)bh * RING + slot, (unsigned)(c + 1), x.wait_limit_ns);
                if (ok) {
                    fence_proxy_async_global();
                    const uint8_t* src = sa.ring + ((size_t)bh * RING + slot) * SLOT_BYTES;
                    // the tiles (Tw only with a separate write strength), the vectors, and V
                    const uint32_t tiles = untied ? SL_VEC : SL_TW;
                    mbar_arrive_expect_tx(bar_full + bufi, tiles + (SLOT_BYTES - SL_VEC) + 16384u);
                    for (uint32_t off = 0; off < tiles; off += 16384u) {
                        const uint32_t n = tiles - off < 16384u ? tiles - off : 16384u;
                        bulk_g2s(sb + slot_base(c) + off, src + off, n, bar_full + bufi);
                    }
                    bulk_g2s(sb + slot_base(c) + SL_VEC, src + SL_VEC, SLOT_BYTES - SL_VEC, bar_full + bufi);
                    // V of this chunk, two 64-column boxes straight into the MN-major layout
                    const int bb = gbh / p.H, hh = gbh % p.H;
                    tma_load_4d(sb + slot_base(c) + SL_V, &tm.v, 0, hh, c * C, bb, bar_full + bufi);
                    tma_load_4d(sb + slot_base(c) + SL_V + 8192u, &tm.v, 64, hh, c * C, bb, bar_full + bufi);
                    ok = mbar_wait_bounded(bar_full + bufi, (c >> 1) & 1, x.wait_limit_ns);
                }
                if (!ok) atomicExch(abort_p, 1);
            }
            if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) break;
            // The slot's bytes have landed here: its L2 lines are dead, so they are dropped
            // without a write-back; then the slot may be reused.
            if (sa.discard) {
                const uint8_t* src = sa.ring + ((size_t)bh * RING + c % RING) * SLOT_BYTES;
                for (uint32_t off = (uint32_t)lane * 128u; off < SLOT_BYTES; off += 32u * 128u) discard_l2_line(src + off);
                __syncwarp();
            }
            if (lane == 0) st_release_gpu(sa.consumed + bh, (unsigned)(c + 1));
        }
    }
    if (nchunks == 0 && p.S_T && chain_cta && GDR_INB(gbh < p.B * p.H, 603)) {
        for (int e = tid; e < D * D; e += nthreads<MODE>())
            p.S_T[(size_t)gbh * D * D + e] = p.S0 ? p.S0[(size_t)gbh * D * D + e] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        unsigned bits = 0;
        if (*abort_p || *abort_c) bits |= STATUS_TIMEOUT;
        if (*range_flag) bits |= STATUS_RANGE;
        if (bits) atomicOr(&g_device_status, bits);
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

}  // namespace tcf
}  // namespace gdr
