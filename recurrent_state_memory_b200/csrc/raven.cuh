// raven.cuh -- Raven's routed slot memory: the chunked forward ("Raven: High-Recall Sequence
// Modeling with Sparse Memory Routing" page, sections 2.1 and 2.2).
//
// Per (batch, head): M = 64 slots, a key state Sk and a value state Sv (M x D each).  Token t:
//   router: the top K of the logits z_t (ties to the lower slot), m = sigmoid of the kept ones,
//           r_t[i] = m_i / sum of the kept m (zero on the other slots);
//   decay and write on the chosen slots only, with a_t = log-decay of the gate:
//           S[i] <- e^{a_t r_t[i]} S[i] + (1 - e^{a_t r_t[i]}) x_t     (x = k for Sk, v for Sv)
//   readout over the updated slots: o_t = sum_i softmax_i(scale q_t . Sk[i]) Sv[i].
// Chunked form (C = 32 tokens, start states Sk0 / Sv0, lam_t[i] the slot's cumulative log-decay
// over the chunk's tokens u <= t, c_s[i] = 1 - e^{a_s r_s[i]}):
//   scores[t,i] = scale e^{lam_t[i]} q_t . Sk0[i] + sum_{s <= t chose i} A[t,s] c_s[i] e^{lam_t[i] - lam_s[i]}
//                 with A = scale Q K^T                                         (tensor cores + sparse)
//   P = softmax over the slots;  PE = P e^{lam};  Bm[t,s] = sum_{i chosen at s} P[t,i] c_s[i] e^{lam_t[i] - lam_s[i]}
//   O = PE Sv0 + Bm V                                                          (tensor cores)
//   S_L[i] = e^{lam_L[i]} S0[i] + sum_{s chose i} c_s[i] e^{lam_L[i] - lam_s[i]} x_s   (fp32, sparse)
// Every exponent is <= 0.  The sums over the chunk's writes run over each slot's tokens in
// token order (a 32-bit mask per slot: bit t set when token t chose the slot), so the results
// do not depend on thread timing; the per-token tables are kept slot-major so that a warp reads
// a slot's tokens from one row.
//
// Sequence parallelism: the transition of a chunk is diagonal in the slots, so a run of chunks
// maps its start state to e^{Lam} S + W (per slot).  A state pass runs the chunks before the
// last output segment, cut into units shorter than a segment (so that its CTAs fill the SMs),
// each from the zero state (W, Lam into the workspace); the output pass then starts segment g
// from S0 composed, in order, with every unit before it.
//
// The router runs first, for every token at once (`raven_route_kernel`: one warp per token and
// head, the whole GPU busy), and leaves each token's chosen slots and weights in the workspace.
// Then one 512-thread CTA per (head, segment) and about 205 KB of shared memory at D = 128: the
// fp32 states, their bf16 copies (the MMA operands), double-buffered q / k / v tiles and routing
// records of the next chunk (cp.async, zero-filled past T), and the chunk's tables.
#pragma once

#include "common.cuh"

namespace gdr {
namespace rvn {

constexpr int C = 32;          // tokens per chunk
constexpr int M = 64;          // slots
constexpr int KMAX = 16;       // largest top-K
constexpr int NT = 512;
constexpr int NW = NT / 32;
static_assert(NT == C * M / 4 && NT == 8 * M && NW == C / 2 && C == 32, "thread mappings below (a token per lane)");

struct RavenParams {
    int B, H, T, K, gate_mode;
    float scale;
    const __nv_bfloat16* q;   // [B,T,H,D]
    const __nv_bfloat16* k;   // [B,T,H,D]
    const __nv_bfloat16* v;   // [B,T,H,D]
    const float* z;           // [B,T,H,M] router logits
    const float* g;           // [B,T,H] decay gate
    const float* S0k;         // [B,H,M,D] or nullptr (zero)
    const float* S0v;         // [B,H,M,D] or nullptr (zero)
    void* o;                  // [B,T,H,D]
    float* SkT;               // [B,H,M,D] or nullptr
    float* SvT;               // [B,H,M,D] or nullptr
    int nseg, seg_chunks;     // output segments per sequence, chunks per segment
    int nsub, sub_chunks;     // state units per sequence (covering the segments before the last),
                              // chunks per unit (a divisor of seg_chunks)
    float* segW;              // [B*H][nsub][2][M][D]: each unit's end states from zero
    float* segL;              // [B*H][nsub][M]: each unit's total log-decay per slot
    unsigned char* route;     // [B*T*H][ROUTE_BYTES]: each token's chosen slots and weights
};

// A token's routing record: the chosen slots (in the order chosen), then a_t r_t[i] and
// c = 1 - e^{a_t r_t[i]} for each of them.
constexpr int ROUTE_BYTES = KMAX + 2 * 4 * KMAX;     // 144
constexpr int ROUTE_LR = KMAX, ROUTE_C = KMAX + 4 * KMAX;

// Shared-memory layout (byte offsets).
template <int D>
struct Sm {
    static constexpr int DP = D + 8;                       // bf16 row stride of tiles and copies
    static constexpr size_t SKF = 0;                       // fp32 [M][D]
    static constexpr size_t SVF = SKF + (size_t)M * D * 4;
    static constexpr size_t SKB = SVF + (size_t)M * D * 4; // bf16 [M][DP]
    static constexpr size_t SVB = SKB + (size_t)M * DP * 2;
    static constexpr size_t QT = SVB + (size_t)M * DP * 2; // bf16 [2][C][DP]
    static constexpr size_t KT = QT + 2ull * C * DP * 2;
    static constexpr size_t VT = KT + 2ull * C * DP * 2;
    static constexpr size_t RT = VT + 2ull * C * DP * 2;   // [2][C][ROUTE_BYTES] routing records
    static constexpr int CS = C + 1;                       // row stride of the slot-major tables
    static constexpr size_t LAMT = RT + 2ull * C * ROUTE_BYTES;   // fp32 [M][CS]: a r, then lam (slot-major)
    static constexpr size_t CT = LAMT + (size_t)M * CS * 4;     // fp32 [M][CS]: c (valid where chosen)
    static constexpr size_t SC = CT + (size_t)M * CS * 4;  // fp32 [C][M + 4]: scores, then P
    static constexpr size_t AB = SC + (size_t)C * (M + 4) * 4;   // fp32 [C][C + 4]: A
    static constexpr size_t PEB = AB + (size_t)C * (C + 4) * 4;  // bf16 [C][M + 8]: P e^{lam}
    static constexpr size_t BB = PEB + (size_t)C * (M + 8) * 2;  // bf16 [C][C + 8]: Bm
    static constexpr size_t PS = BB + (size_t)C * (C + 8) * 2;   // fp32 [8][M]: scan parts
    static constexpr size_t MSK = PS + 8ull * M * 4;             // u32 [2][M]: tokens that chose the slot
    static constexpr size_t SEL = MSK + 2ull * M * 4;            // u8 [C][KMAX]: chosen slots per token
    static constexpr size_t LTOT = SEL + (size_t)C * KMAX;       // fp32 [M]: summed log-decay (state pass)
    static constexpr size_t BYTES = LTOT + (size_t)M * 4;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool ok) {
    const unsigned n = ok ? 16u : 0u;     // 0: the 16 bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
// d += a b for one m16n8k16 bf16 tile (fp32 accumulators)
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// CPL consecutive fp32 / bf16 values of one state row (CPL = 4 or 2).
template <int CPL> struct Vec;
template <> struct Vec<4> {
    __device__ static void ld(float (&x)[4], const float* p) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    __device__ static void st(float* p, const float (&x)[4]) { *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]); }
    __device__ static void ldb(float (&x)[4], const __nv_bfloat16* p) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    }
    __device__ static void stb(__nv_bfloat16* p, const float (&x)[4]) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t*>(&a);
        u.y = *reinterpret_cast<const uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = u;
    }
};
template <> struct Vec<2> {
    __device__ static void ld(float (&x)[2], const float* p) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x[0] = v.x; x[1] = v.y;
    }
    __device__ static void st(float* p, const float (&x)[2]) { *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]); }
    __device__ static void ldb(float (&x)[2], const __nv_bfloat16* p) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
        x[0] = a.x; x[1] = a.y;
    }
    __device__ static void stb(__nv_bfloat16* p, const float (&x)[2]) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(x[0], x[1]);
    }
};

// Order-preserving map of a float to an unsigned key (-0 taken as +0; every non-NaN float maps
// above 0, which marks a slot already taken).
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp's 16 x 16 tile of A (row-major, stride lda elements) times B given as N rows of K
// (row-major, stride ldb: the "col" operand), over kk = 0 .. K in steps of 16.
__device__ __forceinline__ void tile_nt(float (&acc)[2][4], const __nv_bfloat16* A, int lda, const __nv_bfloat16* Bn,
                                        int ldb, int K) {
    const int lane = (int)threadIdx.x & 31;
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[4], b[4];
        ldsm_x4(a, A + (lane & 15) * lda + k0 + (lane >> 4) * 8);
        ldsm_x4(b, Bn + ((lane & 7) + ((lane >> 4) << 3)) * ldb + k0 + ((lane >> 3) & 1) * 8);
        mma_bf16(acc[0], a, b[0], b[1]);
        mma_bf16(acc[1], a, b[2], b[3]);
    }
}
// The same with B given as K rows of N (row-major, stride ldb), read transposed.
__device__ __forceinline__ void tile_nn(float (&acc)[2][4], const __nv_bfloat16* A, int lda, const __nv_bfloat16* Bk,
                                        int ldb, int K) {
    const int lane = (int)threadIdx.x & 31;
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[4], b[4];
        ldsm_x4(a, A + (lane & 15) * lda + k0 + (lane >> 4) * 8);
        ldsm_x4_t(b, Bk + (k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ldb + (lane >> 4) * 8);
        mma_bf16(acc[0], a, b[0], b[1]);
        mma_bf16(acc[1], a, b[2], b[3]);
    }
}

// The router of every token, one warp per (token, head), before the chunked passes: K rounds of
// a warp-wide maximum of order-preserving keys of the fp32 logits (one redux each), the lowest
// slot index among equal keys taken by two ballots (slots lane < slots lane + 32); then the
// kept sigmoid scores normalised, a_t r_t and c = 1 - e^{a_t r_t} per chosen slot.
__global__ void __launch_bounds__(256) raven_route_kernel(RavenParams p) {
    const int lane = (int)threadIdx.x & 31;
    const long long n_tok = (long long)p.B * p.T * p.H;
    const long long W = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long n = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < n_tok; n += W) {
        const float* zr = p.z + n * M;
        uint32_t u0 = order_key(zr[lane]), u1 = order_key(zr[lane + 32]);
        int my_i = 0;
        for (int j = 0; j < p.K; ++j) {
            const bool first = u0 >= u1;
            const uint32_t cand = first ? u0 : u1;
            const uint32_t mx = __reduce_max_sync(0xffffffffu, cand);
            const uint32_t b0 = __ballot_sync(0xffffffffu, cand == mx && first);
            const uint32_t b1 = __ballot_sync(0xffffffffu, cand == mx && !first);
            const int win = b0 ? __ffs(b0) - 1 : 32 + __ffs(b1) - 1;
            if (win == lane) u0 = 0u;
            if (win == lane + 32) u1 = 0u;
            if (lane == j) my_i = win;
        }
        const float m = lane < p.K ? 1.f / (1.f + expf(-zr[my_i])) : 0.f;
        float sum = m;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane < p.K && GDR_INB(n < n_tok, 703)) {
            unsigned char* rec = p.route + n * ROUTE_BYTES;
            const float lr = log_decay(p.g[n], p.gate_mode) * (m / sum);
            rec[lane] = (unsigned char)my_i;
            reinterpret_cast<float*>(rec + ROUTE_LR)[lane] = lr;
            reinterpret_cast<float*>(rec + ROUTE_C)[lane] = -expm1f(lr);
        }
    }
}

// FULL = false: the state pass (segment from the zero state; end state and summed log-decay to
// the workspace).  FULL = true: the output pass.
template <int D, bool FULL, typename OT>
__global__ void __launch_bounds__(NT, 1) raven_fwd_kernel(RavenParams p) {
    using L = Sm<D>;
    constexpr int DP = L::DP;
    extern __shared__ float4 sm4[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(sm4);
    float* Skf = reinterpret_cast<float*>(sm + L::SKF);
    float* Svf = reinterpret_cast<float*>(sm + L::SVF);
    __nv_bfloat16* Skb = reinterpret_cast<__nv_bfloat16*>(sm + L::SKB);
    __nv_bfloat16* Svb = reinterpret_cast<__nv_bfloat16*>(sm + L::SVB);
    float* lamT = reinterpret_cast<float*>(sm + L::LAMT);
    float* cT = reinterpret_cast<float*>(sm + L::CT);
    uint32_t* mskb = reinterpret_cast<uint32_t*>(sm + L::MSK);
    constexpr int CS = L::CS;
    float* sc = reinterpret_cast<float*>(sm + L::SC);
    float* ab = reinterpret_cast<float*>(sm + L::AB);
    __nv_bfloat16* peb = reinterpret_cast<__nv_bfloat16*>(sm + L::PEB);
    __nv_bfloat16* bb = reinterpret_cast<__nv_bfloat16*>(sm + L::BB);
    float* ps = reinterpret_cast<float*>(sm + L::PS);
    unsigned char* sel = sm + L::SEL;
    float* ltot = reinterpret_cast<float*>(sm + L::LTOT);
    constexpr int SCS = M + 4, ABS = C + 4, PES = M + 8, BBS = C + 8;

    const int tid = (int)threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nsegw = FULL ? p.nseg : p.nsub;
    const int hd = (int)blockIdx.x / nsegw, seg = (int)blockIdx.x % nsegw;
    const int b = hd / p.H, h = hd % p.H;
    if (!GDR_INB(hd < p.B * p.H, 701)) return;
    const int nc = (p.T + C - 1) / C;
    const int span = FULL ? p.seg_chunks : p.sub_chunks;
    const int c_begin = seg * span, c_end = min(nc, c_begin + span);
    const size_t MD = (size_t)M * D;
    auto tokrow = [&](int t) -> size_t { return ((size_t)b * p.T + t) * p.H + h; };

    // State rows: warp w owns slots w, w + 16, w + 32, w + 48; lane l the CPL columns from
    // l * CPL (consecutive: conflict-free vector accesses to shared memory).
    constexpr int CPL = D / 32;
    using V = Vec<CPL>;
    const int c0 = lane * CPL;

    // ---- start state: S0 (output pass) composed with the earlier segments, or zero ----
    for (int si = 0; si < M / NW; ++si) {
        const int i = warp + NW * si;
        float ak[CPL] = {}, av[CPL] = {};
        if (FULL && p.S0k) V::ld(ak, p.S0k + (size_t)hd * MD + (size_t)i * D + c0);
        if (FULL && p.S0v) V::ld(av, p.S0v + (size_t)hd * MD + (size_t)i * D + c0);
        if (FULL)
            for (int s2 = 0; s2 < seg * (p.seg_chunks / p.sub_chunks); ++s2) {
                const size_t base = ((size_t)hd * p.nsub + s2);
                const float dk = expf(p.segL[base * M + i]);
                float wk[CPL], wv[CPL];
                V::ld(wk, p.segW + base * 2 * MD + (size_t)i * D + c0);
                V::ld(wv, p.segW + base * 2 * MD + MD + (size_t)i * D + c0);
#pragma unroll
                for (int u = 0; u < CPL; ++u) {
                    ak[u] = dk * ak[u] + wk[u];
                    av[u] = dk * av[u] + wv[u];
                }
            }
        V::st(Skf + i * D + c0, ak);
        V::st(Svf + i * D + c0, av);
        V::stb(Skb + i * DP + c0, ak);
        V::stb(Svb + i * DP + c0, av);
    }
    if (tid < M) ltot[tid] = 0.f;
    if (tid < 2 * M) mskb[tid] = 0u;

    // ---- chunk inputs: asynchronous copies into buffer `buf` ----
    auto load_chunk = [&](int c, int buf) {
        const int t0 = c * C;
        constexpr int PR = D / 8;                      // 16-byte pieces per bf16 row
        __nv_bfloat16* qd = reinterpret_cast<__nv_bfloat16*>(sm + L::QT) + (size_t)buf * C * DP;
        __nv_bfloat16* kd = reinterpret_cast<__nv_bfloat16*>(sm + L::KT) + (size_t)buf * C * DP;
        __nv_bfloat16* vd = reinterpret_cast<__nv_bfloat16*>(sm + L::VT) + (size_t)buf * C * DP;
        for (int i = tid; i < C * PR; i += NT) {
            const int r = i / PR, pc = (i % PR) * 8;
            const bool ok = t0 + r < p.T;
            const size_t src = (ok ? tokrow(t0 + r) : 0) * D + pc;
            if (FULL) cp_async16(qd + r * DP + pc, p.q + src, ok);
            cp_async16(kd + r * DP + pc, p.k + src, ok);
            cp_async16(vd + r * DP + pc, p.v + src, ok);
        }
        unsigned char* rd = sm + L::RT + (size_t)buf * C * ROUTE_BYTES;
        for (int i = tid; i < C * (ROUTE_BYTES / 16); i += NT) {
            const int r = i / (ROUTE_BYTES / 16), pc = (i % (ROUTE_BYTES / 16)) * 16;
            const bool ok = t0 + r < p.T;
            cp_async16(rd + r * ROUTE_BYTES + pc, p.route + (ok ? tokrow(t0 + r) : 0) * ROUTE_BYTES + pc, ok);
        }
        cp_commit();
    };

    if (c_begin < c_end) load_chunk(c_begin, 0);
    for (int c = c_begin; c < c_end; ++c) {
        const int buf = (c - c_begin) & 1, t0 = c * C;
        cp_wait_all();
        __syncthreads();                                            // inputs of chunk c landed
        if (c + 1 < c_end) load_chunk(c + 1, buf ^ 1);
        const __nv_bfloat16* qt = reinterpret_cast<const __nv_bfloat16*>(sm + L::QT) + (size_t)buf * C * DP;
        const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(sm + L::KT) + (size_t)buf * C * DP;
        const __nv_bfloat16* vt = reinterpret_cast<const __nv_bfloat16*>(sm + L::VT) + (size_t)buf * C * DP;
        const unsigned char* rt = sm + L::RT + (size_t)buf * C * ROUTE_BYTES;

        // Slot i's tokens: bit t of msk[i]; its tables lamT[i][t], cT[i][t] hold values only there.
        uint32_t* msk = mskb + buf * M;
        if (tid < M) mskb[(buf ^ 1) * M + tid] = 0u;               // for chunk c + 1
        // ---- the chunk's routing (computed by raven_route_kernel): into the slot-major tables ----
        {
            const int t = tid >> 4, j = tid & 15;                   // 32 tokens x 16 entries
            if (j < p.K && t0 + t < p.T) {                          // padding chooses nothing
                const unsigned char* rr = rt + t * ROUTE_BYTES;
                const int i = rr[j];
                lamT[i * CS + t] = reinterpret_cast<const float*>(rr + ROUTE_LR)[j];
                cT[i * CS + t] = reinterpret_cast<const float*>(rr + ROUTE_C)[j];
                atomicOr(&msk[i], 1u << t);
                sel[t * KMAX + j] = (unsigned char)i;
            }
        }
        __syncthreads();
        // ---- cumulative log-decay per slot (8 parts of 4 tokens) ----
        {
            const int i = tid & (M - 1), part = tid >> 6;
            const uint32_t mk = msk[i];
            float run = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if ((mk >> (part * 4 + u)) & 1u) run += lamT[i * CS + part * 4 + u];
            ps[part * M + i] = run;
            __syncthreads();
            float acc = 0.f;
            for (int pp = 0; pp < part; ++pp) acc += ps[pp * M + i];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = part * 4 + u;
                if ((mk >> t) & 1u) acc += lamT[i * CS + t];
                lamT[i * CS + t] = acc;
            }
        }
        __syncthreads();

        if (FULL) {
            // ---- A = scale Q K^T (4 tiles) and the state's scores scale e^{lam} Q Sk0^T (8 tiles) ----
            if (warp < 12) {
                const bool isA = warp < 4;
                const int tm = isA ? warp >> 1 : (warp - 4) >> 2, tn = isA ? warp & 1 : (warp - 4) & 3;
                float acc[2][4] = {};
                tile_nt(acc, qt + tm * 16 * DP, DP, (isA ? kt : Skb) + tn * 16 * DP, DP, D);
                const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = tm * 16 + gid + ((e >> 1) << 3), col = tn * 16 + hh * 8 + 2 * tig + (e & 1);
                        if (isA) ab[r * ABS + col] = p.scale * acc[hh][e];
                        else sc[r * SCS + col] = p.scale * acc[hh][e] * __expf(lamT[col * CS + r]);
                    }
            }
            __syncthreads();
            // ---- the chunk's own writes in the scores ----
            {
                const int i = tid & (M - 1), tq = tid >> 6;
                const uint32_t mk = msk[i];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t = tq + 8 * u;
                    const float lt = lamT[i * CS + t];
                    float acc = 0.f;
                    for (uint32_t m = mk & ((2u << t) - 1u); m; m &= m - 1u) {      // tokens s <= t
                        const int s = __ffs(m) - 1;
                        acc += ab[t * ABS + s] * cT[i * CS + s] * __expf(lt - lamT[i * CS + s]);
                    }
                    sc[t * SCS + i] += acc;
                }
            }
            __syncthreads();
            // ---- softmax over the slots; P e^{lam} as the bf16 operand of the state's output ----
            for (int t = warp; t < C; t += NW) {
                const float x0 = sc[t * SCS + lane], x1 = sc[t * SCS + lane + 32];
                float mx = fmaxf(x0, x1);
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float e0 = expf(x0 - mx), e1 = expf(x1 - mx);
                float s = e0 + e1;
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                const float p0 = e0 / s, p1 = e1 / s;
                sc[t * SCS + lane] = p0;
                sc[t * SCS + lane + 32] = p1;
                peb[t * PES + lane] = __float2bfloat16_rn(p0 * __expf(lamT[lane * CS + t]));
                peb[t * PES + lane + 32] = __float2bfloat16_rn(p1 * __expf(lamT[(lane + 32) * CS + t]));
            }
            __syncthreads();
            // ---- Bm[t,s] over the K slots token s chose ----
            {
                const int t = tid >> 4;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int s = (tid & 15) + 16 * u;
                    float acc = 0.f;
                    if (s <= t && t0 + s < p.T)
                        for (int j = 0; j < p.K; ++j) {
                            const int i = sel[s * KMAX + j];
                            acc += sc[t * SCS + i] * cT[i * CS + s] * __expf(lamT[i * CS + t] - lamT[i * CS + s]);
                        }
                    bb[t * BBS + s] = __float2bfloat16_rn(acc);
                }
            }
            __syncthreads();
            // ---- O = PE Sv0 + Bm V, one 16 x 16 tile per warp ----
            if (warp < 2 * (D / 16)) {
                const int tm = warp / (D / 16), tn = warp % (D / 16);
                float acc[2][4] = {};
                tile_nn(acc, peb + tm * 16 * PES, PES, Svb + tn * 16, DP, M);
                tile_nn(acc, bb + tm * 16 * BBS, BBS, vt + tn * 16, DP, C);
                const int gid = lane >> 2, tig = lane & 3;
                OT* o = static_cast<OT*>(p.o);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int r = tm * 16 + gid + 8 * e2, col = tn * 16 + hh * 8 + 2 * tig;
                        if (t0 + r < p.T && GDR_INB(t0 + r < p.T, 702)) {
                            OT* dst = o + tokrow(t0 + r) * D + col;
                            st_from_f32<OT>(dst, acc[hh][2 * e2]);
                            st_from_f32<OT>(dst + 1, acc[hh][2 * e2 + 1]);
                        }
                    }
            }
            __syncthreads();                                        // the old states are read
        }

        // ---- state update (fp32) ----
        for (int si = 0; si < M / NW; ++si) {
            const int i = warp + NW * si;
            const uint32_t mk = msk[i];
            const float lL = lamT[i * CS + C - 1], dL = __expf(lL);
            // this lane's token: its weight in the slot's end state (zero unless it chose the slot)
            const float fl = ((mk >> lane) & 1u) ? cT[i * CS + lane] * __expf(lL - lamT[i * CS + lane]) : 0.f;
            float ak[CPL], av[CPL];
            V::ld(ak, Skf + i * D + c0);
            V::ld(av, Svf + i * D + c0);
#pragma unroll
            for (int u = 0; u < CPL; ++u) {
                ak[u] *= dL;
                av[u] *= dL;
            }
            for (uint32_t m = mk; m; m &= m - 1u) {
                const int s = __ffs(m) - 1;
                const float f = __shfl_sync(0xffffffffu, fl, s);
                float xk[CPL], xv[CPL];
                V::ldb(xk, kt + s * DP + c0);
                V::ldb(xv, vt + s * DP + c0);
#pragma unroll
                for (int u = 0; u < CPL; ++u) {
                    ak[u] += f * xk[u];
                    av[u] += f * xv[u];
                }
            }
            V::st(Skf + i * D + c0, ak);
            V::st(Svf + i * D + c0, av);
            V::stb(Skb + i * DP + c0, ak);
            V::stb(Svb + i * DP + c0, av);
            if (!FULL && lane == 0) ltot[i] += lL;
        }
    }
    __syncthreads();

    // ---- end of the segment ----
    for (int si = 0; si < M / NW; ++si) {
        const int i = warp + NW * si;
        float ak[CPL], av[CPL];
        V::ld(ak, Skf + i * D + c0);
        V::ld(av, Svf + i * D + c0);
        if (!FULL) {
            const size_t base = (size_t)hd * p.nsub + seg;
            V::st(p.segW + base * 2 * MD + (size_t)i * D + c0, ak);
            V::st(p.segW + base * 2 * MD + MD + (size_t)i * D + c0, av);
            if (lane == 0) p.segL[base * M + i] = ltot[i];
        } else if (seg == p.nseg - 1) {
            if (p.SkT) V::st(p.SkT + (size_t)hd * MD + (size_t)i * D + c0, ak);
            if (p.SvT) V::st(p.SvT + (size_t)hd * MD + (size_t)i * D + c0, av);
        }
    }
}

}  // namespace rvn
}  // namespace gdr
