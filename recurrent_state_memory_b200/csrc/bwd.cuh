// bwd.cuh -- gradients of the chunk-WY forward (the backward pass of training).
//
// The chain rule through the chunk-parallel WY/UT algebra of the forward ("CARVE" page, section
// 1 item 3, the WY-form chunk solver; "Semidirect Fourier Delta Attention" page, "Constructive
// Chunk-WY Theorem" and the exact affine chunk transfer).  Per chunk of C = 64 tokens with start
// state S0 (dv x dk), in-chunk cumulative log-decay gam (per token and key dim) and the
// reference token m = 31 (so that no factor exceeds the decay of half a chunk):
//   Kt = K e^{gam - gam_m},  Qt = scale Q e^{gam - gam_m},  Kh = K e^{-(gam - gam_m)},
//   Kd = K e^{gam_L - gam},  S0p = S0 e^{gam_m}                           (column scalings)
//   Ap = Kt Kh^T,  A = diag(beta) strict_lower(Ap),  P = incl_lower(Qt Kh^T),  T = (I + A)^{-1}
//   KS = Kt S0p^T,  R = diag(w) V - diag(beta) KS,  E = T R
//   O = Qt S0p^T + P E,  S_L = S0 e^{gam_L} + E^T Kd
// and, backwards, with dO the chunk's output gradient and dS_L that of its end state:
//   dE = P^T dO + Kd dS_L^T,  dP = incl_lower(dO E^T),  dR = T^T dE,  dA = -T^T (dE R^T) T^T
//   dQt = dO S0p + dP Kh,  dKh = dP^T Qt + dAp^T Kt,  dKt = -(diag(beta) dR) S0p + dAp Kh,
//   dKd = E dS_L,  dAp = diag(beta) strict_lower(dA)
//   dS0 = (dO^T Qt - (diag(beta) dR)^T Kt) e^{gam_m} + dS_L e^{gam_L}
//   dv = diag(w) dR,  dbeta = -rowsum(dR . KS) + rowsum(strict_lower(dA . Ap)) [+ rowsum(dR . V)
//   when w = beta],  dw = rowsum(dR . V)
//   dq = scale dQt e^{gam - gam_m},  dk = dKt e^{gam - gam_m} + dKh e^{-(gam - gam_m)} + dKd e^{gam_L - gam}
//   dgam = dKt . Kt + dQt . Qt - dKh . Kh - dKd . Kd, plus, at the last token,
//          e^{gam_L} colsum(S0 . dS_L) + colsum(dKd . Kd);   dg = (reverse cumsum of dgam) dlogalpha/dg
// (the reference token cancels out of every product, so it leaves the gradients unchanged).
//
// One CTA per (batch, head).  A forward sweep over the chunks keeps each chunk's start state
// (checkpoints in the workspace); the backward sweep then runs the chunks in reverse, each
// recomputing its forward quantities from its checkpoint, with dS_L of chunk c the dS0 of chunk
// c + 1 (the caller's dS_T for the last one).  The matrix products are warp-level tf32 tensor-core
// MMAs with each operand split into a tf32 high part and a tf32 remainder (three products per
// step), which keeps fp32 accuracy; the per-chunk matrices live in a per-head region of the
// workspace (they stay in L1/L2).  Tokens past T are zero padding (k = q = v = 0, beta = w = 0,
// log-decay 0): exact identity transitions whose gradients are not written.
//
// Rotation ("Semidirect Fourier Delta Attention" page, "Core architecture", real implementation:
// 2x2 rotation-decay blocks).  Key pair j of a row is the complex number x + i y and the chunk's
// cumulative factor is Lam_r = e^{rho_r + i phi_r} (rho, phi: in-chunk sums of log alpha and of
// theta).  Every tile factor becomes a complex multiplier per pair: Kt = K F, Qt = scale Q F,
// Kh = K Fh, Kd = K Fh (Lam_L / Lam_m), S0p = S0 Lam_m with F = conj(Lam_r / Lam_m) and
// Fh = Lam_m / Lam_r (same phase, inverse magnitude); the products stay real (the dot product of
// the (re, im) pairs).  Backwards the multipliers are conjugated (the adjoint of a complex
// product), dg takes drho and dtheta takes dphi, each summed in reverse over the chunk:
//   drho = Re(conj(dKt) Kt + conj(dQt) Qt - conj(dKh) Kh - conj(dKd) Kd)
//   dphi = Im(conj(dKt) Kt + conj(dQt) Qt + conj(dKh) Kh + conj(dKd) Kd)
// plus, at the last token, Re / -Im of sum_rows conj(dS_L) S0 Lam_L and sum_r conj(dKd) Kd.
//
// L2 normalisation (qk_l2norm): the chunk algebra runs on qn = q / sqrt(|q|^2 + 1e-6) and kn;
// dq = (dqn - qn (qn . dqn)) / sqrt(|q|^2 + 1e-6), and the same for k.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdr {
namespace bwd {

constexpr int C = 64;
constexpr int NT = 512;
static_assert(NT == C * 8, "eight threads per token in the per-token reductions");
constexpr int NW = NT / 32;
constexpr unsigned STATUS_RANGE = 2u;

struct BwdParams {
    int B, H, T, gate_mode;
    float scale;
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* w;          // write strength [B,T,H] or nullptr (w = beta)
    const float* theta;      // rotation angles [B,T,H,dk/2] (rot) or nullptr
    const float* S0;         // [B,H,dv,dk] or nullptr (zero)
    const void* dO;          // [B,T,H,dv] (the output's dtype) or nullptr (zero)
    const float* dS_T;       // [B,H,dv,dk] or nullptr (zero)
    float* dq;               // [B,T,H,dk]
    float* dk;               // [B,T,H,dk]
    float* dv;               // [B,T,H,dv]
    float* dg;               // [B,T,H,dk]
    float* dbeta;            // [B,T,H]
    float* dw;               // [B,T,H] (with w) or nullptr
    float* dS0;              // [B,H,dv,dk] or nullptr
    float* dtheta;           // [B,T,H,dk/2] (rot) or nullptr
    int rot;                 // 1: 2x2 rotation-decay blocks (g and theta have dk/2 entries per token)
    int norm;                // 1: q and k L2-normalised per token first
    // workspace parts (floats)
    float* coef;             // [B*H][nc][3][dv*dk]: A_c (dk x dk, in a dv x dk slot), B_c, G_c
    float* ckpt;             // [B*H][nc][dv*dk]: the state at each chunk start
    float* dsl;              // [B*H][nc][dv*dk]: the gradient of each chunk's end state
    float* scratch;          // [grid][scratch_floats]: each CTA's chunk matrices
    size_t scratch_floats;
};

// Scratch layout of one CTA of the parallel passes (floats): one chunk's matrices.  The raw k
// and q tiles share storage with dKt and dKh, which are written only after k and q are done with.
template <int DK, int DV>
struct Lay {
    static constexpr int V = 0, DO = V + C * DV;
    static constexpr int EG = DO + C * DV;          // e^{gam - gam_m}
    static constexpr int EGI = EG + C * DK;         // e^{-(gam - gam_m)}
    static constexpr int DLG = EGI + C * DK;        // d log alpha / d gate input
    static constexpr int KT = DLG + C * DK, KH = KT + C * DK, QT = KH + C * DK, KD = QT + C * DK;
    static constexpr int AP = KD + C * DK, PM = AP + C * C, TM = PM + C * C, X1 = TM + C * C, X2 = X1 + C * C;
    static constexpr int DA = X2 + C * C, DPM = DA + C * C;
    static constexpr int KS = DPM + C * C, R = KS + C * DV, E = R + C * DV, DE = E + C * DV, DR = DE + C * DV;
    static constexpr int DQT = DR + C * DV, DKH = DQT + C * DK, DKD = DKH + C * DK, DKT = DKD + C * DK;
    static constexpr int K = DKT, Q = DKH;          // raw k and q (chunk_forward only)
    static constexpr int BT = DKT + C * DK, WT = BT + C, DBS = WT + C;   // beta, w, dbeta parts
    static constexpr int E31 = DBS + C, EGL = E31 + DK, ED = EGL + DK;   // column vectors (rotation:
                                                                         // (re, im) per key pair)
    static constexpr int NQV = ED + DK, NKV = NQV + C;   // per-token 1/|q|, 1/|k| (qk_l2norm)
    static constexpr int S0P = NKV + C;
    static constexpr size_t floats() { return (size_t)S0P + (size_t)DV * DK; }
};

__device__ __forceinline__ uint32_t tf32_hi(float x) { return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u; }

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Shared-memory floats the products need: both operands with padded rows.
constexpr int SMEM_FLOATS = 128 * 132 + 128 * 136;
constexpr size_t SMEM_BYTES = sizeof(float) * SMEM_FLOATS;

// rows x cols floats (global, row stride ld, 16-byte aligned rows) -> shared memory with row
// stride ls, float4 at a time
__device__ __forceinline__ void stage(float* dst, int ls, const float* src, int ld, int rows, int cols) {
    const int c4 = cols >> 2;
#pragma unroll 16
    for (int i = (int)threadIdx.x; i < rows * c4; i += NT) {
        const int r = i / c4, c = (i % c4) * 4;
        *reinterpret_cast<float4*>(dst + r * ls + c) = *reinterpret_cast<const float4*>(src + (size_t)r * ld + c);
    }
}

// Cm (M x N, row stride ldc) = alpha op(A) op(B) (+ Cm when acc), with op(A)(i, k) = A[i][k]
// (TA: A[k][i]) and op(B)(k, j) = B[k][j] (TB: B[j][k]).  M, N multiples of 16, K of 8, all at
// most 128.  Both operands are first staged in shared memory `sm`, with row strides padded so
// that the fragment loads hit 32 distinct banks.  All threads of the CTA take part; the caller
// synchronises before (the operands are written) and after (Cm is read).
template <bool TA, bool TB>
__device__ void mm(float* Cm, int ldc, const float* A, int lda, const float* Bm, int ldb, int M, int N, int K,
                   float alpha, bool acc, float* sm) {
    const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const int tn = N / 16, ntiles = (M / 16) * tn;
    const int sa = TA ? M + 8 : K + 4, sbs = TB ? K + 4 : N + 8;
    float* sA = sm;
    float* sB = sm + 128 * 132;
    stage(sA, sa, A, lda, TA ? K : M, TA ? M : K);
    stage(sB, sbs, Bm, ldb, TB ? N : K, TB ? K : N);
    __syncthreads();
    auto a_ = [&](int i, int k) -> float { return TA ? sA[k * sa + i] : sA[i * sa + k]; };
    auto b_ = [&](int k, int j) -> float { return TB ? sB[j * sbs + k] : sB[k * sbs + j]; };
    for (int t = warp; t < ntiles; t += NW) {
        const int r0 = (t / tn) * 16, c0 = (t % tn) * 16;
        // three accumulators per 8-column half (high x high, high x low, low x high), so that
        // six independent MMA chains run side by side; summed at the end, small parts first
        float dhh[2][4] = {}, dhl[2][4] = {}, dlh[2][4] = {};
#pragma unroll 2
        for (int k0 = 0; k0 < K; k0 += 8) {
            const float af[4] = {a_(r0 + gid, k0 + tig), a_(r0 + gid + 8, k0 + tig), a_(r0 + gid, k0 + tig + 4),
                                 a_(r0 + gid + 8, k0 + tig + 4)};
            const float bf[2][2] = {{b_(k0 + tig, c0 + gid), b_(k0 + tig + 4, c0 + gid)},
                                    {b_(k0 + tig, c0 + 8 + gid), b_(k0 + tig + 4, c0 + 8 + gid)}};
            uint32_t ah[4], al[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ah[e] = tf32_hi(af[e]);
                al[e] = tf32_hi(af[e] - __uint_as_float(ah[e]));
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t bh[2], bl[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    bh[e] = tf32_hi(bf[h][e]);
                    bl[e] = tf32_hi(bf[h][e] - __uint_as_float(bh[e]));
                }
                mma_tf32(dlh[h], al, bh);
                mma_tf32(dhl[h], ah, bl);
                mma_tf32(dhh[h], ah, bh);
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int row = r0 + gid + ((e >> 1) << 3), col = c0 + 8 * h + 2 * tig + (e & 1);
                float x = alpha * ((dlh[h][e] + dhl[h][e]) + dhh[h][e]);
                if (acc) x += Cm[(size_t)row * ldc + col];
                Cm[(size_t)row * ldc + col] = x;
            }
    }
    __syncthreads();     // the staged operands may be overwritten by the next product
}

template <typename T>
__device__ __forceinline__ float ldx(const T* p, size_t i) {
    return ld_f32<T>(p + i);
}

// One chunk's inputs and forward quantities up to E (every thread; ends synchronised).
// S0 is the chunk's start state (dv x dk, row-major).
template <int DK, int DV, typename QT, typename OT>
__device__ void chunk_forward(const BwdParams& p, float* W, int b, int h, int t0, const float* S0, bool want_dO,
                              int* range_f, float* sm) {
    using L = Lay<DK, DV>;
    const int tid = (int)threadIdx.x;
    const QT* q = static_cast<const QT*>(p.q);
    const QT* k = static_cast<const QT*>(p.k);
    const QT* v = static_cast<const QT*>(p.v);
    auto tok = [&](int r) -> size_t { return ((size_t)b * p.T + (t0 + r)) * p.H + h; };
    // raw inputs of the chunk, zero past T (four loads in flight per thread); the log-decays go
    // to shared memory for the scan below
    // (rotation: column 2j holds log alpha of pair j, column 2j + 1 its angle theta)
    float* sg = sm;                       // [C][DK] log alpha, then gam
    float* sg31 = sm + C * DK;            // [DK] gam at the reference token
    float* sgl = sg31 + DK;               // [DK] gam at the last token
    const int ng = p.rot ? DK / 2 : DK;   // gate entries per token
    constexpr int NK = C * DK / NT, NV = C * DV / NT;
#pragma unroll
    for (int u = 0; u < NK; ++u) {
        const int i = tid + u * NT, r = i / DK, d = i % DK;
        const bool ok = t0 + r < p.T;
        const size_t o = tok(r) * DK + d;
        const float kk = ok ? ldx(k, o) : 0.f, qq = ok ? ldx(q, o) : 0.f;
        W[L::K + i] = kk;
        W[L::Q + i] = qq;
        float lg = 0.f, dl = 0.f;
        if (ok) {
            if (p.rot && (d & 1)) {
                lg = p.theta[tok(r) * ng + (d >> 1)];          // d phi / d theta = 1
                dl = 1.f;
            } else {
                const float a = p.g[tok(r) * ng + (p.rot ? d >> 1 : d)];
                lg = log_decay(a, p.gate_mode);
                dl = p.gate_mode == 1 ? -1.f / (1.f + expf(-a)) : 1.f;   // d(-softplus a)/da = -sigmoid(a)
            }
        }
        sg[i] = lg;
        W[L::DLG + i] = dl;
    }
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int i = tid + u * NT, r = i / DV, d = i % DV;
        const bool ok = t0 + r < p.T;
        const size_t o = tok(r) * DV + d;
        const float vv = ok ? ldx(v, o) : 0.f;
        const float dd = (want_dO && ok && p.dO) ? ldx(static_cast<const OT*>(p.dO), o) : 0.f;
        W[L::V + i] = vv;
        if (want_dO) W[L::DO + i] = dd;
    }
    if (tid < C) {
        const bool ok = t0 + tid < p.T;
        const float bt = ok ? p.beta[tok(tid)] : 0.f;
        W[L::BT + tid] = bt;
        W[L::WT + tid] = ok ? (p.w ? p.w[tok(tid)] : bt) : 0.f;
    }
    __syncthreads();
    // qk_l2norm: 1/|k| and 1/|q| per token, eight threads a token
    if (p.norm) {
        const int r = tid >> 3, part = tid & 7;
        float sk = 0.f, sq = 0.f;
        for (int d = part; d < DK; d += 8) {
            const float a = W[L::K + r * DK + d], c = W[L::Q + r * DK + d];
            sk += a * a;
            sq += c * c;
        }
#pragma unroll
        for (int off = 4; off >= 1; off >>= 1) {
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        if (part == 0) {
            W[L::NKV + r] = rsqrtf(sk + 1e-6f);
            W[L::NQV + r] = rsqrtf(sq + 1e-6f);
        }
    }
    // cumulative log-decay (rotation: and angle) per key dim, the reference token m = 31
    if (tid < DK) {
        const int d = tid;
        float gam = 0.f, g31 = 0.f;
        for (int r = 0; r < C; ++r) {
            gam += sg[r * DK + d];
            sg[r * DK + d] = gam;
            if (r == 31) g31 = gam;
        }
        sg31[d] = g31;
        sgl[d] = gam;
    }
    __syncthreads();
    // column factors e^{gam_m}, e^{gam_L}, e^{gam_L - gam_m} (rotation: Lam_m, Lam_L, Lam_L / Lam_m
    // as (re, im) per pair) and the tile multipliers EG = e^{gam - gam_m}, EGI = e^{-(gam - gam_m)}
    // (rotation: F and Fh per pair)
    if (tid < DK) {
        const int d = tid;
        if (!p.rot) {
            W[L::E31 + d] = expf(sg31[d]);
            W[L::EGL + d] = expf(sgl[d]);
            W[L::ED + d] = expf(sgl[d] - sg31[d]);
        } else {
            const int e = d & ~1;
            const bool im = d & 1;
            auto cs = [&](float ang) -> float {
                float sn, c;
                sincosf(ang, &sn, &c);
                return im ? sn : c;
            };
            W[L::E31 + d] = expf(sg31[e]) * cs(sg31[e + 1]);
            W[L::EGL + d] = expf(sgl[e]) * cs(sgl[e + 1]);
            W[L::ED + d] = expf(sgl[e] - sg31[e]) * cs(sgl[e + 1] - sg31[e + 1]);
        }
    }
    {
        bool bad = false;
        for (int i = tid; i < C * DK; i += NT) {
            const int d = i % DK;
            float e, ei;
            if (!p.rot) {
                const float x = sg[i] - sg31[d];
                e = expf(x);
                ei = expf(-x);
                if (!(e < 3e38f) || !(ei < 3e38f)) bad = true;
            } else {
                const int i0 = i & ~1, d0 = d & ~1;
                const float x = sg[i0] - sg31[d0];
                float sn, c;
                sincosf(sg[i0 + 1] - sg31[d0 + 1], &sn, &c);
                const float m = expf(x), mi = expf(-x), f = (d & 1) ? -sn : c;    // e^{-i dphi}
                if (!(m < 3e38f) || !(mi < 3e38f)) bad = true;
                e = m * f;
                ei = mi * f;
            }
            W[L::EG + i] = e;
            W[L::EGI + i] = ei;
        }
        if (bad) atomicExch(range_f, 1);
    }
    __syncthreads();
    for (int i = tid; i < C * DK; i += NT) {
        const int r = i / DK, d = i % DK;
        const float nk = p.norm ? W[L::NKV + r] : 1.f, nq = p.norm ? p.scale * W[L::NQV + r] : p.scale;
        if (!p.rot) {
            const float kk = W[L::K + i] * nk;
            W[L::KT + i] = kk * W[L::EG + i];
            W[L::KH + i] = kk * W[L::EGI + i];
            W[L::QT + i] = nq * W[L::Q + i] * W[L::EG + i];
            W[L::KD + i] = kk * W[L::EGI + i] * W[L::ED + d];
        } else {
            // complex products per pair: component im of (ar + i ai)(br + i bi)
            const int i0 = i & ~1, d0 = d & ~1;
            const bool im = d & 1;
            auto cm = [im](float ar, float ai, float br, float bi) { return im ? ar * bi + ai * br : ar * br - ai * bi; };
            const float kx = W[L::K + i0] * nk, ky = W[L::K + i0 + 1] * nk;
            const float qx = W[L::Q + i0] * nq, qy = W[L::Q + i0 + 1] * nq;
            const float fr = W[L::EG + i0], fi = W[L::EG + i0 + 1], hr = W[L::EGI + i0], hi = W[L::EGI + i0 + 1];
            const float dr = W[L::ED + d0], di = W[L::ED + d0 + 1];
            W[L::KT + i] = cm(kx, ky, fr, fi);
            W[L::KH + i] = cm(kx, ky, hr, hi);
            W[L::QT + i] = cm(qx, qy, fr, fi);
            W[L::KD + i] = cm(kx, ky, hr * dr - hi * di, hr * di + hi * dr);
        }
    }
    if (S0)
        for (int i = tid; i < DV * DK; i += NT) {
            if (!p.rot) {
                W[L::S0P + i] = S0[i] * W[L::E31 + i % DK];
            } else {
                const int i0 = i & ~1, d0 = i0 % DK;
                const float x = S0[i0], y = S0[i0 + 1], mr = W[L::E31 + d0], mi = W[L::E31 + d0 + 1];
                W[L::S0P + i] = (i & 1) ? x * mi + y * mr : x * mr - y * mi;
            }
        }
    __syncthreads();
    mm<false, true>(W + L::AP, C, W + L::KT, DK, W + L::KH, DK, C, C, DK, 1.f, false, sm);      // Ap = Kt Kh^T
    mm<false, true>(W + L::PM, C, W + L::QT, DK, W + L::KH, DK, C, C, DK, 1.f, false, sm);      // Qt Kh^T
    if (S0) mm<false, true>(W + L::KS, DV, W + L::KT, DK, W + L::S0P, DK, C, DV, DK, 1.f, false, sm);   // KS = Kt S0p^T
    __syncthreads();
    // masks; R = diag(w) V - diag(beta) KS; T = (I + A)^{-1} by forward substitution, eight
    // threads per column
    for (int i = tid; i < C * C; i += NT) {
        const int r = i / C, c = i % C;
        if (c > r) W[L::PM + i] = 0.f;
    }
    if (S0)
        for (int i = tid; i < C * DV; i += NT) {
            const int r = i / DV;
            W[L::R + i] = W[L::WT + r] * W[L::V + i] - W[L::BT + r] * W[L::KS + i];
        }
    {   // A = diag(beta) strict_lower(Ap) and T in shared memory (row stride C + 1)
        float* sAm = sm;
        float* sT = sm + C * (C + 1);
        for (int i = tid; i < C * C; i += NT) {
            const int r = i / C, c = i % C;
            sAm[r * (C + 1) + c] = W[L::BT + r] * W[L::AP + i];
        }
        __syncthreads();
        const int j = tid >> 3, part = tid & 7;            // column j, eighth of the sum
        for (int r = 0; r < C; ++r) {
            float s = 0.f;
            if (r > j)
                for (int i = j + part; i < r; i += 8) s += sAm[r * (C + 1) + i] * sT[i * (C + 1) + j];
#pragma unroll
            for (int off = 4; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (part == 0) sT[r * (C + 1) + j] = (r == j) ? 1.f : (r > j ? -s : 0.f);
            __syncwarp();
        }
        __syncthreads();
        for (int i = tid; i < C * C; i += NT) W[L::TM + i] = sT[(i / C) * (C + 1) + i % C];
    }
    __syncthreads();
    if (S0) mm<false, false>(W + L::E, DV, W + L::TM, C, W + L::R, DV, C, DV, C, 1.f, false, sm);   // E = T R
    __syncthreads();
}

// The gradients of one chunk, every thread taking part, after chunk_forward on the chunk's start
// state S0c (its quantities are in W); dSL is the gradient of the chunk's end state.
template <int DK, int DV, typename QT, typename OT>
__device__ void chunk_grads(const BwdParams& p, float* W, int b, int h, int t0, const float* S0c, const float* dSL,
                            float* sm) {
    using L = Lay<DK, DV>;
    const int tid = (int)threadIdx.x;
    // dE = P^T dO + Kd dSL^T ; dP = incl_lower(dO E^T) ; dKd = E dSL
    mm<true, false>(W + L::DE, DV, W + L::PM, C, W + L::DO, DV, C, DV, C, 1.f, false, sm);
    mm<false, true>(W + L::DPM, C, W + L::DO, DV, W + L::E, DV, C, C, DV, 1.f, false, sm);
    mm<false, false>(W + L::DKD, DK, W + L::E, DV, dSL, DK, C, DK, DV, 1.f, false, sm);
    __syncthreads();
    mm<false, true>(W + L::DE, DV, W + L::KD, DK, dSL, DK, C, DV, DK, 1.f, true, sm);
    for (int i = tid; i < C * C; i += NT) {
        const int r = i / C, cc = i % C;
        if (cc > r) W[L::DPM + i] = 0.f;
    }
    __syncthreads();
    // dR = T^T dE ; X1 = dE R^T ; dQt = dO S0p + dP Kh ; dKh = dP^T Qt
    mm<true, false>(W + L::DR, DV, W + L::TM, C, W + L::DE, DV, C, DV, C, 1.f, false, sm);
    mm<false, true>(W + L::X1, C, W + L::DE, DV, W + L::R, DV, C, C, DV, 1.f, false, sm);
    mm<false, false>(W + L::DQT, DK, W + L::DO, DV, W + L::S0P, DK, C, DK, DV, 1.f, false, sm);
    mm<true, false>(W + L::DKH, DK, W + L::DPM, C, W + L::QT, DK, C, DK, C, 1.f, false, sm);
    __syncthreads();
    mm<false, false>(W + L::DQT, DK, W + L::DPM, C, W + L::KH, DK, C, DK, C, 1.f, true, sm);
    mm<true, false>(W + L::X2, C, W + L::TM, C, W + L::X1, C, C, C, C, 1.f, false, sm);      // T^T X1
    // beta dR (in place) after dv, dw and the dR parts of dbeta
    __syncthreads();
    mm<false, true>(W + L::DA, C, W + L::X2, C, W + L::TM, C, C, C, C, -1.f, false, sm);     // dA = -X2 T^T
    if (tid < C * 8) {
        // per token r (eight threads each): dbeta and dw parts from dR
        const int r = tid >> 3, part = tid & 7;
        float sks = 0.f, sv = 0.f;
        for (int j = part; j < DV; j += 8) {
            const float dr = W[L::DR + r * DV + j];
            sks += dr * W[L::KS + r * DV + j];
            sv += dr * W[L::V + r * DV + j];
        }
#pragma unroll
        for (int off = 4; off >= 1; off >>= 1) {
            sks += __shfl_xor_sync(0xffffffffu, sks, off);
            sv += __shfl_xor_sync(0xffffffffu, sv, off);
        }
        if (part == 0) {
            W[L::DBS + r] = -sks + (p.w ? 0.f : sv);         // dbeta so far
            if (p.dw && t0 + r < p.T) p.dw[((size_t)b * p.T + t0 + r) * p.H + h] = sv;
        }
    }
    for (int i = tid; i < C * DV; i += NT) {
        const int r = i / DV, j = i % DV;
        if (t0 + r < p.T) p.dv[(((size_t)b * p.T + t0 + r) * p.H + h) * DV + j] = W[L::WT + r] * W[L::DR + i];
    }
    __syncthreads();
    // dAp = diag(beta) strict_lower(dA) (in place, after the dA . Ap part of dbeta)
    if (tid < C * 8) {
        const int r = tid >> 3, part = tid & 7;
        float s = 0.f;
        for (int i = part; i < r; i += 8) s += W[L::DA + r * C + i] * W[L::AP + r * C + i];
#pragma unroll
        for (int off = 4; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (part == 0 && t0 + r < p.T)
            p.dbeta[((size_t)b * p.T + t0 + r) * p.H + h] = W[L::DBS + r] + s;
    }
    __syncthreads();
    for (int i = tid; i < C * C; i += NT) {
        const int r = i / C, cc = i % C;
        W[L::DA + i] = cc < r ? W[L::BT + r] * W[L::DA + i] : 0.f;
    }
    for (int i = tid; i < C * DV; i += NT) W[L::DR + i] *= W[L::BT + i / DV];
    __syncthreads();
    // dKt = -(beta dR) S0p + dAp Kh ; dKh += dAp^T Kt
    mm<false, false>(W + L::DKT, DK, W + L::DR, DV, W + L::S0P, DK, C, DK, DV, -1.f, false, sm);
    mm<true, false>(W + L::DKH, DK, W + L::DA, C, W + L::KT, DK, C, DK, C, 1.f, true, sm);
    __syncthreads();
    mm<false, false>(W + L::DKT, DK, W + L::DA, C, W + L::KH, DK, C, DK, C, 1.f, true, sm);
    __syncthreads();
    // dq, dk (qk_l2norm: those of the normalised q and k, in X1.. and DA.., C x DK each); dgam
    // (rotation: drho in column 2j, dphi in column 2j + 1) in shared memory
    float* sdg = sm;                  // [C][DK] dgam, then dg
    float* sdl = sm + C * DK;         // [C][DK] d log alpha / d gate input (rotation: 1 for the angle)
    float* scs = sm + 2 * C * DK;     // [NT / DK][DK] column-sum parts
    float* gqn = W + L::X1;
    float* gkn = W + L::DA;
    static_assert(L::X2 == L::X1 + C * C && L::DPM == L::DA + C * C && DK <= 2 * C, "C x DK over two C x C tiles");
    for (int i = tid; i < C * DK; i += NT) {
        const int r = i / DK, d = i % DK;
        float gq, gk, dgm;
        if (!p.rot) {
            const float eg = W[L::EG + i], egi = W[L::EGI + i];
            const float gkt = W[L::DKT + i], gkh = W[L::DKH + i], gqt = W[L::DQT + i], gkd = W[L::DKD + i];
            gq = p.scale * gqt * eg;
            gk = gkt * eg + gkh * egi + gkd * egi * W[L::ED + d];
            dgm = gkt * W[L::KT + i] + gqt * W[L::QT + i] - gkh * W[L::KH + i] - gkd * W[L::KD + i];
        } else {
            const int i0 = i & ~1, d0 = d & ~1;
            const bool im = d & 1;
            // component im of a conj(b); Re and Im of conj(a) b over the pair at offset o
            auto cmc = [im](float ar, float ai, float br, float bi) { return im ? ai * br - ar * bi : ar * br + ai * bi; };
            auto pr = [&](int ga, int x) {
                const float ar = W[ga + i0], ai = W[ga + i0 + 1], br = W[x + i0], bi = W[x + i0 + 1];
                return im ? ar * bi - ai * br : ar * br + ai * bi;
            };
            const float fr = W[L::EG + i0], fi = W[L::EG + i0 + 1], hr = W[L::EGI + i0], hi = W[L::EGI + i0 + 1];
            const float dr = W[L::ED + d0], di = W[L::ED + d0 + 1];
            const float gr = hr * dr - hi * di, gi = hr * di + hi * dr;       // Fh Lam_L / Lam_m
            gq = p.scale * cmc(W[L::DQT + i0], W[L::DQT + i0 + 1], fr, fi);
            gk = cmc(W[L::DKT + i0], W[L::DKT + i0 + 1], fr, fi) + cmc(W[L::DKH + i0], W[L::DKH + i0 + 1], hr, hi) +
                 cmc(W[L::DKD + i0], W[L::DKD + i0 + 1], gr, gi);
            const float sgn = im ? 1.f : -1.f;       // Kh and Kd: -Re for drho, +Im for dphi
            dgm = pr(L::DKT, L::KT) + pr(L::DQT, L::QT) + sgn * (pr(L::DKH, L::KH) + pr(L::DKD, L::KD));
        }
        if (p.norm) {
            gqn[i] = gq;
            gkn[i] = gk;
        } else if (t0 + r < p.T) {
            const size_t o = (((size_t)b * p.T + t0 + r) * p.H + h) * DK + d;
            p.dq[o] = gq;
            p.dk[o] = gk;
        }
        sdg[i] = dgm;
        sdl[i] = W[L::DLG + i];
    }
    {   // column sums for the last token's decay terms: NT / DK threads per key dim
        constexpr int NP = NT / DK;
        const int d = tid % DK, part = tid / DK;
        float s0 = 0.f, sd = 0.f;
        if (!p.rot) {
            for (int i = part; i < DV; i += NP) s0 += S0c[i * DK + d] * dSL[i * DK + d];
            for (int r = part; r < C; r += NP) sd += W[L::DKD + r * DK + d] * W[L::KD + r * DK + d];
            scs[part * DK + d] = W[L::EGL + d] * s0 + sd;
        } else {
            // drho_L: Re sum conj(dS_L) S0 Lam_L + Re sum conj(dKd) Kd; dphi_L: -Im of the same
            const int d0 = d & ~1;
            const bool im = d & 1;
            const float lr = W[L::EGL + d0], li = W[L::EGL + d0 + 1];
            auto pr = [im](float ar, float ai, float br, float bi) { return im ? -(ar * bi - ai * br) : ar * br + ai * bi; };
            for (int i = part; i < DV; i += NP) {
                const float x = S0c[i * DK + d0], y = S0c[i * DK + d0 + 1];
                s0 += pr(dSL[i * DK + d0], dSL[i * DK + d0 + 1], x * lr - y * li, x * li + y * lr);
            }
            for (int r = part; r < C; r += NP)
                sd += pr(W[L::DKD + r * DK + d0], W[L::DKD + r * DK + d0 + 1], W[L::KD + r * DK + d0],
                         W[L::KD + r * DK + d0 + 1]);
            scs[part * DK + d] = s0 + sd;
        }
    }
    __syncthreads();
    if (tid < DK) {     // reverse cumulative sum over the chunk's tokens
        const int d = tid;
        float acc = 0.f;
        for (int pp = 0; pp < NT / DK; ++pp) acc += scs[pp * DK + d];
        for (int r = C - 1; r >= 0; --r) {
            acc += sdg[r * DK + d];
            sdg[r * DK + d] = acc * sdl[r * DK + d];
        }
    }
    __syncthreads();
    const int ng = p.rot ? DK / 2 : DK;
    for (int i = tid; i < C * DK; i += NT) {
        const int r = i / DK, d = i % DK;
        if (t0 + r >= p.T) continue;
        const size_t tk = ((size_t)b * p.T + t0 + r) * p.H + h;
        if (!p.rot) p.dg[tk * DK + d] = sdg[i];
        else (d & 1 ? p.dtheta : p.dg)[tk * ng + (d >> 1)] = sdg[i];
    }
    if (p.norm) {
        // through the normalisation, per token (eight threads each; rows past T are computed
        // from the zero padding and not written): d x = r (dxn - xn (xn . dxn)), r = 1 / |x|
        const QT* q = static_cast<const QT*>(p.q);
        const QT* k = static_cast<const QT*>(p.k);
        const int r = tid >> 3, part = tid & 7;
        const bool ok = t0 + r < p.T;
        const size_t ob = (((size_t)b * p.T + (ok ? t0 + r : 0)) * p.H + h) * DK;
        float sk = 0.f, sq = 0.f, pk = 0.f, pq = 0.f;
        for (int d = part; d < DK; d += 8) {
            const float kk = ok ? ldx(k, ob + d) : 0.f, qq = ok ? ldx(q, ob + d) : 0.f;
            sk += kk * kk;
            sq += qq * qq;
            pk += kk * gkn[r * DK + d];
            pq += qq * gqn[r * DK + d];
        }
#pragma unroll
        for (int off = 4; off >= 1; off >>= 1) {
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            pk += __shfl_xor_sync(0xffffffffu, pk, off);
            pq += __shfl_xor_sync(0xffffffffu, pq, off);
        }
        const float rk = rsqrtf(sk + 1e-6f), rq = rsqrtf(sq + 1e-6f);
        const float ck = rk * rk * rk * pk, cq = rq * rq * rq * pq;
        if (ok)
            for (int d = part; d < DK; d += 8) {
                p.dk[ob + d] = rk * gkn[r * DK + d] - ck * ldx(k, ob + d);
                p.dq[ob + d] = rq * gqn[r * DK + d] - cq * ldx(q, ob + d);
            }
    }
    __syncthreads();
}

// Tasks of the two parallel passes: chunk c of head hd, as t = hd * nc + c; each CTA takes
// tasks blockIdx.x, blockIdx.x + gridDim.x, ... with its own region of the scratch.

// Pass 1: each chunk's transfer coefficients, which need no state:
//   M = T^T Kd,  A_c = diag(e^{gam_L}) - diag(e^{gam_m}) Kt^T diag(beta) M     (dk x dk)
//   B_c = (T diag(w) V)^T Kd                                                  (dv x dk)
//   G_c = dO^T (Qt - P T diag(beta) Kt) diag(e^{gam_m})                        (dv x dk)
// so that a chunk's end state is S_L = S0 A_c + B_c and its start state's gradient is
// dS0 = G_c + dS_L A_c^T.
template <int DK, int DV, typename QT, typename OT>
__global__ void __launch_bounds__(NT, 1) bwd_coef_kernel(BwdParams p) {
    using L = Lay<DK, DV>;
    extern __shared__ float4 sm4[];
    float* sm = reinterpret_cast<float*>(sm4);
    __shared__ int range_f;
    const int tid = (int)threadIdx.x;
    const int nc = (p.T + C - 1) / C, ntask = p.B * p.H * nc;
    float* W = p.scratch + (size_t)blockIdx.x * p.scratch_floats;
    if (tid == 0) range_f = 0;
    for (int t = (int)blockIdx.x; t < ntask; t += (int)gridDim.x) {
        const int hd = t / nc, c = t % nc, b = hd / p.H, h = hd % p.H;
        if (!GDR_INB(hd < p.B * p.H, 402)) break;
        chunk_forward<DK, DV, QT, OT>(p, W, b, h, c * C, nullptr, true, &range_f, sm);
        float* A = p.coef + ((size_t)t * 3 + 0) * DV * DK;
        float* Bc = p.coef + ((size_t)t * 3 + 1) * DV * DK;
        float* G = p.coef + ((size_t)t * 3 + 2) * DV * DK;
        // M = T^T Kd (in DQT); diag(w) V (in V); diag(beta) Kt (in DKT)
        mm<true, false>(W + L::DQT, DK, W + L::TM, C, W + L::KD, DK, C, DK, C, 1.f, false, sm);
        for (int i = tid; i < C * DV; i += NT) W[L::V + i] *= W[L::WT + i / DV];
        for (int i = tid; i < C * DK; i += NT) W[L::DKT + i] = W[L::BT + i / DK] * W[L::KT + i];
        __syncthreads();
        // N = (diag(beta) Kt)^T M (into A); E0 = T diag(w) V (in E); W1 = T diag(beta) Kt (in DKH)
        mm<true, false>(A, DK, W + L::DKT, DK, W + L::DQT, DK, DK, DK, C, 1.f, false, sm);
        mm<false, false>(W + L::E, DV, W + L::TM, C, W + L::V, DV, C, DV, C, 1.f, false, sm);
        mm<false, false>(W + L::DKH, DK, W + L::TM, C, W + L::DKT, DK, C, DK, C, 1.f, false, sm);
        __syncthreads();
        // A_c = diag(e^{gam_L}) - diag(e^{gam_m}) N ; B_c = E0^T Kd ; X = P W1 (in DKD)
        if (!p.rot)
            for (int i = tid; i < DK * DK; i += NT) {
                const int r = i / DK, cc = i % DK;
                A[i] = (r == cc ? W[L::EGL + r] : 0.f) - W[L::E31 + r] * A[i];
            }
        else    // the 2x2 blocks of right-multiplication by Lam_L and Lam_m: [[re, im], [-im, re]]
            for (int i = tid; i < DK / 2 * DK; i += NT) {
                const int r0 = 2 * (i / DK), cc = i % DK;
                const float n0 = A[r0 * DK + cc], n1 = A[(r0 + 1) * DK + cc];
                const float lr = W[L::EGL + r0], li = W[L::EGL + r0 + 1], mr = W[L::E31 + r0], mi = W[L::E31 + r0 + 1];
                A[r0 * DK + cc] = (cc == r0 ? lr : cc == r0 + 1 ? li : 0.f) - (mr * n0 + mi * n1);
                A[(r0 + 1) * DK + cc] = (cc == r0 ? -li : cc == r0 + 1 ? lr : 0.f) - (mr * n1 - mi * n0);
            }
        mm<true, false>(Bc, DK, W + L::E, DV, W + L::KD, DK, DV, DK, C, 1.f, false, sm);
        mm<false, false>(W + L::DKD, DK, W + L::PM, C, W + L::DKH, DK, C, DK, C, 1.f, false, sm);
        __syncthreads();
        // G_c = dO^T (Qt - X) diag(e^{gam_m})
        for (int i = tid; i < C * DK; i += NT) W[L::DKD + i] = W[L::QT + i] - W[L::DKD + i];
        __syncthreads();
        mm<true, false>(G, DK, W + L::DO, DV, W + L::DKD, DK, DV, DK, C, 1.f, false, sm);
        if (!p.rot)
            for (int i = tid; i < DV * DK; i += NT) G[i] *= W[L::E31 + i % DK];
        else    // rows times conj(Lam_m): the transpose of the right-multiplication by Lam_m
            for (int i = 2 * tid; i < DV * DK; i += 2 * NT) {
                const float x = G[i], y = G[i + 1], mr = W[L::E31 + i % DK], mi = W[L::E31 + i % DK + 1];
                G[i] = x * mr + y * mi;
                G[i + 1] = y * mr - x * mi;
            }
        __syncthreads();
    }
    if (tid == 0 && range_f) atomicOr(&g_device_status, STATUS_RANGE);
}

// 16-byte copy global -> shared that completes asynchronously (cp.async, L2 only).
__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Pass 2, one CTA per head: the chunk start states S_{c+1} = S_c A_c + B_c (kept for pass 3),
// then, backwards, the end-state gradients dS_L(c-1) = G_c + dS_L(c) A_c^T (kept), and the
// gradient of S0.  The carried matrix stays in shared memory; the next chunk's A_c is fetched
// with asynchronous copies while the current product runs, and B_c / G_c are loaded into
// registers at the start of the step.
template <int D>
__global__ void __launch_bounds__(NT, 1) bwd_chain_kernel(BwdParams p) {
    extern __shared__ float4 sm4[];
    float* sm = reinterpret_cast<float*>(sm4);
    constexpr int SS = D + 4;                  // row stride of the carried matrix (the A operand)
    constexpr int SA = D + 8;                  // row stride of A_c read as it is (forwards)
    constexpr int SAT = D + 4;                 // row stride of A_c read transposed (backwards)
    constexpr int DD = D * D;
    constexpr int TN = D / 16, NTILE = TN * TN, TPW = (NTILE + NW - 1) / NW;   // 16x16 tiles per warp
    float* S = sm;                             // [D][SS]
    float* Abuf[2] = {sm + D * SS, sm + D * SS + D * SA};
    const int tid = (int)threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
    const int hd = (int)blockIdx.x, nc = (p.T + C - 1) / C;
    if (!GDR_INB(hd < p.B * p.H, 403)) return;     // (the whole CTA)
    auto coef = [&](int c, int k) -> const float* { return p.coef + (((size_t)hd * nc + c) * 3 + k) * DD; };
    auto prefetch_A = [&](int c, int buf, int stride) {
        for (int i = tid; i < DD / 4; i += NT) {
            const int r = (4 * i) / D, cc = (4 * i) % D;
            cp_async16(Abuf[buf] + r * stride + cc, coef(c, 0) + 4 * i);
        }
        cp_async_commit();
    };
    // n steps of the chain from chunk c0 in direction dc: S <- coef(c, add_k) + S op(A_c); the new
    // S of chunk c is also stored at keep + (hd * nc + c + shift) * DD unless keep is null
    auto run = [&](bool fwd, int c0, int dc, int n, float* keep, int shift, int add_k) {
        const int stride = fwd ? SA : SAT;
        if (n > 0) prefetch_A(c0, 0, stride);
        for (int st = 0; st < n; ++st) {
            const int c = c0 + st * dc, buf = st & 1;
            const float* addp = coef(c, add_k);
            float res[TPW][8];
#pragma unroll
            for (int u = 0; u < TPW; ++u) {
                const int t = warp + u * NW, r0 = (t / TN) * 16, col0 = (t % TN) * 16;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int row = r0 + gid + (((e >> 1) & 1) << 3), col = col0 + 8 * (e >> 2) + 2 * tig + (e & 1);
                    res[u][e] = t < NTILE ? addp[row * D + col] : 0.f;
                }
            }
            cp_async_wait_all();
            __syncthreads();                                   // A_c landed; S is the current matrix
            if (st + 1 < n) prefetch_A(c + dc, buf ^ 1, stride);
            const float* Ab = Abuf[buf];
#pragma unroll
            for (int u = 0; u < TPW; ++u) {
                const int t = warp + u * NW, r0 = (t / TN) * 16, col0 = (t % TN) * 16;
                if (t >= NTILE) continue;
                float dhh[2][4] = {}, dhl[2][4] = {}, dlh[2][4] = {};
#pragma unroll 2
                for (int k0 = 0; k0 < D; k0 += 8) {
                    const float af[4] = {S[(r0 + gid) * SS + k0 + tig], S[(r0 + gid + 8) * SS + k0 + tig],
                                         S[(r0 + gid) * SS + k0 + tig + 4], S[(r0 + gid + 8) * SS + k0 + tig + 4]};
                    uint32_t ah[4], al[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        ah[e] = tf32_hi(af[e]);
                        al[e] = tf32_hi(af[e] - __uint_as_float(ah[e]));
                    }
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int j = col0 + 8 * hh + gid;
                        // op(A_c)(k, j): A_c[k][j] forwards, A_c[j][k] backwards
                        const float bf[2] = {fwd ? Ab[(k0 + tig) * SA + j] : Ab[j * SAT + k0 + tig],
                                             fwd ? Ab[(k0 + tig + 4) * SA + j] : Ab[j * SAT + k0 + tig + 4]};
                        uint32_t bh[2], bl[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            bh[e] = tf32_hi(bf[e]);
                            bl[e] = tf32_hi(bf[e] - __uint_as_float(bh[e]));
                        }
                        mma_tf32(dlh[hh], al, bh);
                        mma_tf32(dhl[hh], ah, bl);
                        mma_tf32(dhh[hh], ah, bh);
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    res[u][e] += (dlh[e >> 2][e & 3] + dhl[e >> 2][e & 3]) + dhh[e >> 2][e & 3];
            }
            __syncthreads();                                   // every read of S is done
            float* kp = keep ? keep + ((size_t)hd * nc + c + shift) * DD : nullptr;
#pragma unroll
            for (int u = 0; u < TPW; ++u) {
                const int t = warp + u * NW, r0 = (t / TN) * 16, col0 = (t % TN) * 16;
                if (t >= NTILE) continue;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int row = r0 + gid + (((e >> 1) & 1) << 3), col = col0 + 8 * (e >> 2) + 2 * tig + (e & 1);
                    S[row * SS + col] = res[u][e];
                    if (kp) kp[row * D + col] = res[u][e];
                }
            }
        }
        __syncthreads();
    };
    // forward: S_0 kept at ckpt[0]; S_{c+1} = B_c + S_c A_c kept at ckpt[c + 1], c = 0 .. nc-2
    for (int i = tid; i < DD; i += NT) {
        const float x = p.S0 ? p.S0[(size_t)hd * DD + i] : 0.f;
        S[(i / D) * SS + i % D] = x;
        p.ckpt[(size_t)hd * nc * DD + i] = x;
    }
    __syncthreads();
    run(true, 0, 1, nc - 1, p.ckpt, 1, 1);
    // backward: dS_L(nc-1) = dS_T kept at dsl[nc-1]; dS_L(c-1) = G_c + dS_L(c) A_c^T kept at
    // dsl[c-1], c = nc-1 .. 1; then dS0 = G_0 + dS_L(0) A_0^T
    for (int i = tid; i < DD; i += NT) {
        const float x = p.dS_T ? p.dS_T[(size_t)hd * DD + i] : 0.f;
        S[(i / D) * SS + i % D] = x;
        p.dsl[((size_t)hd * nc + nc - 1) * DD + i] = x;
    }
    __syncthreads();
    run(false, nc - 1, -1, nc - 1, p.dsl, -1, 2);
    run(false, 0, -1, 1, nullptr, 0, 2);
    if (p.dS0)
        for (int i = tid; i < DD; i += NT) p.dS0[(size_t)hd * DD + i] = S[(i / D) * SS + i % D];
}

// Pass 2 on the tensor cores (d = 128): the same chains, one step S <- X_c + S op(A_c) as
// tcgen05 kind::tf32 MMAs (M = N = 128) with each operand split into a tf32 high part and
// remainder (hi hi + hi lo + lo hi: fp32 accuracy).  S (hi, lo) is the A operand in tensor memory
// (lane = row), op(A_c) (hi, lo) the B operand in shared memory (K-major, 128-byte swizzle), and
// the accumulator starts as X_c (B_c forwards, G_c backwards).  Warps 0-3 own the TMEM rows
// (X_c in, the new S out to the workspace and back into TMEM as hi / lo); the other warps split
// A_c into the B operand; thread 0 issues the MMAs; the next A_c is fetched asynchronously
// while the MMAs run.
constexpr uint32_t TC_BHI = 0, TC_BLO = 65536, TC_RAW = 131072;     // byte offsets (1024-aligned base)
constexpr int TC_RS = 132;                                            // row stride of the raw A_c (floats)
constexpr uint32_t TC_BAR = TC_RAW + 128u * TC_RS * 4u;
constexpr size_t TC_SMEM_BYTES = TC_BAR + 64 + 1024;                 // + barrier, TMEM slot, alignment
constexpr uint32_t TC_COL_D = 0, TC_COL_HI = 128, TC_COL_LO = 256;   // TMEM columns

// byte offset of element (row n, k) of a 128 x 128 tf32 operand, K-major, 128-byte swizzle
__device__ __forceinline__ uint32_t tf32_koff(uint32_t n, uint32_t k) {
    return (k >> 5) * 16384u + tc::sw128_off(n, (k & 31u) >> 2) + (k & 3u) * 4u;
}

__global__ void __launch_bounds__(NT, 1) bwd_chain_tc_kernel(BwdParams p) {
    using namespace tc;
    constexpr int D = 128;
    constexpr int DD = D * D;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (sb - raw_u32);
    float* raw = reinterpret_cast<float*>(base + TC_RAW);
    uint64_t* bar = reinterpret_cast<uint64_t*>(base + TC_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + TC_BAR + 16);
    int* fail = reinterpret_cast<int*>(base + TC_BAR + 20);
    const int tid = (int)threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hd = (int)blockIdx.x, nc = (p.T + C - 1) / C;
    const uint64_t limit = 2000000000ull;
    if (!GDR_INB(hd < p.B * p.H, 405)) return;     // (the whole CTA)
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        *fail = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tq = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    const int row = (warp & 3) * 32 + lane;          // warps 0-3: this thread's row of S
    auto coef = [&](int c, int k) -> const float* { return p.coef + (((size_t)hd * nc + c) * 3 + k) * DD; };
    auto prefetch = [&](int c) {
        for (int i = tid; i < DD / 4; i += NT) {
            const int r = (4 * i) / D, cc = (4 * i) % D;
            cp_async16(raw + r * TC_RS + cc, coef(c, 0) + 4 * i);
        }
        cp_async_commit();
    };
    // row `row` of S (fp32, 128 values) -> TMEM hi / lo columns; also to `keep` (a workspace row)
    auto put_rows = [&](const float (&v)[32], int g) {
        float hi[32], lo[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            hi[u] = __uint_as_float(tf32_hi(v[u]));
            lo[u] = v[u] - hi[u];
        }
        tmem_st16(tq + TC_COL_HI + g * 32, *reinterpret_cast<const float(*)[16]>(hi));
        tmem_st16(tq + TC_COL_HI + g * 32 + 16, *reinterpret_cast<const float(*)[16]>(hi + 16));
        tmem_st16(tq + TC_COL_LO + g * 32, *reinterpret_cast<const float(*)[16]>(lo));
        tmem_st16(tq + TC_COL_LO + g * 32 + 16, *reinterpret_cast<const float(*)[16]>(lo + 16));
    };
    // the start matrix (S0 forwards, dS_T backwards) into TMEM and kept at `keep`
    auto start = [&](const float* src, float* keep) {
        if (warp < 4) {
#pragma unroll 1
            for (int g = 0; g < 4; ++g) {
                float v[32];
#pragma unroll
                for (int u4 = 0; u4 < 8; ++u4) {
                    const float4 x = src ? *reinterpret_cast<const float4*>(src + (size_t)row * D + g * 32 + 4 * u4)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[4 * u4] = x.x; v[4 * u4 + 1] = x.y; v[4 * u4 + 2] = x.z; v[4 * u4 + 3] = x.w;
                }
                put_rows(v, g);
                if (keep) {
#pragma unroll
                    for (int u4 = 0; u4 < 8; ++u4)
                        *reinterpret_cast<float4*>(keep + (size_t)row * D + g * 32 + 4 * u4) =
                            make_float4(v[4 * u4], v[4 * u4 + 1], v[4 * u4 + 2], v[4 * u4 + 3]);
                }
            }
            tmem_wait_st();
        }
    };
    uint32_t phase = 0;
    // n steps from chunk c0 in direction dc: S <- coef(c, add_k) + S op(A_c), kept at
    // keep + (hd * nc + c + shift) * DD unless keep is null; returns false on a timeout
    auto run = [&](bool fwd, int c0, int dc, int n, float* keep, int shift, int add_k, float* last_out) -> bool {
        if (n > 0) prefetch(c0);
        for (int st = 0; st < n; ++st) {
            const int c = c0 + st * dc;
            cp_async_wait_all();
            __syncthreads();                          // A_c landed; the last step's MMAs are done
            if (warp >= 4) {                          // A_c -> B operand (hi, lo)
                const int t = tid - 128;
                for (int e = t; e < DD; e += NT - 128) {
                    // B(n, k) = A_c[k][n] forwards, A_c[n][k] backwards; consecutive threads take
                    // consecutive k, so that the swizzled stores are conflict-free
                    const int nn = e / D, kk = e % D;
                    const float x = fwd ? raw[kk * TC_RS + nn] : raw[nn * TC_RS + kk];
                    const float hi = __uint_as_float(tf32_hi(x));
                    const uint32_t off = tf32_koff((uint32_t)nn, (uint32_t)kk);
                    *reinterpret_cast<float*>(base + TC_BHI + off) = hi;
                    *reinterpret_cast<float*>(base + TC_BLO + off) = x - hi;
                }
            } else {                                   // X_c -> the accumulator
                const float* xs = coef(c, add_k);
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    float v[32];
#pragma unroll
                    for (int u4 = 0; u4 < 8; ++u4) {
                        const float4 x = *reinterpret_cast<const float4*>(xs + (size_t)row * D + g * 32 + 4 * u4);
                        v[4 * u4] = x.x; v[4 * u4 + 1] = x.y; v[4 * u4 + 2] = x.z; v[4 * u4 + 3] = x.w;
                    }
                    tmem_st16(tq + TC_COL_D + g * 32, *reinterpret_cast<const float(*)[16]>(v));
                    tmem_st16(tq + TC_COL_D + g * 32 + 16, *reinterpret_cast<const float(*)[16]>(v + 16));
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();                          // B operand and accumulator ready; raw is free
            tc_fence_after();
            if (st + 1 < n) prefetch(c + dc);
            if (tid == 0) {
                const uint32_t id = idesc_tf32(128, 128);
#pragma unroll 1
                for (int term = 0; term < 3; ++term) {      // hi hi, lo hi, hi lo
                    const uint32_t acol = term == 1 ? TC_COL_LO : TC_COL_HI;
                    const uint32_t boff = term == 2 ? TC_BLO : TC_BHI;
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks) {
                        const uint32_t kb = ks >> 2, kin = (ks & 3) * 32;
                        mma_tf32_ts(tbase + TC_COL_D, tbase + acol + ks * 8,
                                    sdesc_sw128(sb + boff + kb * 16384 + kin, 16, 1024), id, 1);
                    }
                }
                mma_commit(bar);
                if (!mbar_wait_bounded(bar, phase, limit)) *fail = 1;
            }
            phase ^= 1u;
            __syncthreads();
            tc_fence_after();
            if (*fail) return false;
            if (warp < 4) {                            // the new S: kept, and back into TMEM
                float* kp = keep ? keep + ((size_t)hd * nc + c + shift) * DD : last_out;
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    float v[32];
                    tmem_ld32(tq + TC_COL_D + g * 32, v);
                    if (kp) {
#pragma unroll
                        for (int u4 = 0; u4 < 8; ++u4)
                            *reinterpret_cast<float4*>(kp + (size_t)row * D + g * 32 + 4 * u4) =
                                make_float4(v[4 * u4], v[4 * u4 + 1], v[4 * u4 + 2], v[4 * u4 + 3]);
                    }
                    put_rows(v, g);
                }
                tmem_wait_st();
            }
            tc_fence_before();
        }
        return true;
    };
    bool ok = true;
    // forward: S_0 kept at ckpt[0]; S_{c+1} = B_c + S_c A_c kept at ckpt[c + 1], c = 0 .. nc-2
    start(p.S0 ? p.S0 + (size_t)hd * DD : nullptr, p.ckpt + (size_t)hd * nc * DD);
    ok = run(true, 0, 1, nc - 1, p.ckpt, 1, 1, nullptr);
    // backward: dS_L(nc-1) = dS_T kept at dsl[nc-1]; dS_L(c-1) = G_c + dS_L(c) A_c^T kept at
    // dsl[c-1], c = nc-1 .. 1; then dS0 = G_0 + dS_L(0) A_0^T
    if (ok) {
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        start(p.dS_T ? p.dS_T + (size_t)hd * DD : nullptr, p.dsl + ((size_t)hd * nc + nc - 1) * DD);
        ok = run(false, nc - 1, -1, nc - 1, p.dsl, -1, 2, nullptr);
    }
    if (ok) ok = run(false, 0, -1, 1, nullptr, 0, 2, p.dS0 ? p.dS0 + (size_t)hd * DD : nullptr);
    if (!ok && tid == 0) atomicOr(&g_device_status, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

// Shared memory of the chain kernel: the carried matrix and two buffers of A_c.
template <int D>
constexpr size_t chain_smem_bytes() { return sizeof(float) * ((size_t)D * (D + 4) + 2 * (size_t)D * (D + 8)); }

// Pass 3: every chunk's gradients from its start state and its end state's gradient.
template <int DK, int DV, typename QT, typename OT>
__global__ void __launch_bounds__(NT, 1) bwd_grad_kernel(BwdParams p) {
    extern __shared__ float4 sm4[];
    float* sm = reinterpret_cast<float*>(sm4);
    __shared__ int range_f;
    const int tid = (int)threadIdx.x;
    const int nc = (p.T + C - 1) / C, ntask = p.B * p.H * nc;
    float* W = p.scratch + (size_t)blockIdx.x * p.scratch_floats;
    if (tid == 0) range_f = 0;
    for (int t = (int)blockIdx.x; t < ntask; t += (int)gridDim.x) {
        const int hd = t / nc, c = t % nc, b = hd / p.H, h = hd % p.H;
        if (!GDR_INB(hd < p.B * p.H, 404)) break;
        const float* S0c = p.ckpt + (size_t)t * DV * DK;
        const float* dSL = p.dsl + (size_t)t * DV * DK;
        chunk_forward<DK, DV, QT, OT>(p, W, b, h, c * C, S0c, true, &range_f, sm);
        chunk_grads<DK, DV, QT, OT>(p, W, b, h, c * C, S0c, dSL, sm);
    }
    if (tid == 0 && range_f) atomicOr(&g_device_status, STATUS_RANGE);
}

}  // namespace bwd
}  // namespace gdr
