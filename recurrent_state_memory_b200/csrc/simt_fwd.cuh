// simt_fwd.cuh -- fp32 CUDA-core chunk-WY forward (every supported shape and mode).
//
// The WY/UT-transform chunk solver ("CARVE" page, section 1 item 3; "Semidirect
// Fourier Delta Attention" page, "Constructive Chunk-WY Theorem" and the exact
// affine chunk transfer) evaluated in fp32 on CUDA cores.  It is the precise path
// (fp32 mode) and the path for shapes the tensor-core kernel does not take.
//
// One CTA owns one (batch, head) and a DVT-wide slice of the value rows of S; the
// value rows are independent because every gate acts on the key axis ("CARVE"
// page, section 2 and Theorem 11).  Per chunk of C = 64 tokens, with Gamma_r the
// in-chunk cumulative log-decay (and Theta_r the cumulative angle in rotation
// mode), P_r = D_1 ... D_r:
//   A[r,i]  = beta_r k_i^T P_i^{-1} P_r k_r        (i < r)
//   Pm[r,i] = k_i^T P_i^{-1} P_r q_r               (i <= r)
//   E       = (I + A)^{-1} (diag(w) V - diag(beta) Ktil S^T),   Ktil_r = P_r k_r
//             (w: the write strength, w = beta unless given; beta erases)
//   O       = Qtil S^T + Pm E,                          Qtil_r = P_r q_r
//   S      <- S P_C + E^T Kdec,                         Kdec_i = P_C^T P_i^{-T} k_i
// A and Pm are formed with exp(Gamma_r - Gamma_i) inside the sum (no factoring),
// so no intermediate can overflow; E comes from forward substitution.
#pragma once

#include "common.cuh"

namespace gdr {

struct FwdParams {
    int B, H, T, dv;
    int head0, nheads;      // tensor-core kernels: heads [head0, head0 + nheads) of b*H + h
    int qk_norm;            // 1: L2-normalise q_t and k_t first (x / sqrt(sum x^2 + 1e-6))
    int gate_mode;
    float scale;
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* w;         // write strength [B,T,H], or nullptr: w = beta
    const float* theta;
    const float* S0;
    void* o;
    float* S_T;
    float* chunk_mean;      // [B, ceil(T/64), H, dv] fp32 mean of o over each chunk, or nullptr
    // Split tensor-core kernel only: with nseg > 1 each head's sequence runs as segments of
    // seg_len tokens (a multiple of 64), segments seg0 .. nseg-1, each as its own chain (a
    // "virtual head"): segment 0 starts from S0 (or zero), the others from zero, or every one
    // from the identity when s0_identity is set (dk = dv); S_T then holds one state per virtual
    // head.  v == nullptr means zero values.
    int nseg, seg_len, seg0, s0_identity;
};

namespace simt {

constexpr int C = 64;     // chunk length
constexpr int DVT = 32;   // value rows per CTA
constexpr int NT = 256;   // threads per CTA

template <int DK, bool ROT>
struct Smem {
    static constexpr int NG = ROT ? DK / 2 : DK;  // gate columns
    static constexpr int KS = DK + 1;             // padded row stride of k/q tiles
    static constexpr int off_k = 0;                         // raw k, later Kdec      [C][KS]
    static constexpr int off_q = off_k + C * KS;            // scale*q, later Qtil    [C][KS]
    static constexpr int off_kt = off_q + C * KS;           // Ktil                   [C][KS]
    static constexpr int off_G = off_kt + C * KS;           // cumulative log-decay   [C][NG]
    static constexpr int off_Th = off_G + C * NG;           // cumulative angle       [C][DK/2] (ROT)
    static constexpr int off_b = off_Th + (ROT ? C * (DK / 2) : 0);   // beta   [C]
    static constexpr int off_w = off_b + C;                 // write strength         [C]
    static constexpr int off_A = off_w + C;                 // A (strict lower)       [C][C+1]
    static constexpr int off_P = off_A + C * (C + 1);       // Pm (lower, inclusive)  [C][C+1]
    static constexpr int off_S = off_P + C * (C + 1);       // state slice            [DVT][KS]
    static constexpr int off_R = off_S + DVT * KS;          // RHS, then E            [C][DVT+1]
    static constexpr int off_QS = off_R + C * (DVT + 1);    // Qtil S^T               [C][DVT+1]
    static constexpr int off_dec = off_QS + C * (DVT + 1);  // chunk decay: re / im   [2][NG]
    static constexpr int total = off_dec + 2 * NG;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int DK, bool ROT, typename QT, typename OT>
__global__ void __launch_bounds__(NT) chunk_fwd_kernel(FwdParams p) {
    using L = Smem<DK, ROT>;
    constexpr int NG = L::NG;
    constexpr int KS = L::KS;
    extern __shared__ float sm[];
    float* kc = sm + L::off_k;
    float* qc = sm + L::off_q;
    float* kt = sm + L::off_kt;
    float* Gc = sm + L::off_G;
    float* Th = sm + L::off_Th;
    float* bc = sm + L::off_b;
    float* wc = sm + L::off_w;
    float* Am = sm + L::off_A;
    float* Pm = sm + L::off_P;
    float* S = sm + L::off_S;
    float* R = sm + L::off_R;
    float* QS = sm + L::off_QS;
    float* dec = sm + L::off_dec;

    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh % p.H;
    const int j0 = blockIdx.y * DVT;
    const int dv = p.dv;
    const QT* __restrict__ q = static_cast<const QT*>(p.q);
    const QT* __restrict__ k = static_cast<const QT*>(p.k);
    const QT* __restrict__ v = static_cast<const QT*>(p.v);
    OT* __restrict__ o = static_cast<OT*>(p.o);

    // Initial state slice.
    for (int idx = tid; idx < DVT * DK; idx += NT) {
        const int j = idx / DK, d = idx % DK;
        S[j * KS + d] = p.S0 ? p.S0[((size_t)bh * dv + j0 + j) * DK + d] : 0.f;
    }

    const int nchunks = (p.T + C - 1) / C;
    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * C;
        const int Lc = min(C, p.T - t0);
        auto tok = [&](int r) -> size_t { return ((size_t)b * p.T + (t0 + r)) * p.H + h; };
        __syncthreads();  // previous chunk fully consumed

        // 1. Load the chunk; apply the gate activation.
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int r = idx / DK, d = idx % DK;
            float kv = 0.f, qv = 0.f;
            if (r < Lc) {
                kv = ld_f32(k + tok(r) * DK + d);
                qv = ld_f32(q + tok(r) * DK + d);
                if (!p.qk_norm) qv *= p.scale;
            }
            kc[r * KS + d] = kv;
            qc[r * KS + d] = qv;
        }
        if (p.qk_norm) {
            // L2-normalise every token's k and q (one warp per row), then scale q
            __syncthreads();
            const int wid = tid >> 5, ln = tid & 31;
            for (int r = wid; r < C; r += NT / 32) {
                float sk = 0.f, sq = 0.f;
                for (int d = ln; d < DK; d += 32) {
                    sk = fmaf(kc[r * KS + d], kc[r * KS + d], sk);
                    sq = fmaf(qc[r * KS + d], qc[r * KS + d], sq);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                }
                const float ik = rsqrtf(sk + 1e-6f), iq = p.scale * rsqrtf(sq + 1e-6f);
                for (int d = ln; d < DK; d += 32) {
                    kc[r * KS + d] *= ik;
                    qc[r * KS + d] *= iq;
                }
            }
        }
        for (int idx = tid; idx < C * NG; idx += NT) {
            const int r = idx / NG, jg = idx % NG;
            Gc[idx] = r < Lc ? log_decay(p.g[tok(r) * NG + jg], p.gate_mode) : 0.f;
            if (ROT) Th[idx] = r < Lc ? p.theta[tok(r) * (DK / 2) + jg] : 0.f;
        }
        if (tid < C) bc[tid] = tid < Lc ? p.beta[tok(tid)] : 0.f;
        if (tid < C) wc[tid] = tid < Lc ? (p.w ? p.w[tok(tid)] : p.beta[tok(tid)]) : 0.f;
        __syncthreads();

        // 2. In-chunk prefix sums: Gamma_r (and Theta_r, kept in [-pi, pi]).
        for (int col = tid; col < NG * (ROT ? 2 : 1); col += NT) {
            if (col < NG) {
                float acc = 0.f;
                for (int r = 0; r < Lc; ++r) { acc += Gc[r * NG + col]; Gc[r * NG + col] = acc; }
            } else {
                const int jc = col - NG;
                float acc = 0.f;
                for (int r = 0; r < Lc; ++r) { acc = wrap_angle(acc + Th[r * NG + jc]); Th[r * NG + jc] = acc; }
            }
        }
        __syncthreads();

        // 3. A and Pm, with the exact decay exp(Gamma_r - Gamma_i) <= 1 in every term.
        for (int idx = tid; idx < C * C; idx += NT) {
            const int r = idx / C, i = idx % C;
            float sa = 0.f, sp = 0.f;
            if (i <= r && r < Lc) {
                const float* kr = kc + r * KS;
                const float* ki = kc + i * KS;
                const float* qr = qc + r * KS;
                const float* Gr = Gc + r * NG;
                const float* Gi = Gc + i * NG;
                if (!ROT) {
#pragma unroll 8
                    for (int d = 0; d < DK; ++d) {
                        const float e = __expf(Gr[d] - Gi[d]);
                        const float ke = ki[d] * e;
                        sa = fmaf(kr[d], ke, sa);
                        sp = fmaf(qr[d], ke, sp);
                    }
                } else {
                    const float* Tr = Th + r * NG;
                    const float* Ti = Th + i * NG;
#pragma unroll 4
                    for (int jp = 0; jp < NG; ++jp) {
                        const float e = __expf(Gr[jp] - Gi[jp]);
                        float sn, cs;
                        __sincosf(Tr[jp] - Ti[jp], &sn, &cs);
                        const float ki0 = ki[2 * jp], ki1 = ki[2 * jp + 1];
                        const float kr0 = kr[2 * jp], kr1 = kr[2 * jp + 1];
                        const float qr0 = qr[2 * jp], qr1 = qr[2 * jp + 1];
                        sa += e * (cs * (ki0 * kr0 + ki1 * kr1) + sn * (ki0 * kr1 - ki1 * kr0));
                        sp += e * (cs * (ki0 * qr0 + ki1 * qr1) + sn * (ki0 * qr1 - ki1 * qr0));
                    }
                }
            }
            Am[r * (C + 1) + i] = (i < r) ? bc[r] * sa : 0.f;
            Pm[r * (C + 1) + i] = sp;
        }
        // Chunk-end decay of the state (per key dim, or per pair as a complex factor).
        for (int jg = tid; jg < NG; jg += NT) {
            const float GC = Lc > 0 ? Gc[(Lc - 1) * NG + jg] : 0.f;
            const float m = expf(GC);
            if (ROT) {
                const float ThC = Lc > 0 ? Th[(Lc - 1) * NG + jg] : 0.f;
                float sn, cs;
                sincosf(ThC, &sn, &cs);
                dec[jg] = m * cs;
                dec[NG + jg] = m * sn;
            } else {
                dec[jg] = m;
            }
        }
        __syncthreads();

        // 4. Ktil, Qtil (in place of q) and Kdec (in place of k).
        for (int idx = tid; idx < C * NG; idx += NT) {
            const int r = idx / NG, jg = idx % NG;
            const float G = Gc[r * NG + jg];
            const float GC = Lc > 0 ? Gc[(Lc - 1) * NG + jg] : 0.f;
            if (!ROT) {
                const float m = expf(G), md = expf(GC - G);
                const float kv = kc[r * KS + jg];
                kt[r * KS + jg] = kv * m;
                qc[r * KS + jg] *= m;
                kc[r * KS + jg] = kv * md;
            } else {
                const float Tr = Th[r * NG + jg];
                const float ThC = Lc > 0 ? Th[(Lc - 1) * NG + jg] : 0.f;
                float s1, c1, s2, c2;
                sincosf(Tr, &s1, &c1);
                sincosf(wrap_angle(ThC - Tr), &s2, &c2);
                const float m = expf(G), md = expf(GC - G);
                const float k0 = kc[r * KS + 2 * jg], k1 = kc[r * KS + 2 * jg + 1];
                const float q0 = qc[r * KS + 2 * jg], q1 = qc[r * KS + 2 * jg + 1];
                kt[r * KS + 2 * jg] = m * (c1 * k0 + s1 * k1);          // e^{G} e^{-i Theta} kappa
                kt[r * KS + 2 * jg + 1] = m * (c1 * k1 - s1 * k0);
                qc[r * KS + 2 * jg] = m * (c1 * q0 + s1 * q1);
                qc[r * KS + 2 * jg + 1] = m * (c1 * q1 - s1 * q0);
                kc[r * KS + 2 * jg] = md * (c2 * k0 - s2 * k1);         // e^{GC-G} e^{i(ThC-Th)} kappa
                kc[r * KS + 2 * jg + 1] = md * (s2 * k0 + c2 * k1);
            }
        }
        __syncthreads();

        // 5. R = diag(w) V - diag(beta) Ktil S^T and QS = Qtil S^T.
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int r = idx / DVT, j = idx % DVT;
            float ks = 0.f, qs = 0.f;
            if (r < Lc) {
                const float* kr = kt + r * KS;
                const float* qr = qc + r * KS;
                const float* Sj = S + j * KS;
#pragma unroll 8
                for (int d = 0; d < DK; ++d) {
                    ks = fmaf(kr[d], Sj[d], ks);
                    qs = fmaf(qr[d], Sj[d], qs);
                }
                const float vv = ld_f32(v + tok(r) * dv + j0 + j);
                R[r * (DVT + 1) + j] = wc[r] * vv - bc[r] * ks;
            } else {
                R[r * (DVT + 1) + j] = 0.f;
            }
            QS[r * (DVT + 1) + j] = qs;
        }
        __syncthreads();

        // 6. Forward substitution (I + A) E = R, row by row; 8 lanes share a column.
        {
            const int part = tid & 7, j = tid >> 3;   // 32 columns x 8 partial sums
            for (int r = 1; r < Lc; ++r) {
                float s = 0.f;
                for (int i = part; i < r; i += 8) s = fmaf(Am[r * (C + 1) + i], R[i * (DVT + 1) + j], s);
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                s += __shfl_xor_sync(0xffffffffu, s, 4);
                if (part == 0) R[r * (DVT + 1) + j] -= s;
                __syncthreads();
            }
        }

        // 7. O = QS + Pm E.
        float msum = 0.f;     // chunk mean: this thread's column j = tid % DVT over its rows
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int r = idx / DVT, j = idx % DVT;
            if (r < Lc) {
                float acc = QS[r * (DVT + 1) + j];
                for (int i = 0; i <= r; ++i) acc = fmaf(Pm[r * (C + 1) + i], R[i * (DVT + 1) + j], acc);
                if (GDR_INB(t0 + r < p.T && bh < p.B * p.H && j0 + j < dv, 501)) st_from_f32(o + tok(r) * dv + j0 + j, acc);
                msum += acc;
            }
        }
        if (p.chunk_mean) {
            // mean of this chunk's outputs (fp32, before rounding to the output type); QS is
            // free once every thread is past step 7
            __syncthreads();
            QS[tid] = msum;
            __syncthreads();
            if (tid < DVT) {
                float s = 0.f;
                for (int w8 = 0; w8 < NT / DVT; ++w8) s += QS[w8 * DVT + tid];
                p.chunk_mean[(((size_t)b * nchunks + c) * p.H + h) * dv + j0 + tid] = s / (float)Lc;
            }
        }

        // 8. S <- S P_C + E^T Kdec.
        for (int idx = tid; idx < DVT * NG; idx += NT) {
            const int j = idx / NG, jg = idx % NG;
            if (!ROT) {
                float acc = S[j * KS + jg] * dec[jg];
                for (int i = 0; i < Lc; ++i) acc = fmaf(R[i * (DVT + 1) + j], kc[i * KS + jg], acc);
                S[j * KS + jg] = acc;
            } else {
                const float x = S[j * KS + 2 * jg], y = S[j * KS + 2 * jg + 1];
                const float cr = dec[jg], ci = dec[NG + jg];
                float a0 = cr * x - ci * y, a1 = ci * x + cr * y;
                for (int i = 0; i < Lc; ++i) {
                    const float e = R[i * (DVT + 1) + j];
                    a0 = fmaf(e, kc[i * KS + 2 * jg], a0);
                    a1 = fmaf(e, kc[i * KS + 2 * jg + 1], a1);
                }
                S[j * KS + 2 * jg] = a0;
                S[j * KS + 2 * jg + 1] = a1;
            }
        }
    }
    __syncthreads();
    if (p.S_T && GDR_INB(bh < p.B * p.H && j0 + DVT <= dv, 502)) {
        for (int idx = tid; idx < DVT * DK; idx += NT) {
            const int j = idx / DK, d = idx % DK;
            p.S_T[((size_t)bh * dv + j0 + j) * DK + d] = S[j * KS + d];
        }
    }
}

}  // namespace simt
}  // namespace gdr
