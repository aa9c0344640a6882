// decode.cuh -- one recurrent decode step, HBM-bound: S is read once and written once.
//
// Per value row s (one row of S, dk wide), with X = S D_t:
//   x_k = (s D_t) . k,   x_q = (s D_t) . q,   e = w v_row - beta x_k  (w = beta unless given)
//   s  <- s D_t + e k^T,   o_row = x_q + e (k . q)
// which is the token update of the "Semidirect Fourier Delta Attention" page
// ("Core architecture": decay, erase along k, write v) transposed to value rows,
// with the readout o = S_t q taken from the updated row without a second pass.
//
// Layout: one warp owns a row at a time; lane l holds dims [VEC*l, VEC*l + VEC)
// (VEC = dk/32), so a row is one coalesced 128-bit (dk = 128) access per lane.
// Streaming: a persistent grid (2 CTAs of 8 warps per SM); each warp walks work items of 16
// rows of one head (items w, w + W, ...), 8 rows at a time, with the loads of the next 8 rows
// (of this item or of the next one) in flight while the current rows are computed, so that the
// state streams through the SM without gaps between items.  (Measured against 4 CTAs of
// 4-row batches, which spill at the 64-register cap, and the earlier one-shot CTAs of 64 rows:
// 108-112 us per 256 x 16 step against 119-120 and 113-114 us.)
#pragma once

#include "common.cuh"

namespace gdr {
namespace dec {

struct DecParams {
    int N, H, dv;
    int gate_mode;
    float scale;
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* w;         // write strength [N,H], or nullptr: w = beta
    int qk_norm;            // 1: L2-normalise q and k first (x / sqrt(sum x^2 + 1e-6))
    const float* theta;
    float* S;
    void* o;
};

constexpr int WARPS = 8;
constexpr int CTAS_PER_SM = 2;
constexpr int RB = 8;                         // rows per batch (one load each per lane, in flight)
constexpr int RI = 16;                        // rows per work item
constexpr int NB = RI / RB;

template <int VEC> struct Vec;
template <> struct Vec<4> { using T = float4; };
template <> struct Vec<2> { using T = float2; };
template <> struct Vec<1> { using T = float; };

template <int VEC>
__device__ __forceinline__ void unpack(const typename Vec<VEC>::T& x, float (&a)[VEC]) {
    if constexpr (VEC == 4) { a[0] = x.x; a[1] = x.y; a[2] = x.z; a[3] = x.w; }
    else if constexpr (VEC == 2) { a[0] = x.x; a[1] = x.y; }
    else { a[0] = x; }
}
template <int VEC>
__device__ __forceinline__ typename Vec<VEC>::T pack(const float (&a)[VEC]) {
    if constexpr (VEC == 4) return make_float4(a[0], a[1], a[2], a[3]);
    else if constexpr (VEC == 2) return make_float2(a[0], a[1]);
    else return a[0];
}

template <int DK, bool ROT, typename QT, typename OT>
__global__ void __launch_bounds__(WARPS * 32, CTAS_PER_SM) decode_kernel(DecParams p) {
    constexpr int VEC = DK / 32;
    static_assert(!ROT || VEC % 2 == 0 || VEC == 1, "pairs");
    using VT = typename Vec<VEC>::T;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int iph = p.dv / RI;                                // items per head (dv: 32, 64, 128)
    const int items = p.N * p.H * iph;
    const int W = (int)gridDim.x * WARPS;
    auto row_ptr = [&](int item, int r) -> VT* {
        const int nh = item / iph, row = (item % iph) * RI + r;
        return reinterpret_cast<VT*>(p.S + ((size_t)nh * p.dv + row) * DK) + lane;
    };
    VT sv[2][RB];
    int it = (int)blockIdx.x * WARPS + warp;
    if (it < items && GDR_INB(it / iph < p.N * p.H, 301)) {
#pragma unroll
        for (int r = 0; r < RB; ++r) sv[0][r] = __ldcs(row_ptr(it, r));
    }
    int cur = 0;
    for (; it < items; it += W) {
        const int nh = it / iph, row0 = (it % iph) * RI;
        if (!GDR_INB(nh < p.N * p.H, 302)) break;
        const QT* q = static_cast<const QT*>(p.q) + (size_t)nh * DK;
        const QT* k = static_cast<const QT*>(p.k) + (size_t)nh * DK;
        const QT* v = static_cast<const QT*>(p.v) + (size_t)nh * p.dv;
        OT* o = static_cast<OT*>(p.o) + (size_t)nh * p.dv;

        // This lane's slice of k, q and the decay (real: per dim; rotation: per pair).
        float kk[VEC], qq[VEC], al[VEC], cs[VEC], sn[VEC];
#pragma unroll
        for (int u = 0; u < VEC; ++u) {
            const int d = lane * VEC + u;
            kk[u] = ld_f32(k + d);
            qq[u] = ld_f32(q + d);
        }
        {
            float ik = 1.f, iq = p.scale;
            if (p.qk_norm) {
                float sk = 0.f, sq = 0.f;
#pragma unroll
                for (int u = 0; u < VEC; ++u) { sk = fmaf(kk[u], kk[u], sk); sq = fmaf(qq[u], qq[u], sq); }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                }
                ik = rsqrtf(sk + 1e-6f);
                iq = p.scale * rsqrtf(sq + 1e-6f);
            }
#pragma unroll
            for (int u = 0; u < VEC; ++u) { kk[u] *= ik; qq[u] *= iq; }
        }
        if constexpr (!ROT) {
#pragma unroll
            for (int u = 0; u < VEC; ++u) al[u] = decay_factor(p.g[(size_t)nh * DK + lane * VEC + u], p.gate_mode);
        } else if constexpr (VEC >= 2) {
#pragma unroll
            for (int u = 0; u < VEC; u += 2) {
                const int jp = (lane * VEC + u) / 2;
                const float a = decay_factor(p.g[(size_t)nh * (DK / 2) + jp], p.gate_mode);
                float s_, c_;
                sincosf(p.theta[(size_t)nh * (DK / 2) + jp], &s_, &c_);
                al[u] = a; cs[u] = c_; sn[u] = s_;
            }
        }
        // Rotation with one dim per lane (dk = 32): a pair spans lanes 2m, 2m+1.
        float pair_c = 0.f, pair_s = 0.f, pair_a = 0.f;
        if constexpr (ROT && VEC == 1) {
            const int jp = lane / 2;
            pair_a = decay_factor(p.g[(size_t)nh * (DK / 2) + jp], p.gate_mode);
            sincosf(p.theta[(size_t)nh * (DK / 2) + jp], &pair_s, &pair_c);
        }
        float kq = 0.f;
#pragma unroll
        for (int u = 0; u < VEC; ++u) kq = fmaf(kk[u], qq[u], kq);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        const float bt = p.beta[nh];
        const float wt = p.w ? p.w[nh] : bt;
        const float vrow = lane < RI ? ld_f32(v + row0 + lane) : 0.f;   // lane r: v of row r

        float orow = 0.f;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            // loads of the next batch: this item's, or the next item's first
            const int nit = b + 1 < NB ? it : it + W;
            const int nb = b + 1 < NB ? b + 1 : 0;
            if (nit < items) {
#pragma unroll
                for (int r = 0; r < RB; ++r) sv[cur ^ 1][r] = __ldcs(row_ptr(nit, nb * RB + r));
            }
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const int rr = b * RB + r;               // row within the item
                float s[VEC];
                unpack<VEC>(sv[cur][r], s);
                // X = s D_t
                if constexpr (!ROT) {
#pragma unroll
                    for (int u = 0; u < VEC; ++u) s[u] *= al[u];
                } else if constexpr (VEC >= 2) {
#pragma unroll
                    for (int u = 0; u < VEC; u += 2) {
                        const float x = s[u], y = s[u + 1];
                        s[u] = al[u] * (cs[u] * x - sn[u] * y);
                        s[u + 1] = al[u] * (sn[u] * x + cs[u] * y);
                    }
                } else {
                    const float other = __shfl_xor_sync(0xffffffffu, s[0], 1);
                    const float x = (lane & 1) ? other : s[0];
                    const float y = (lane & 1) ? s[0] : other;
                    s[0] = pair_a * ((lane & 1) ? (pair_s * x + pair_c * y) : (pair_c * x - pair_s * y));
                }
                float xk = 0.f, xq = 0.f;
#pragma unroll
                for (int u = 0; u < VEC; ++u) { xk = fmaf(s[u], kk[u], xk); xq = fmaf(s[u], qq[u], xq); }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    xk += __shfl_xor_sync(0xffffffffu, xk, off);
                    xq += __shfl_xor_sync(0xffffffffu, xq, off);
                }
                const float e = wt * __shfl_sync(0xffffffffu, vrow, rr) - bt * xk;
#pragma unroll
                for (int u = 0; u < VEC; ++u) s[u] = fmaf(e, kk[u], s[u]);
                __stcs(row_ptr(it, rr), pack<VEC>(s));
                if (lane == rr) orow = fmaf(e, kq, xq);
            }
            cur ^= 1;
        }
        if (lane < RI) st_from_f32(o + row0 + lane, orow);
    }
}

}  // namespace dec
}  // namespace gdr
