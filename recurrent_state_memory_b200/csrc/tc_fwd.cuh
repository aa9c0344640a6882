// tc_fwd.cuh -- chunk-WY forward on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// The WY/UT-transform triangular chunk solver ("CARVE" page, section 1 item 3 and
// section 3 item 1; "Semidirect Fourier Delta Attention" page, "Constructive Chunk-WY
// Theorem" and the exact affine chunk transfer), bf16 operands, fp32 accumulation,
// dk = dv = 128, chunk C = 64.  One CTA owns one (batch, head); the state S (dv x dk,
// fp32) stays resident in tensor memory for the whole sequence.
//
// Per chunk, with P_r = D_1 ... D_r and a reference token m = 31 (the middle of the
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
// which is the same algebra as the SIMT kernel with the reference moved from the chunk
// start to its middle.  A tail chunk is padded with identity tokens (g = 0, beta = 0).
//
// Shared-memory tiles use the 128-byte swizzle; every tile is either K-major (rows of
// 128 B along K) or MN-major (rows of 128 B along M/N), and the K-major Khat tile doubles
// as the MN-major B operand of the state update.  TMEM columns (lane = row):
//   [0,128) S   [128,192) O^T   [192,256) U^T / E^T   [256,320) [A' ; Pmat]   [320,384) Wm^T
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdr {
namespace tcf {

constexpr int C = 64;
constexpr int D = 128;          // dk = dv
constexpr int NT = 256;
constexpr uint32_t COL_S = 0, COL_O = 128, COL_E = 192, COL_A1 = 256, COL_W = 320;
constexpr uint32_t TMEM_COLS = 512;

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_KQ = 0;                      // [Ktil ; Qtil] K-major: 2 kblocks x 128 rows x 128 B
constexpr uint32_t OFF_KH = OFF_KQ + 32768;         // Khat K-major: 2 kblocks x 64 rows x 128 B
constexpr uint32_t OFF_V = OFF_KH + 16384;          // V, MN-major for V^T: 2 groups x 64 tokens x 128 B
constexpr uint32_t OFF_S = OFF_V + 16384;           // Stil bf16 K-major: 2 kblocks x 128 rows x 128 B
constexpr uint32_t OFF_E = OFF_S + 32768;           // E^T bf16 K-major: 128 rows x 128 B
constexpr uint32_t OFF_W = OFF_E + 16384;           // Wm^T bf16 MN-major: 128 dk rows x 128 B
constexpr uint32_t OFF_TB = OFF_W + 16384;          // Tb K-major: 64 rows x 128 B
constexpr uint32_t OFF_PM = OFF_TB + 8192;          // Pm K-major: 64 rows x 128 B
constexpr uint32_t OFF_AF = OFF_PM + 8192;          // fp32 A [64][65]
constexpr uint32_t OFF_TF = OFF_AF + 64 * 65 * 4;   // fp32 Tm [64][65]
constexpr uint32_t OFF_XF = OFF_TF + 64 * 65 * 4;   // fp32 scratch [3][16][17]
constexpr uint32_t OFF_VEC = OFF_XF + 3 * 16 * 17 * 4;  // beta[64], rho_ref[2][128], rho_C[2][128]
constexpr uint32_t OFF_BAR = (OFF_VEC + (64 + 4 * 128) * 4 + 15) & ~15u;
constexpr uint32_t SMEM_USED = OFF_BAR + 32;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // slack for 1024-byte alignment

// Device status bits (gdr_query_device_status).
constexpr unsigned STATUS_TIMEOUT = 1u;
constexpr unsigned STATUS_RANGE = 2u;

struct TcExtra {
    unsigned long long wait_limit_ns;   // bound on every mbarrier wait
    int fault_skip_commit;              // test hook: 1 = never signal the first MMA barrier
};

template <bool ROT, typename OT>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_tc_kernel(FwdParams p, TcExtra x) {
    using namespace tc;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;          // shared-window base address
    uint8_t* base = smem_raw + (sb - raw_u32);               // generic pointer to the same byte
    float* Af = reinterpret_cast<float*>(base + OFF_AF);
    float* Tf = reinterpret_cast<float*>(base + OFF_TF);
    float* Xf = reinterpret_cast<float*>(base + OFF_XF);
    float* sbeta = reinterpret_cast<float*>(base + OFF_VEC);
    float* rho_ref = sbeta + 64;          // [2][128]: re, im (real mode uses re only)
    float* rho_C = rho_ref + 256;         // [2][128]
    uint64_t* bar = reinterpret_cast<uint64_t*>(base + OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + OFF_BAR + 8);
    int* abort_flag = reinterpret_cast<int*>(base + OFF_BAR + 12);
    int* range_flag = reinterpret_cast<int*>(base + OFF_BAR + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;                        // TMEM lane owned by this thread
    const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
    const __nv_bfloat16* __restrict__ q = static_cast<const __nv_bfloat16*>(p.q);
    const __nv_bfloat16* __restrict__ k = static_cast<const __nv_bfloat16*>(p.k);
    const __nv_bfloat16* __restrict__ v = static_cast<const __nv_bfloat16*>(p.v);
    OT* __restrict__ o = static_cast<OT*>(p.o);

    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        *abort_flag = 0;
        *range_flag = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tq = tbase + ((uint32_t)(quad * 32) << 16);   // this warp's lane quadrant
    uint32_t phase = 0;
    bool skip_commit = x.fault_skip_commit != 0;

    // Issue-side helper: one thread commits, every thread waits (bounded).
    auto commit_and_wait = [&]() -> bool {
        if (tid == 0) {
            if (!skip_commit) mma_commit(bar);
            skip_commit = false;
        }
        bool ok = mbar_wait_bounded(bar, phase, x.wait_limit_ns);
        phase ^= 1u;
        if (!ok) atomicExch(abort_flag, 1);
        tc_fence_after();
        __syncthreads();
        return *abort_flag == 0;
    };
    // Make generic smem writes and TMEM stores visible to the MMA issued next.
    auto publish = [&]() {
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    const uint32_t ID_128x64_KK = idesc_bf16(128, 64, 0, 0, 0);
    const uint32_t ID_128x64_MK = idesc_bf16(128, 64, 1, 0, 0);
    const uint32_t ID_128x64_KMneg = idesc_bf16(128, 64, 0, 1, 1);
    const uint32_t ID_128x128_KM = idesc_bf16(128, 128, 0, 1, 0);

    const int nchunks = (p.T + C - 1) / C;
    bool failed = false;
    for (int c = 0; c < nchunks && !failed; ++c) {
        const int t0 = c * C;
        const int Lc = min(C, p.T - t0);
        auto tok = [&](int r) -> size_t { return ((size_t)b * p.T + (t0 + r)) * p.H + h; };

        // ---------------- prep: gate, decay factors, operand tiles -------------
        if (tid < 128) {
            const int pp = tid & 63;                 // key pair: dims 2pp, 2pp+1
            const int hf = tid >> 6;                 // 0: tokens 31..0 (backward), 1: 32..63
            const uint32_t kb = (uint32_t)(pp >> 5);
            const uint32_t ch = (uint32_t)((pp & 31) >> 2);
            const uint32_t in_ch = (uint32_t)(pp & 3) * 4u;
            bool bad = false;
            float P0 = 1.f, P1 = 1.f, Q0 = 1.f, Q1 = 1.f;    // alpha / (1/alpha) products
            float Rre = 1.f, Rim = 0.f;                     // rotation phase product
            for (int s = 0; s < 32; ++s) {
                const int r = hf ? 32 + s : 31 - s;
                float k0 = 0.f, k1 = 0.f, q0 = 0.f, q1 = 0.f;
                float al0 = 1.f, al1 = 1.f, iv0 = 1.f, iv1 = 1.f, cth = 1.f, sth = 0.f;
                if (r < Lc) {
                    const size_t tk = tok(r);
                    const __nv_bfloat162 kk = *reinterpret_cast<const __nv_bfloat162*>(k + tk * D + 2 * pp);
                    const __nv_bfloat162 qq = *reinterpret_cast<const __nv_bfloat162*>(q + tk * D + 2 * pp);
                    k0 = __low2float(kk); k1 = __high2float(kk);
                    q0 = p.scale * __low2float(qq); q1 = p.scale * __high2float(qq);
                    if (!ROT) {
                        const float2 a2 = *reinterpret_cast<const float2*>(p.g + tk * D + 2 * pp);
                        if (p.gate_mode == 1) {
                            const float e0 = __expf(a2.x), e1 = __expf(a2.y);
                            iv0 = 1.f + e0; iv1 = 1.f + e1;
                            al0 = __frcp_rn(iv0); al1 = __frcp_rn(iv1);
                        } else {
                            al0 = __expf(a2.x); al1 = __expf(a2.y);
                            iv0 = __expf(-a2.x); iv1 = __expf(-a2.y);
                        }
                    } else {
                        const float a1 = p.g[tk * (D / 2) + pp];
                        if (p.gate_mode == 1) {
                            const float e0 = __expf(a1);
                            iv0 = 1.f + e0;
                            al0 = __frcp_rn(iv0);
                        } else {
                            al0 = __expf(a1);
                            iv0 = __expf(-a1);
                        }
                        al1 = al0; iv1 = iv0;
                        sincosf(p.theta[tk * (D / 2) + pp], &sth, &cth);
                    }
                }
                float F0, F1, G0, G1, Fim = 0.f, Gim = 0.f;
                if (hf) {   // include token r, then use it
                    P0 *= al0; P1 *= al1; Q0 *= iv0; Q1 *= iv1;
                    if (ROT) {   // R *= e^{-i theta}
                        const float nre = Rre * cth + Rim * sth, nim = Rim * cth - Rre * sth;
                        Rre = nre; Rim = nim;
                    }
                    F0 = P0; F1 = P1; G0 = Q0; G1 = Q1;
                } else {    // use the product over tokens r+1..31, then include r
                    F0 = Q0; F1 = Q1; G0 = P0; G1 = P1;
                }
                float kt0, kt1, qt0, qt1, kh0, kh1;
                if (!ROT) {
                    kt0 = k0 * F0; kt1 = k1 * F1; qt0 = q0 * F0; qt1 = q1 * F1;
                    kh0 = k0 * G0; kh1 = k1 * G1;
                } else {
                    // F = |F| R, G = |G| R (complex), applied to kappa = k0 + i k1
                    const float fr = F0 * Rre, fi = F0 * Rim, gr = G0 * Rre, gi = G0 * Rim;
                    kt0 = fr * k0 - fi * k1; kt1 = fr * k1 + fi * k0;
                    qt0 = fr * q0 - fi * q1; qt1 = fr * q1 + fi * q0;
                    kh0 = gr * k0 - gi * k1; kh1 = gr * k1 + gi * k0;
                    (void)Fim; (void)Gim;
                }
                if (!(isfinite(kt0) && isfinite(kt1) && isfinite(kh0) && isfinite(kh1) &&
                      isfinite(qt0) && isfinite(qt1))) bad = true;
                *reinterpret_cast<uint32_t*>(base + OFF_KQ + kb * 16384u + sw128_off(r, ch) + in_ch) = pack_bf16x2(kt0, kt1);
                *reinterpret_cast<uint32_t*>(base + OFF_KQ + kb * 16384u + sw128_off(64 + r, ch) + in_ch) = pack_bf16x2(qt0, qt1);
                *reinterpret_cast<uint32_t*>(base + OFF_KH + kb * 8192u + sw128_off(r, ch) + in_ch) = pack_bf16x2(kh0, kh1);
                if (!hf) {
                    P0 *= al0; P1 *= al1; Q0 *= iv0; Q1 *= iv1;
                    if (ROT) {   // Rb *= e^{+i theta}
                        const float nre = Rre * cth - Rim * sth, nim = Rim * cth + Rre * sth;
                        Rre = nre; Rim = nim;
                    }
                }
            }
            if (bad) atomicExch(range_flag, 1);
            // hf = 0 ends with prod_{0..31} alpha = e^{Gamma_m} (and e^{i Theta_m});
            // hf = 1 ends with prod_{32..63} alpha = e^{Gamma_C - Gamma_m} (and e^{-i(...)}).
            float* dst = hf ? rho_C : rho_ref;
            if (!ROT) {
                dst[2 * pp] = P0; dst[2 * pp + 1] = P1;
            } else {
                dst[pp] = P0 * Rre;
                dst[128 + pp] = hf ? -P0 * Rim : P0 * Rim;   // forward product holds conj
            }
        } else {
            // V tile (MN-major: rows = tokens, 64 dv per group) and beta.
            const int u = tid - 128;
            const int j = u & 15;                    // 16-byte chunk of the 256-byte row
            for (int pass = 0; pass < 8; ++pass) {
                const int i = pass * 8 + (u >> 4);
                uint4 val = make_uint4(0, 0, 0, 0);
                if (i < Lc) val = *reinterpret_cast<const uint4*>(v + tok(i) * D + j * 8);
                *reinterpret_cast<uint4*>(base + OFF_V + (uint32_t)(j >> 3) * 8192u + sw128_off(i, j & 7)) = val;
            }
            if (u < 64) sbeta[u] = u < Lc ? p.beta[tok(u)] : 0.f;
        }
        publish();

        // ---------------- MMA1: [Ktil ; Qtil] Khat^T -> TMEM ----------------------
        if (tid == 0) {
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kb = ks >> 2, kin = (ks & 3) * 32;
                mma_bf16_ss(tbase + COL_A1, sdesc_sw128(sb + OFF_KQ + kb * 16384 + kin, 16, 1024),
                            sdesc_sw128(sb + OFF_KH + kb * 8192 + kin, 16, 1024), ID_128x64_KK, ks > 0);
            }
        }
        // Meanwhile: Stil = S P_m into TMEM (fp32) and shared memory (bf16 operand).
        {
            const int j = row;
            for (int g = 0; g < 4; ++g) {
                const int col0 = half * 64 + g * 16;
                float s[16];
                if (c == 0) {
                    if (p.S0) {
                        const float4* src = reinterpret_cast<const float4*>(p.S0 + ((size_t)bh * D + j) * D + col0);
#pragma unroll
                        for (int u4 = 0; u4 < 4; ++u4) {
                            const float4 t4 = src[u4];
                            s[4 * u4] = t4.x; s[4 * u4 + 1] = t4.y; s[4 * u4 + 2] = t4.z; s[4 * u4 + 3] = t4.w;
                        }
                    } else {
#pragma unroll
                        for (int u = 0; u < 16; ++u) s[u] = 0.f;
                    }
                } else {
                    tmem_ld16(tq + COL_S + col0, s);
                }
                if (!ROT) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) s[u] *= rho_ref[col0 + u];
                } else {
#pragma unroll
                    for (int u = 0; u < 16; u += 2) {
                        const int pr = (col0 + u) >> 1;
                        const float cr = rho_ref[pr], ci = rho_ref[128 + pr];
                        const float xr = s[u], xi = s[u + 1];
                        s[u] = xr * cr - xi * ci;
                        s[u + 1] = xr * ci + xi * cr;
                    }
                }
                tmem_st16(tq + COL_S + col0, s);
                const uint32_t kb = (uint32_t)col0 >> 6, c0 = ((uint32_t)col0 & 63u) >> 3;
                uint4 w0 = make_uint4(pack_bf16x2(s[0], s[1]), pack_bf16x2(s[2], s[3]),
                                      pack_bf16x2(s[4], s[5]), pack_bf16x2(s[6], s[7]));
                uint4 w1 = make_uint4(pack_bf16x2(s[8], s[9]), pack_bf16x2(s[10], s[11]),
                                      pack_bf16x2(s[12], s[13]), pack_bf16x2(s[14], s[15]));
                *reinterpret_cast<uint4*>(base + OFF_S + kb * 16384u + sw128_off(j, c0)) = w0;
                *reinterpret_cast<uint4*>(base + OFF_S + kb * 16384u + sw128_off(j, c0 + 1)) = w1;
            }
            tmem_wait_st();
        }
        if (!commit_and_wait()) { failed = true; break; }

        // ---------------- solve: Tm = (I + A)^{-1}, Pm masked --------------------
        {
            float vals[32];
            tmem_ld16(tq + COL_A1 + half * 32, *reinterpret_cast<float(*)[16]>(vals));
            tmem_ld16(tq + COL_A1 + half * 32 + 16, *reinterpret_cast<float(*)[16]>(vals + 16));
            if (row < 64) {
                const int r = row;
                const float br = sbeta[r];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const int i = half * 32 + u;
                    Af[r * 65 + i] = (i < r) ? br * vals[u] : 0.f;
                }
            } else {
                const int r = row - 64;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float m8[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int i = half * 32 + cc * 8 + u;
                        m8[u] = (i <= r) ? vals[cc * 8 + u] : 0.f;
                    }
                    *reinterpret_cast<uint4*>(base + OFF_PM + sw128_off(r, half * 4 + cc)) =
                        make_uint4(pack_bf16x2(m8[0], m8[1]), pack_bf16x2(m8[2], m8[3]),
                                   pack_bf16x2(m8[4], m8[5]), pack_bf16x2(m8[6], m8[7]));
                }
            }
            for (int e = tid; e < 64 * 65; e += NT) Tf[e] = 0.f;
        }
        __syncthreads();
        // 16x16 diagonal blocks by forward substitution (one warp per block, lane = column).
        if (warp < 4 && lane < 16) {
            const int bb = warp * 16, jj = lane;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float s_ = (r == jj) ? 1.f : 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i) s_ = fmaf(-Af[(bb + r) * 65 + bb + i], t[i], s_);
                t[r] = s_;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tf[(bb + r) * 65 + bb + jj] = t[r];
        }
        __syncthreads();
        // Off-diagonal blocks: T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ, by block distance.
        for (int dist = 1; dist < 4; ++dist) {
            const int nb = 4 - dist;
            for (int e = tid; e < nb * 256; e += NT) {
                const int J = e >> 8, I = J + dist, rr = (e >> 4) & 15, cc = e & 15;
                float acc = 0.f;
                for (int kk = 16 * J; kk < 16 * I; ++kk)
                    acc = fmaf(Af[(16 * I + rr) * 65 + kk], Tf[kk * 65 + 16 * J + cc], acc);
                Xf[J * 272 + rr * 17 + cc] = acc;
            }
            __syncthreads();
            for (int e = tid; e < nb * 256; e += NT) {
                const int J = e >> 8, I = J + dist, rr = (e >> 4) & 15, cc = e & 15;
                float acc = 0.f;
                for (int s_ = 0; s_ <= rr; ++s_)
                    acc = fmaf(Tf[(16 * I + rr) * 65 + 16 * I + s_], Xf[J * 272 + s_ * 17 + cc], acc);
                Tf[(16 * I + rr) * 65 + 16 * J + cc] = -acc;
            }
            __syncthreads();
        }
        // Tb = Tm diag(beta) -> bf16, K-major [r][i].
        {
            const int r = tid >> 2, qq = tid & 3;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float m8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = qq * 16 + hh * 8 + u;
                    m8[u] = Tf[r * 65 + i] * sbeta[i];
                }
                *reinterpret_cast<uint4*>(base + OFF_TB + sw128_off(r, qq * 2 + hh)) =
                    make_uint4(pack_bf16x2(m8[0], m8[1]), pack_bf16x2(m8[2], m8[3]),
                               pack_bf16x2(m8[4], m8[5]), pack_bf16x2(m8[6], m8[7]));
            }
        }
        publish();

        // ---------------- U^T = V^T Tb^T and Wm^T = Ktil^T Tb^T -------------------
        if (tid == 0) {
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t bdesc = sdesc_sw128(sb + OFF_TB + ks * 32, 16, 1024);
                mma_bf16_ss(tbase + COL_E, sdesc_sw128(sb + OFF_V + ks * 2048, 8192, 1024), bdesc, ID_128x64_MK, ks > 0);
                mma_bf16_ss(tbase + COL_W, sdesc_sw128(sb + OFF_KQ + ks * 2048, 16384, 1024), bdesc, ID_128x64_MK, ks > 0);
            }
        }
        if (!commit_and_wait()) { failed = true; break; }

        // Wm^T -> bf16 MN-major tile (row = dk, 64 tokens per row).
        {
            float vals[32];
            tmem_ld16(tq + COL_W + half * 32, *reinterpret_cast<float(*)[16]>(vals));
            tmem_ld16(tq + COL_W + half * 32 + 16, *reinterpret_cast<float(*)[16]>(vals + 16));
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const float* m8 = vals + cc * 8;
                *reinterpret_cast<uint4*>(base + OFF_W + sw128_off(row, half * 4 + cc)) =
                    make_uint4(pack_bf16x2(m8[0], m8[1]), pack_bf16x2(m8[2], m8[3]),
                               pack_bf16x2(m8[4], m8[5]), pack_bf16x2(m8[6], m8[7]));
            }
        }
        publish();

        // ---------------- E^T = U^T - Stil Wm^T ;  O^T = Stil Qtil^T ---------------
        if (tid == 0) {
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kb = ks >> 2, kin = (ks & 3) * 32;
                const uint64_t adesc = sdesc_sw128(sb + OFF_S + kb * 16384 + kin, 16, 1024);
                mma_bf16_ss(tbase + COL_E, adesc, sdesc_sw128(sb + OFF_W + ks * 2048, 8192, 1024), ID_128x64_KMneg, 1);
                mma_bf16_ss(tbase + COL_O, adesc, sdesc_sw128(sb + OFF_KQ + kb * 16384 + 8192 + kin, 16, 1024),
                            ID_128x64_KK, ks > 0);
            }
        }
        if (!commit_and_wait()) { failed = true; break; }

        // E^T -> bf16 K-major tile (row = dv, 64 tokens per row).
        {
            float vals[32];
            tmem_ld16(tq + COL_E + half * 32, *reinterpret_cast<float(*)[16]>(vals));
            tmem_ld16(tq + COL_E + half * 32 + 16, *reinterpret_cast<float(*)[16]>(vals + 16));
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const float* m8 = vals + cc * 8;
                *reinterpret_cast<uint4*>(base + OFF_E + sw128_off(row, half * 4 + cc)) =
                    make_uint4(pack_bf16x2(m8[0], m8[1]), pack_bf16x2(m8[2], m8[3]),
                               pack_bf16x2(m8[4], m8[5]), pack_bf16x2(m8[6], m8[7]));
            }
        }
        publish();

        // ---------------- O^T += E^T Pm^T ;  S_acc += E^T Khat ----------------------
        if (tid == 0) {
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t adesc = sdesc_sw128(sb + OFF_E + ks * 32, 16, 1024);
                mma_bf16_ss(tbase + COL_O, adesc, sdesc_sw128(sb + OFF_PM + ks * 32, 16, 1024), ID_128x64_KK, 1);
                mma_bf16_ss(tbase + COL_S, adesc, sdesc_sw128(sb + OFF_KH + ks * 2048, 8192, 1024), ID_128x128_KM, 1);
            }
        }
        if (!commit_and_wait()) { failed = true; break; }

        // ---------------- epilogue: o, and S <- S_acc (P_m^{-1} P_C) ---------------
        {
            const int j = row;
            float vals[32];
            tmem_ld16(tq + COL_O + half * 32, *reinterpret_cast<float(*)[16]>(vals));
            tmem_ld16(tq + COL_O + half * 32 + 16, *reinterpret_cast<float(*)[16]>(vals + 16));
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int r = half * 32 + u;
                if (r < Lc) st_from_f32(o + tok(r) * D + j, vals[u]);
            }
            const bool last = (c == nchunks - 1);
            for (int g = 0; g < 4; ++g) {
                const int col0 = half * 64 + g * 16;
                float s[16];
                tmem_ld16(tq + COL_S + col0, s);
                if (!ROT) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) s[u] *= rho_C[col0 + u];
                } else {
#pragma unroll
                    for (int u = 0; u < 16; u += 2) {
                        const int pr = (col0 + u) >> 1;
                        const float cr = rho_C[pr], ci = rho_C[128 + pr];
                        const float xr = s[u], xi = s[u + 1];
                        s[u] = xr * cr - xi * ci;
                        s[u + 1] = xr * ci + xi * cr;
                    }
                }
                if (last) {
                    if (p.S_T) {
                        float4* dst = reinterpret_cast<float4*>(p.S_T + ((size_t)bh * D + j) * D + col0);
#pragma unroll
                        for (int u4 = 0; u4 < 4; ++u4)
                            dst[u4] = make_float4(s[4 * u4], s[4 * u4 + 1], s[4 * u4 + 2], s[4 * u4 + 3]);
                    }
                } else {
                    tmem_st16(tq + COL_S + col0, s);
                }
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (nchunks == 0 && p.S_T) {
        for (int e = tid; e < D * D; e += NT)
            p.S_T[(size_t)bh * D * D + e] = p.S0 ? p.S0[(size_t)bh * D * D + e] : 0.f;
    }
    if (tid == 0) {
        unsigned bits = 0;
        if (*abort_flag) bits |= STATUS_TIMEOUT;
        if (*range_flag) bits |= STATUS_RANGE;
        if (bits) atomicOr(&g_device_status, bits);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

}  // namespace tcf
}  // namespace gdr
