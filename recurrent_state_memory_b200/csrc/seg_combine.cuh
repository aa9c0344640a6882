// seg_combine.cuh -- the sequence-parallel forward's combine step: an affine scan over segments
// and the output correction.
//
// "Semidirect Fourier Delta Attention" page, "Main contributions": the state at the end of a
// chunk (here: of a segment of many chunks) is an exact affine function of the state at its
// start, S_end = S_start A + B, where B is the end state reached from the zero state and A the
// one reached from the identity with zero values.  Every segment runs independently twice (the
// split kernel: from zero for o0 and B, from the identity with v = 0 for y_t = A_{start->t} q_t
// and A); then, per head, with St_s the true state at the start of segment s:
//   St_1 = B_0 (segment 0 runs from the real initial state),  St_{s+1} = St_s A_s + B_s,
//   S_T = St_nseg,   o_t = o0_t + St_s y_t   (t in segment s >= 1).
// Because the gates act on the key axis only, the value rows of S are independent, so the scan
// runs in blocks of rows.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdr {
namespace seg {

constexpr int D = 128;
constexpr int RB = 16;          // state rows per scan CTA
constexpr int SCAN_NT = 256;
constexpr uint32_t SCAN_SMEM = (D * D + RB * D) * 4;   // A_s and this CTA's rows of St
constexpr int TOK = 64;         // tokens per correction tile (a segment is a whole number of tiles)
constexpr int CORR_NT = 128;
constexpr uint32_t CORR_A = 0, CORR_B = 65536, CORR_BAR = CORR_B + 32768;
constexpr uint32_t CORR_SMEM = CORR_BAR + 64 + 1024;   // + base alignment

struct ScanParams {
    int nheads, nseg;
    const float* Bz;      // [nheads][nseg][D][D]: segment end states from zero (segment 0: from S0)
    const float* A;       // [nheads][nseg - 1][D][D]: transitions of segments 1 .. nseg-1
    float* St;            // [nheads][nseg - 1][D * D]: start states of segments 1.., tf32 in the
                          //   correction's A-operand layout (4 kblocks x 128 rows x 128 B, swizzled)
    float* S_T;           // [nheads][D][D] final states, or nullptr
};

// Byte offset of element (r, m) of a 128 x 128 fp32 matrix in the K-major, 128-byte swizzled
// tf32 operand layout (kblocks of 32 columns, rows of 128 bytes).
__device__ __forceinline__ uint32_t tf32_kmajor_off(uint32_t r, uint32_t m) {
    return (m >> 5) * 16384u + tc::sw128_off(r, (m & 31u) >> 2) + (m & 3u) * 4u;
}
// fp32 -> tf32 (round to nearest, ties away from zero), kept in an fp32 container.
__device__ __forceinline__ float round_tf32(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// grid (nheads, D / RB), SCAN_NT threads, SCAN_SMEM dynamic shared memory.
// Thread t updates row r0 + t / 16, columns 8 (t % 16) .. 8 (t % 16) + 7, in fp32.
__global__ void __launch_bounds__(SCAN_NT) seg_scan_kernel(ScanParams sp) {
    extern __shared__ __align__(16) float sm[];
    float* sA = sm;                  // [D][D] A_s
    float* sS = sm + D * D;          // [RB][D] rows r0 .. r0 + RB - 1 of St_s
    const int h = blockIdx.x, r0 = blockIdx.y * RB;
    const int t = threadIdx.x, rr = t >> 4, cb = (t & 15) * 8;
    const size_t DD = (size_t)D * D;
    const size_t ns1 = (size_t)sp.nseg - 1;
    for (int e = t; e < RB * D; e += SCAN_NT)
        sS[e] = sp.Bz[(size_t)h * sp.nseg * DD + (size_t)(r0 + e / D) * D + e % D];
    __syncthreads();
    for (int s = 1; s < sp.nseg; ++s) {
        uint8_t* dst = reinterpret_cast<uint8_t*>(sp.St + ((size_t)h * ns1 + (s - 1)) * DD);
        for (int e = t; e < RB * D; e += SCAN_NT)
            *reinterpret_cast<float*>(dst + tf32_kmajor_off((uint32_t)(r0 + e / D), (uint32_t)(e % D))) = round_tf32(sS[e]);
        const float4* a4 = reinterpret_cast<const float4*>(sp.A + ((size_t)h * ns1 + (s - 1)) * DD);
        for (int e = t; e < D * D / 4; e += SCAN_NT) reinterpret_cast<float4*>(sA)[e] = a4[e];
        __syncthreads();
        float acc[8];
        const float* bz = sp.Bz + ((size_t)h * sp.nseg + s) * DD + (size_t)(r0 + rr) * D + cb;
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = bz[u];
#pragma unroll 4
        for (int m = 0; m < D; ++m) {
            const float sv = sS[rr * D + m];
            const float4 x0 = *reinterpret_cast<const float4*>(sA + m * D + cb);
            const float4 x1 = *reinterpret_cast<const float4*>(sA + m * D + cb + 4);
            acc[0] = fmaf(sv, x0.x, acc[0]); acc[1] = fmaf(sv, x0.y, acc[1]);
            acc[2] = fmaf(sv, x0.z, acc[2]); acc[3] = fmaf(sv, x0.w, acc[3]);
            acc[4] = fmaf(sv, x1.x, acc[4]); acc[5] = fmaf(sv, x1.y, acc[5]);
            acc[6] = fmaf(sv, x1.z, acc[6]); acc[7] = fmaf(sv, x1.w, acc[7]);
        }
        __syncthreads();             // every thread has read St_s and A_s
#pragma unroll
        for (int u = 0; u < 8; ++u) sS[rr * D + cb + u] = acc[u];
        __syncthreads();
    }
    if (sp.S_T && GDR_INB(h < sp.nheads && r0 + RB <= D, 201)) {
        for (int e = t; e < RB * D; e += SCAN_NT) sp.S_T[(size_t)h * DD + (size_t)(r0 + e / D) * D + e % D] = sS[e];
    }
}

struct CorrParams {
    int B, H, T, nseg, seg_len, head0;
    const float* St;     // from seg_scan_kernel
    void* o;             // [B, T, H, D] in the output type: o0 in, o out
    float* chunk_mean;   // [B, ceil(T/64), H, D] means of o0 in, of o out; or nullptr
};

// In-register transpose of an 8x8 block held by 8 consecutive lanes (lane j enters with row j
// and leaves with column j).
__device__ __forceinline__ void transpose8x8(float (&v)[8], int j) {
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

// One CTA per (head, segment >= 1, 64-token tile): O^T (dv x tokens) = St_s (dv x dk) Y^T
// (tf32, 128 x 64 x 128, fp32 in TMEM), then o += O for the tile's tokens inside T.
// ymap: y [B, T, H, D] fp32 with boxes {32, 1, 64, 1} and the 128-byte swizzle.
template <typename OT>
__global__ void __launch_bounds__(CORR_NT, 1) seg_correct_kernel(CorrParams cp, const __grid_constant__ CUtensorMap ymap,
                                                               unsigned long long wait_limit_ns) {
    using namespace tc;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sb = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (sb - raw_u32);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + CORR_BAR);     // [0] loads, [1] MMA
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + CORR_BAR + 16);
    int* fail = reinterpret_cast<int*>(base + CORR_BAR + 20);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles = cp.seg_len / TOK, ns1 = cp.nseg - 1;
    const int h = blockIdx.x / (ns1 * tiles);
    const int rem = blockIdx.x - h * ns1 * tiles;
    const int s = 1 + rem / tiles, tile = rem % tiles;
    const int gx = cp.head0 + h;
    const int t0 = s * cp.seg_len + tile * TOK;
    if (warp == 0) {
        tmem_alloc(tmem_slot, 64);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bars, 1);
        mbar_init(bars + 1, 1);
        fence_mbar_init();
        *fail = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    if (t0 < cp.T) {
        if (tid == 0) {
            const uint8_t* src = reinterpret_cast<const uint8_t*>(cp.St + ((size_t)h * ns1 + (s - 1)) * D * D);
            mbar_arrive_expect_tx(bars, 65536u + 32768u);
            for (uint32_t off = 0; off < 65536u; off += 16384u) bulk_g2s(sb + CORR_A + off, src + off, 16384u, bars);
            for (int kb = 0; kb < 4; ++kb)
                tma_load_4d(sb + CORR_B + kb * 8192u, &ymap, kb * 32, gx % cp.H, t0, gx / cp.H, bars);
            bool ok = mbar_wait_bounded(bars, 0u, wait_limit_ns);
            if (ok) {
                tc_fence_after();
                const uint32_t idesc = idesc_tf32(128, TOK);
#pragma unroll
                for (int ks = 0; ks < 16; ++ks) {
                    const uint32_t kb = ks >> 2, kin = (ks & 3) * 32;
                    mma_tf32_ss(tbase, sdesc_sw128(sb + CORR_A + kb * 16384 + kin, 16, 1024),
                                sdesc_sw128(sb + CORR_B + kb * 8192 + kin, 16, 1024), idesc, ks > 0);
                }
                mma_commit(bars + 1);
                ok = mbar_wait_bounded(bars + 1, 0u, wait_limit_ns);
            }
            if (!ok) {
                *fail = 1;
                atomicOr(&g_device_status, 1u);
            }
        }
        __syncthreads();
        tc_fence_after();
        if (*fail == 0) {
            // lane = value row of this warp's quadrant, columns = the tile's tokens
            const int j8 = lane & 7, grp = lane >> 3;
            const uint32_t tq = tbase + ((uint32_t)(warp * 32) << 16);
            OT* o = static_cast<OT*>(cp.o);
            const size_t tstride = (size_t)cp.H * D;
            OT* obase = o + (((size_t)(gx / cp.H) * cp.T + t0) * cp.H + gx % cp.H) * D + warp * 32 + grp * 8;
            const int Lt = min(TOK, cp.T - t0);      // tokens of this tile (one chunk) inside T
            float csum = 0.f;                         // this value row's correction summed over them
#pragma unroll 1
            for (int g = 0; g < 2; ++g) {
                float vals[32];
                tmem_ld32(tq + g * 32, vals);
                if (cp.chunk_mean) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) csum += (g * 32 + u < Lt) ? vals[u] : 0.f;
                }
#pragma unroll
                for (int blk8 = 0; blk8 < 4; ++blk8) {
                    float v8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v8[e] = vals[blk8 * 8 + e];
                    transpose8x8(v8, j8);
                    const int r = g * 32 + blk8 * 8 + j8;
                    if (t0 + r < cp.T && GDR_INB(gx < cp.B * cp.H, 204)) {
                        OT* dst = obase + (size_t)r * tstride;
                        if constexpr (sizeof(OT) == 2) {
                            const uint4 cur = *reinterpret_cast<const uint4*>(dst);
                            const uint32_t cw[4] = {cur.x, cur.y, cur.z, cur.w};
                            float m8[8];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                m8[2 * e] = v8[2 * e] + __uint_as_float(cw[e] << 16);
                                m8[2 * e + 1] = v8[2 * e + 1] + __uint_as_float(cw[e] & 0xFFFF0000u);
                            }
                            *reinterpret_cast<uint4*>(dst) =
                                make_uint4(pack_bf16x2(m8[0], m8[1]), pack_bf16x2(m8[2], m8[3]),
                                           pack_bf16x2(m8[4], m8[5]), pack_bf16x2(m8[6], m8[7]));
                        } else {
                            float4* d4 = reinterpret_cast<float4*>(dst);
                            const float4 a = d4[0], b = d4[1];
                            d4[0] = make_float4(a.x + v8[0], a.y + v8[1], a.z + v8[2], a.w + v8[3]);
                            d4[1] = make_float4(b.x + v8[4], b.y + v8[5], b.z + v8[6], b.w + v8[7]);
                        }
                    }
                }
            }
            if (cp.chunk_mean) {     // the mean is linear: mean(o) = mean(o0) + mean(correction)
                const int nct = (cp.T + TOK - 1) / TOK;
                float* cm = cp.chunk_mean + (((size_t)(gx / cp.H) * nct + t0 / TOK) * cp.H + gx % cp.H) * D + warp * 32 + lane;
                *cm += csum / (float)Lt;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 64);
    }
}

}  // namespace seg
}  // namespace gdr
