// common.cuh -- small device helpers shared by the gdr kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

// Device status word: kernels OR in a bit when a bounded wait gives up (bit 0) or a
// decay factor leaves the range of the factored tensor-core form (bit 1).  Read and
// cleared by gdr_query_device_status.  (All kernels live in one translation unit.)
__device__ unsigned int g_device_status = 0;

// Index checks of the debug build (compiled with -DGDR_BOUNDS_CHECK).  GDR_INB(cond, site)
// guards one global-memory access: when cond fails, the site number goes to g_bounds_site (the
// first failure is kept), bit 2 of the status word is set and the access is skipped.  In the
// default build the macro is the constant true and costs nothing.
constexpr unsigned STATUS_BOUNDS = 4u;
__device__ unsigned int g_bounds_site = 0;
#ifdef GDR_BOUNDS_CHECK
__device__ __forceinline__ bool in_bounds(bool c, unsigned site) {
    if (!c) {
        atomicCAS(&g_bounds_site, 0u, site);
        atomicOr(&g_device_status, STATUS_BOUNDS);
    }
    return c;
}
#define GDR_INB(cond, site) ::gdr::in_bounds((cond), (site))
#else
#define GDR_INB(cond, site) true
#endif

// Element loads/stores with the storage type chosen at compile time.
template <typename T> __device__ __forceinline__ float ld_f32(const T* p);
template <> __device__ __forceinline__ float ld_f32<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

template <typename T> __device__ __forceinline__ void st_from_f32(T* p, float x);
template <> __device__ __forceinline__ void st_from_f32<float>(float* p, float x) { *p = x; }
template <> __device__ __forceinline__ void st_from_f32<__nv_bfloat16>(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
}

// Log-decay of one gate value.  gate_mode 1: g = -softplus(a) = -(max(a,0) + log1p(e^{-|a|})),
// the activation the workloads state; gate_mode 0: the value is g itself.
__device__ __forceinline__ float log_decay(float a, int gate_mode) {
    if (gate_mode == 1) return -(fmaxf(a, 0.f) + log1pf(expf(-fabsf(a))));
    return a;
}

// Multiplicative decay alpha = exp(g) of one gate value, computed without the
// log: for gate_mode 1, exp(-softplus(a)) = 1 / (1 + e^{a}) (a -> +inf gives 0).
__device__ __forceinline__ float decay_factor(float a, int gate_mode) {
    if (gate_mode == 1) return 1.f / (1.f + expf(a));
    return expf(a);
}

// Reduce an angle to [-pi, pi] so that sums of many angles keep full accuracy.
__device__ __forceinline__ float wrap_angle(float x) {
    const float two_pi = 6.283185307179586f;
    return x - two_pi * rintf(x * (1.f / two_pi));
}

}  // namespace gdr
