// Device helpers shared by the kernels: element conversion and small reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace m3 {

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The step scalars of one token from what the caller passed (the fused scalar prologue):
// with the flag, dt holds the raw projection and the step is softplus(raw + bias), and lam
// holds u and the trapezoid weight is sigmoid(u). Calls only cover real tokens: positions past
// the end of a sequence keep their zeros. kRaw = false (no flag set) compiles to the identity,
// so kernels instantiated for plain scalars carry none of this code.
template <bool kRaw = true>
__device__ __forceinline__ float step_dt(float raw, float bias, uint32_t flags) {
    if constexpr (!kRaw) {
        return raw;
    } else {
        if (!(flags & 1u)) return raw;
        // softplus(v) = max(v, 0) + log(1 + e^{-|v|}): the exponential never overflows and the
        // logarithm's argument stays in (1, 2]. Below v ~ -16 the log term rounds to zero (an
        // absolute error of e^v < 1e-7 in a step that is then negligible).
        const float v = raw + bias;
        return fmaxf(v, 0.f) + __logf(1.f + __expf(-fabsf(v)));
    }
}
template <bool kRaw = true>
__device__ __forceinline__ float step_lam(float raw, uint32_t flags) {
    if constexpr (!kRaw) return raw;
    else return (flags & 2u) ? __frcp_rn(1.f + __expf(-raw)) : raw;   // e^{-raw} = inf gives 0
}

// The zero-order-hold input weight (e^{dt A} - 1) / A ("Mamba-3：推理优先的状态空间模型",
// Sec. 1.2), dt in the limit A -> 0; with M3_DISC_ZOH it replaces gamma and beta is 0.
__device__ __forceinline__ float zoh_gamma(float dt, float A) {
    const float x = dt * A;
    return x != 0.f ? expm1f(x) / A : dt;
}

// x reduced by a whole number of turns into [-pi, pi]: Cody-Waite reduction with 2*pi split
// into an exactly representable head and a tail (Cody & Waite, "Software Manual for the
// Elementary Functions", 1980). Absolute error ~1e-6 for |x| < 1e4.
__device__ __forceinline__ float reduce_2pi(float x) {
    constexpr float kInv2Pi = 0.15915494309189535f;
    constexpr float k2PiHi = 6.28125f;                  // exactly representable head of 2*pi
    constexpr float k2PiLo = 1.9353071795864769e-3f;    // 2*pi - 6.28125
    const float k = rintf(x * kInv2Pi);
    return fmaf(-k, k2PiLo, fmaf(-k, k2PiHi, x));
}

// Inclusive prefix sum across the 32 lanes of a warp.
__device__ __forceinline__ float warp_inclusive_scan(float v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

}  // namespace m3
