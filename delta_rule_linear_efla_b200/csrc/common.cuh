// common.cuh -- small device helpers shared by the EFLA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace efla {

// Element access for the two supported input types.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// alpha = (1 - exp(-beta*lambda)) / lambda  ("Exact Flow Linear Attention",
// technical summary, Methodology 3), evaluated as -expm1(-x)/lambda with
// x = beta*lambda so that small x keeps full relative precision.  For
// |x| < 2^-40 the first two terms of the series (1 - e^{-x})/x = 1 - x/2 + x^2/6 - ...
// give alpha = beta (1 - x/2) to fp32 precision; this also covers the
// lambda -> 0 limit (alpha -> beta) without a 0/0.
__device__ __forceinline__ float alpha_from(float lambda, float beta) {
    const float x = beta * lambda;
    if (fabsf(x) < 9.094947e-13f)  // 2^-40
        return beta * (1.0f - 0.5f * x);
    return -expm1f(-x) / lambda;
}

// The coefficient under the selected rule: the exact flow above, or the explicit Euler
// step of the same ODE ("Exact Flow Linear Attention", technical summary, Key
// Contributions: the delta rule is that Euler step), whose coefficient is beta itself.
__device__ __forceinline__ float alpha_rule(float lambda, float beta, bool euler) {
    return euler ? beta : alpha_from(lambda, beta);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace efla
