// Small device helpers shared by the library's kernels (element conversion).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Four consecutive elements starting at p (p aligned to 4 elements), widened.
__device__ __forceinline__ float4 load4(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}

// Optional input prologue (gdn_flag_t bits of the _ex entry points): q and k
// divided by sqrt(|x|^2 + kNormEps) per token and head; gates given as logits,
// log alpha = -softplus(x), beta = sigmoid(y).
constexpr unsigned kFlagL2Norm = 1u, kFlagGateLogits = 2u;
constexpr float kNormEps = 1e-6f;

// -softplus(x) = -(max(x, 0) + log(1 + e^-|x|)): no overflow on either side.
__device__ __forceinline__ float neg_softplus(float x) {
    return -(fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))));
}
// 1 / (1 + e^-y); saturates to 0 or 1 without producing NaN.
__device__ __forceinline__ float sigmoid(float y) { return 1.f / (1.f + expf(-y)); }

// The gate pair of one token and head as the kernels use it: (log alpha, beta).
__device__ __forceinline__ float2 gate_pair(float la, float be, unsigned flags) {
    return (flags & kFlagGateLogits) ? make_float2(neg_softplus(la), sigmoid(be))
                                     : make_float2(la, be);
}

}  // namespace gdn
