// gdn_common.cuh -- small device helpers shared by the Gated DeltaNet kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace gdn {

constexpr int kDk = 128;             // key dimension (columns i of M[j][i])
constexpr int kDv = 128;             // value dimension (rows j of M[j][i])
constexpr int kConvK = 4;            // causal conv kernel length
constexpr unsigned kFull = 0xffffffffu;
// 1 / sqrt(128), the output scale of step 5, rounded to float.
constexpr float kOutScale = 0.08838834764831845f;

// Streaming 16-byte load/store of state rows: each row is touched once per
// token, so the lines are marked evict-first in L1 and L2.
__device__ __forceinline__ float4 ld_stream(const float* p) {
    return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream(float* p, float4 v) {
    __stcs(reinterpret_cast<float4*>(p), v);
}
// Read-only 16-byte load through the non-coherent path (q, k, v rows that
// many warps share).
__device__ __forceinline__ float4 ld_ro4(const float* p) {
    return __ldg(reinterpret_cast<const float4*>(p));
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, a.x * b.x)));
}

// Sum over the 32 lanes of a warp; every lane receives the total.
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
    return x;
}

// Sum over aligned groups of W lanes (W a power of two <= 32).
template <int W>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int off = W / 2; off > 0; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
    return x;
}

__device__ __forceinline__ float sigmoidf_acc(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float siluf_acc(float x) { return x / (1.0f + expf(-x)); }
// softplus(x) = ln(1 + e^x) = max(x, 0) + ln(1 + e^-|x|)
__device__ __forceinline__ float softplusf_acc(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

}  // namespace gdn
