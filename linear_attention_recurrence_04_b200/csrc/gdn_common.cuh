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

// One halving step of warp_sum_many: a lane keeps one half of its 2 HALF
// values (the upper half if its `o` bit is set), adds its partner's copy of
// that half, and sends the other half.
template <int HALF, typename T>
__device__ __forceinline__ void fold_step(T* v, int lane, int o) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < HALF; ++i) {
        const T send = up ? v[i] : v[i + HALF];
        const T keep = up ? v[i + HALF] : v[i];
        v[i] = keep + __shfl_xor_sync(kFull, send, o);
    }
}

// Sums each of the N values v[0..N-1] over aligned groups of W lanes (N and W
// powers of two, N <= W <= 32) with N - 1 + log2(W / N) shuffles instead of
// N log2(W). Lane c of a group (c = lane % W) returns the total of value
// c >> log2(W / N).
template <int N, int W, typename T>
__device__ __forceinline__ T group_sum_many(T (&v)[N], int lane) {
    static_assert(N >= 1 && N <= W && W <= 32 && (N & (N - 1)) == 0 && (W & (W - 1)) == 0,
                  "N and W must be powers of two with N <= W <= 32");
    int o = W / 2;
    if constexpr (N >= 32) { fold_step<16>(v, lane, o); o >>= 1; }
    if constexpr (N >= 16) { fold_step<8>(v, lane, o); o >>= 1; }
    if constexpr (N >= 8) { fold_step<4>(v, lane, o); o >>= 1; }
    if constexpr (N >= 4) { fold_step<2>(v, lane, o); o >>= 1; }
    if constexpr (N >= 2) { fold_step<1>(v, lane, o); o >>= 1; }
    T s = v[0];
    for (; o >= 1; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
    return s;
}

// The same over the whole warp: lane L returns the total of value
// L >> (5 - log2 N).
template <int N, typename T>
__device__ __forceinline__ T warp_sum_many(T (&v)[N], int lane) {
    return group_sum_many<N, 32>(v, lane);
}

// The lane that warp_sum_many<N> leaves value `i`'s total on.
template <int N>
__device__ __forceinline__ int sum_many_lane(int i) {
    return i << (N == 32 ? 0 : N == 16 ? 1 : N == 8 ? 2 : N == 4 ? 3 : N == 2 ? 4 : 5);
}

__device__ __forceinline__ float sigmoidf_acc(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float siluf_acc(float x) { return x / (1.0f + expf(-x)); }
// softplus(x) = ln(1 + e^x) = max(x, 0) + ln(1 + e^-|x|)
__device__ __forceinline__ float softplusf_acc(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

}  // namespace gdn
