// gdn_forward_batch.cu -- the recurrent layer over T positions of B sequences
// with dense projections.
//
// Page "Module linear_core", entry "gdn_forward_batch": the qkv/z/a/b and
// out_proj projections are matrix-matrix products over the batch, and the
// recurrence runs sequentially over positions, elementwise as the
// one-position path; stages from "Red Lite dev15e -- complete recurrent
// DeltaNet layer composition" (opening list) and "Red Lite dev15a --
// DeltaNet projection field validation" ("Validation boundary").
//
// Pipeline (every stage a kernel of this library, on the caller's stream):
//   1. mixed = hidden . W_qkv^T, z = hidden . W_z^T, ba = hidden . W_ba^T
//      (tcgen05 GEMMs, bf16 in, fp32 out, into the workspace);
//   2. conv: the positions in parallel tiles, in place after a halo pass that
//      saves the K-1 raw inputs before each tile; mixed becomes SiLU(conv) and
//      the ring ends as the last K-1 raw inputs;
//   3. qk_norm_gates: per position, L2-normalise each q and k head in place
//      and form beta = sigmoid(b), gate = -exp(A_log) softplus(a + dt_bias);
//   4. the sequential prefill recurrence, reading q, k, v straight out of the
//      conv buffer (row stride C), writing o [B][T][Hv][dv];
//   5. tail: per (position, value head) gated RMSNorm in double, rounded to
//      bf16 (the output projection's input type);
//   6. out = y . W_out^T (tcgen05 GEMM).
#include <cuda_bf16.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

// 2. causal depthwise conv over positions, SiLU, in place, with the ring.
//    Every output needs only the K-1 raw inputs before it, so the positions
//    run in parallel in tiles of kConvTile; to convolve in place, the K-1 raw
//    inputs before each tile are copied out first (conv_halo_kernel), then
//    every (sequence, tile, channel) thread convolves its tile
//    (conv_tile_kernel). Tile 0 reads its K-1 inputs from the old ring, so
//    the halo holds n_tiles slots per sequence: slot j - 1 for tile j >= 1,
//    and slot n_tiles - 1 (the inputs before position T) is also the ring the
//    call leaves behind, which the tile-0 thread of each channel writes after
//    it has read the old ring -- the only thread that reads it.
constexpr int kConvTile = 32;

// Both conv kernels move four adjacent channels per thread (16-byte
// accesses; C is a multiple of 4), so that the pass is bound by HBM rather
// than by load/store instruction issue.
__device__ __forceinline__ float conv_tap(float4 w, float w0, float w1, float w2, float x) {
    return fmaf(w.w, x, fmaf(w.z, w2, fmaf(w.y, w1, w.x * w0)));
}

__global__ void __launch_bounds__(256)
conv_halo_kernel(const float* __restrict__ act, const float* __restrict__ ring,
                 float* __restrict__ halo, int64_t T, int64_t C, int n_tiles) {
    const int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (c >= C) return;
    const int j = blockIdx.y + 1;                        // tiles 1 .. n_tiles (n_tiles: the ring)
    const int64_t b = blockIdx.z;
    const int64_t end = j < n_tiles ? static_cast<int64_t>(j) * kConvTile : T;
    float* dst = halo + ((b * n_tiles + (j - 1)) * (kConvK - 1)) * C + c;
#pragma unroll
    for (int i = 0; i < kConvK - 1; ++i) {
        const int64_t t = end - (kConvK - 1) + i;        // raw input position (slot i)
        const float* src = t >= 0 ? act + (b * T + t) * C + c
                                  : ring + (b * (kConvK - 1) + (kConvK - 1 + t)) * C + c;
        *reinterpret_cast<float4*>(dst + i * C) = *reinterpret_cast<const float4*>(src);
    }
}

__global__ void __launch_bounds__(256)
conv_tile_kernel(float* __restrict__ act, float* __restrict__ ring,
                 const float* __restrict__ halo, const float* __restrict__ conv_w, int64_t T,
                 int64_t C, int n_tiles) {
    const int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (c >= C) return;
    const int j = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int64_t t0 = static_cast<int64_t>(j) * kConvTile;
    const int n = (T - t0) < kConvTile ? static_cast<int>(T - t0) : kConvTile;
    float4 w[4];                                         // taps of channels c .. c + 3
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = ld_ro4(conv_w + (c + q) * kConvK);
    const float* hs = j == 0 ? ring + b * (kConvK - 1) * C + c
                             : halo + ((b * n_tiles + (j - 1)) * (kConvK - 1)) * C + c;
    // raw inputs, oldest first, of the four channels
    float4 w0 = *reinterpret_cast<const float4*>(hs);
    float4 w1 = *reinterpret_cast<const float4*>(hs + C);
    float4 w2 = *reinterpret_cast<const float4*>(hs + 2 * C);
    float* col = act + (b * T + t0) * C + c;
    constexpr int kSub = 8;                              // positions loaded together
#pragma unroll 1
    for (int i0 = 0; i0 < n; i0 += kSub) {
        float4 xs[kSub];
#pragma unroll
        for (int i = 0; i < kSub; ++i)
            if (i0 + i < n) xs[i] = *reinterpret_cast<const float4*>(col + static_cast<int64_t>(i0 + i) * C);
#pragma unroll
        for (int i = 0; i < kSub; ++i) {
            if (i0 + i < n) {
                const float4 x = xs[i];
                float4 y;
                y.x = siluf_acc(conv_tap(w[0], w0.x, w1.x, w2.x, x.x));
                y.y = siluf_acc(conv_tap(w[1], w0.y, w1.y, w2.y, x.y));
                y.z = siluf_acc(conv_tap(w[2], w0.z, w1.z, w2.z, x.z));
                y.w = siluf_acc(conv_tap(w[3], w0.w, w1.w, w2.w, x.w));
                *reinterpret_cast<float4*>(col + static_cast<int64_t>(i0 + i) * C) = y;
                w0 = w1;
                w1 = w2;
                w2 = x;
            }
        }
    }
    if (j == 0) {            // the ring after the call (this thread read the old one above)
        const float* nr = halo + ((b * n_tiles + (n_tiles - 1)) * (kConvK - 1)) * C + c;
        float* rg = ring + b * (kConvK - 1) * C + c;
        const float4 r0 = *reinterpret_cast<const float4*>(nr);
        const float4 r1 = *reinterpret_cast<const float4*>(nr + C);
        const float4 r2 = *reinterpret_cast<const float4*>(nr + 2 * C);
        *reinterpret_cast<float4*>(rg) = r0;
        *reinterpret_cast<float4*>(rg + C) = r1;
        *reinterpret_cast<float4*>(rg + 2 * C) = r2;
    }
}

// 3. per position: L2-normalise the 2 Hk q/k heads (one warp each, in turn)
//    and compute the Hv decay gates and write strengths.
__global__ void __launch_bounds__(256)
qk_norm_gates_kernel(float* __restrict__ act, const float* __restrict__ ba,
                     const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                     float* __restrict__ beta, float* __restrict__ gate, int64_t C, int Hk,
                     int Hv, float l2_eps) {
    const int64_t bt = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_warps = blockDim.x >> 5;
    float* row = act + bt * C;
    for (int vec = warp; vec < 2 * Hk; vec += n_warps) {
        float4* p = reinterpret_cast<float4*>(row + static_cast<int64_t>(vec) * kDk) + lane;
        float4 x = *p;
        float ss = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, x.w * x.w)));
        ss = warp_sum(ss);
        const float inv = 1.0f / fmaxf(sqrtf(ss), l2_eps);
        x.x *= inv; x.y *= inv; x.z *= inv; x.w *= inv;
        *p = x;
    }
    for (int h = threadIdx.x; h < Hv; h += blockDim.x) {
        const float bv = ba[bt * 2 * Hv + h];
        const float av = ba[bt * 2 * Hv + Hv + h];
        beta[bt * Hv + h] = sigmoidf_acc(bv);
        gate[bt * Hv + h] = -expf(A_log[h]) * softplusf_acc(av + dt_bias[h]);
    }
}

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
    return x;
}

// 5. gated RMSNorm per (position, value head); y in bf16. The sum of squares
//    and 1/rms are taken in double, the gate in fp32: y is rounded to bf16
//    (relative step 2^-8) right after, far coarser than fp32's error.
__global__ void __launch_bounds__(256)
tail_bf16_kernel(const float* __restrict__ o, const float* __restrict__ z,
                 const float* __restrict__ norm_w, __nv_bfloat16* __restrict__ y, int64_t rows,
                 float norm_eps) {
    const int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;                                   // r = (b t) * Hv + h
    const int lane = threadIdx.x & 31;
    const float4 ov = ld_ro4(o + r * kDv + lane * 4);
    const float4 zv = ld_ro4(z + r * kDv + lane * 4);
    const float4 wv = ld_ro4(norm_w + lane * 4);
    const float o4[4] = {ov.x, ov.y, ov.z, ov.w};
    const float z4[4] = {zv.x, zv.y, zv.z, zv.w};
    const float w4[4] = {wv.x, wv.y, wv.z, wv.w};
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) ss = fma(static_cast<double>(o4[i]), static_cast<double>(o4[i]), ss);
    ss = warp_sum_d(ss);
    const float inv_rms =
        static_cast<float>(1.0 / sqrt(ss / static_cast<double>(kDv) + static_cast<double>(norm_eps)));
    __nv_bfloat16 out4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        out4[i] = __float2bfloat16_rn(o4[i] * inv_rms * w4[i] * siluf_acc(z4[i]));
    *reinterpret_cast<uint2*>(y + r * kDv + lane * 4) = *reinterpret_cast<const uint2*>(out4);
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

ForwardBatchLayout forward_batch_layout(int64_t B, int64_t T, int Hk, int Hv) {
    const int64_t BT = B * T;
    const int64_t C = static_cast<int64_t>(2 * Hk) * kDk + static_cast<int64_t>(Hv) * kDv;
    const int64_t HD = static_cast<int64_t>(Hv) * kDv;
    ForwardBatchLayout L;
    size_t off = 0;
    L.act = off;   off = align256(off + BT * C * 4);
    L.z = off;     off = align256(off + BT * HD * 4);
    L.ba = off;    off = align256(off + BT * 2 * Hv * 4);
    L.beta = off;  off = align256(off + BT * Hv * 4);
    L.gate = off;  off = align256(off + BT * Hv * 4);
    L.o = off;     off = align256(off + BT * HD * 4);
    L.y = off;     off = align256(off + BT * HD * 2);
    const int64_t n_tiles = (T + kConvTile - 1) / kConvTile;
    L.halo = off;  off = align256(off + B * n_tiles * (kConvK - 1) * C * 4);
    L.total = off;
    return L;
}

cudaError_t launch_forward_batch(const ForwardBatchArgs& a, cudaStream_t stream) {
    const int64_t BT = a.B * a.T;
    if (BT == 0) return cudaSuccess;
    const int64_t C = static_cast<int64_t>(2 * a.Hk) * kDk + static_cast<int64_t>(a.Hv) * kDv;
    const int64_t HD = static_cast<int64_t>(a.Hv) * kDv;
    const ForwardBatchLayout L = forward_batch_layout(a.B, a.T, a.Hk, a.Hv);
    char* ws = static_cast<char*>(a.workspace);
    float* act = reinterpret_cast<float*>(ws + L.act);
    float* z = reinterpret_cast<float*>(ws + L.z);
    float* ba = reinterpret_cast<float*>(ws + L.ba);
    float* beta = reinterpret_cast<float*>(ws + L.beta);
    float* gate = reinterpret_cast<float*>(ws + L.gate);
    float* o = reinterpret_cast<float*>(ws + L.o);
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(ws + L.y);
    float* halo = reinterpret_cast<float*>(ws + L.halo);

    // 1. input projections
    cudaError_t err;
    if ((err = launch_linear_bf16(LinearArgs{a.hidden, a.w_qkv, act, BT, C, a.D, a.status}, stream)))
        return err;
    if ((err = launch_linear_bf16(LinearArgs{a.hidden, a.w_z, z, BT, HD, a.D, a.status}, stream)))
        return err;
    if ((err = launch_linear_bf16(LinearArgs{a.hidden, a.w_ba, ba, BT, 2 * a.Hv, a.D, a.status},
                                  stream)))
        return err;
    // 2. conv over positions with the ring, SiLU (halo pass, then in place)
    {
        const int n_tiles = static_cast<int>((a.T + kConvTile - 1) / kConvTile);
        const unsigned cblocks = static_cast<unsigned>((C / 4 + 255) / 256);   // 4 channels a thread
        conv_halo_kernel<<<dim3(cblocks, static_cast<unsigned>(n_tiles),
                                static_cast<unsigned>(a.B)), 256, 0, stream>>>(
            act, a.conv_ring, halo, a.T, C, n_tiles);
        if ((err = cudaGetLastError())) return err;
        conv_tile_kernel<<<dim3(cblocks, static_cast<unsigned>(n_tiles),
                                static_cast<unsigned>(a.B)), 256, 0, stream>>>(
            act, a.conv_ring, halo, a.conv_w, a.T, C, n_tiles);
        if ((err = cudaGetLastError())) return err;
    }
    // 3. q/k L2 norm, beta and gate
    qk_norm_gates_kernel<<<static_cast<unsigned>(BT), 256, 0, stream>>>(
        act, ba, a.A_log, a.dt_bias, beta, gate, C, a.Hk, a.Hv, a.l2_eps);
    if ((err = cudaGetLastError())) return err;
    // 4. the sequential recurrence, reading q, k, v from the conv rows
    {
        PrefillArgs p{a.state, act, act + static_cast<int64_t>(a.Hk) * kDk,
                      act + static_cast<int64_t>(2 * a.Hk) * kDk, beta, gate, o, a.B, a.T, a.Hk,
                      a.Hv, C, C, a.Hv};
        p.status = a.status;
        if ((err = launch_prefill(p, stream))) return err;
    }
    // 5. gated RMSNorm tail -> bf16
    {
        const int64_t rows = BT * a.Hv;
        tail_bf16_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
            o, z, a.norm_w, y, rows, a.norm_eps);
        if ((err = cudaGetLastError())) return err;
    }
    // 6. output projection
    return launch_linear_bf16(LinearArgs{y, a.w_out, a.out, BT, a.D, HD, a.status}, stream);
}

}  // namespace gdn
