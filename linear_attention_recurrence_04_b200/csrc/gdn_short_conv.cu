// gdn_short_conv.cu -- the LFM2 short-convolution mixer over T positions of B
// sequences ("Module linear_core", struct "ShortConvWeights" and entries
// "short_conv_forward", "short_conv_forward_batch", "short_conv_pair").
//
// The mixer has no recurrent state: its only state is the causal conv ring,
// the last K-1 gated inputs of every channel. Per position t and channel d:
//   (bg | cg | xv) = W_in h_t            rows [0,D) | [D,2D) | [2D,3D)
//   u_t[d]  = bg[d] * xv[d]              (the gated input the ring keeps)
//   conv[d] = sum_tau conv_w[d][tau] * window[tau],
//             window = (u_{t-K+1} .. u_t), entries before position 0 from the ring
//   y_t[d]  = cg[d] * conv[d]            (rounded to bf16, out_proj's input type)
//   out_t   = W_out y_t
//
// Pipeline (each stage a kernel of this library, on the caller's stream):
//   1. proj = hidden . W_in^T          (tcgen05 GEMM, fp32 out, workspace)
//   2. gate_conv: every (sequence, 32-position tile, channel) in parallel --
//      u is a function of proj alone, so no position waits for another; each
//      thread rebuilds its K-1 halo from proj (or from the ring before
//      position 0) with the same fp32 product, so every tile sees exactly the
//      ring values a position-by-position walk would hold;
//   3. ring_update: per (sequence, channel), the ring after position
//      n_commit - 1 goes to conv_ring and, for the two-position verify, the
//      ring after the last position to scratch_ring (a separate kernel so
//      that no tile of step 2 can read a ring slot that was already replaced;
//      a call of one tile -- decode, verify -- has one thread per channel,
//      which writes the rings itself at the end of step 2);
//   4. out = y . W_out^T              (tcgen05 GEMM).
// Calls of at most 128 rows (B*T) run stages 1-3 as one kernel: the input
// projection split over K in a thread-block cluster, whose epilogue sums the
// partials and does the gate, conv and rings for its 64 channels (the same
// arithmetic as the gate kernel below); stage 4 is split the same way. The
// rows of such calls agree bit for bit with one another, and with larger
// calls to fp32 rounding of the projections' accumulation order. Calls of
// one or two positions whose two splits agree run all four stages as one
// kernel (the split kernel's fused form: a grid-wide barrier on a word of the
// workspace between the conv and the output projection), with the same bits.
// u is rounded to fp32 (the ring's type) before it enters the window; the
// window sum and the output gate run in double, and y is rounded once.
#include <cuda_bf16.h>

#include <cstdlib>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_tc.cuh"

// 1: calls of one or two positions run the whole mixer as one kernel; 0:
// they take the two-kernel path (the same bits).
#ifndef GDN_SHORT_CONV_FUSED
#define GDN_SHORT_CONV_FUSED 1
#endif

namespace gdn {

namespace {

constexpr int kConvTile = 32;            // positions per thread in gate_conv

// kWriteRing (calls of at most kConvTile positions: one tile, so one thread
// per (sequence, channel)): the thread that read the old ring also writes the
// ring after position n_commit - 1 and, for the verify, the ring after the
// last position to scratch_ring; no separate ring pass is needed.
template <int K, bool kWriteRing>
__global__ void __launch_bounds__(256)
short_conv_gate_kernel(const float* __restrict__ proj, float* ring, float* scratch_ring,
                       const float* __restrict__ conv_w, __nv_bfloat16* __restrict__ y,
                       int64_t B, int64_t T, int64_t D, int64_t n_commit) {
    tc::grid_dep_launch();
    tc::grid_dep_wait();           // proj comes from the previous kernel
    const int64_t d = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (d >= D) return;
    const int64_t b = blockIdx.z;
    const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kConvTile;
    const int64_t D3 = 3 * D;
    const float* pb = proj + b * T * D3 + d;          // (b, t, d) at pb[t * D3]
    double w[K];
#pragma unroll
    for (int tau = 0; tau < K; ++tau) w[tau] = conv_w[d * K + tau];
    // window[0..K-2] = u at positions t0-K+1 .. t0-1
    float win[K - 1];
#pragma unroll
    for (int i = 0; i < K - 1; ++i) {
        const int64_t t = t0 - (K - 1) + i;
        if (t >= 0) {
            win[i] = __fmul_rn(pb[t * D3], pb[t * D3 + 2 * D]);
        } else {
            // slot K-1+t of the ring holds u at position t (t = -1 newest)
            win[i] = ring[(b * (K - 1) + (K - 1 + t)) * D + d];
        }
    }
    const int n = static_cast<int>((T - t0) < kConvTile ? (T - t0) : kConvTile);
    // Blocks of kSub positions: all loads of a block first, then the window
    // walk. A decode call (one position) runs one block, not the whole tile.
    constexpr int kSub = 8;
    __nv_bfloat16* yb = y + (b * T + t0) * D + d;
    float committed[K - 1];                              // kWriteRing: ring after n_commit - 1
#pragma unroll
    for (int tau = 0; tau < K - 1; ++tau) committed[tau] = win[tau];
#pragma unroll 1
    for (int i0 = 0; i0 < n; i0 += kSub) {
        float bg[kSub], cg[kSub], xv[kSub];
#pragma unroll
        for (int i = 0; i < kSub; ++i) {
            if (i0 + i < n) {
                const float* p = pb + (t0 + i0 + i) * D3;
                bg[i] = p[0];
                cg[i] = p[D];
                xv[i] = p[2 * D];
            }
        }
#pragma unroll
        for (int i = 0; i < kSub; ++i) {
            if (i0 + i < n) {
                const float u = __fmul_rn(bg[i], xv[i]);
                double conv = 0.0;
#pragma unroll
                for (int tau = 0; tau < K - 1; ++tau)
                    conv = fma(w[tau], static_cast<double>(win[tau]), conv);
                conv = fma(w[K - 1], static_cast<double>(u), conv);
                yb[static_cast<int64_t>(i0 + i) * D] =
                    __double2bfloat16(static_cast<double>(cg[i]) * conv);
#pragma unroll
                for (int tau = 0; tau < K - 2; ++tau) win[tau] = win[tau + 1];
                win[K - 2] = u;
                if (kWriteRing && t0 + i0 + i == n_commit - 1) {
#pragma unroll
                    for (int tau = 0; tau < K - 1; ++tau) committed[tau] = win[tau];
                }
            }
        }
    }
    if constexpr (kWriteRing) {
        float* rg = ring + b * (K - 1) * D + d;
#pragma unroll
        for (int tau = 0; tau < K - 1; ++tau) rg[tau * D] = committed[tau];
        if (scratch_ring) {
            float* sg = scratch_ring + b * (K - 1) * D + d;
#pragma unroll
            for (int tau = 0; tau < K - 1; ++tau) sg[tau * D] = win[tau];
        }
    }
}

// For one (sequence, channel): the ring after position n_commit - 1 (its K-1
// newest gated inputs) into `ring`, and the ring after position T - 1 into
// `scratch_ring` when one is given; gated inputs come from proj and, before
// position 0, from the old ring. Every read precedes every write of the
// thread's own column, so the update is safe in place.
template <int K>
__global__ void __launch_bounds__(256)
short_conv_ring_kernel(const float* __restrict__ proj, float* ring, float* scratch_ring,
                       int64_t B, int64_t T, int64_t D, int64_t n_commit) {
    tc::grid_dep_launch();
    tc::grid_dep_wait();
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= B * D) return;
    const int64_t b = idx / D;
    const int64_t d = idx - b * D;
    const int64_t D3 = 3 * D;
    const float* pb = proj + b * T * D3 + d;
    float* rg = ring + b * (K - 1) * D + d;
    float old[K - 1];
#pragma unroll
    for (int i = 0; i < K - 1; ++i) old[i] = rg[i * D];
    // gated input at position t; slot K-1+t of the old ring before position 0
    auto u_at = [&](int64_t t) -> float {
        return t >= 0 ? __fmul_rn(pb[t * D3], pb[t * D3 + 2 * D]) : old[K - 1 + t];
    };
    float committed[K - 1], tentative[K - 1];
#pragma unroll
    for (int i = 0; i < K - 1; ++i) {
        committed[i] = u_at(n_commit - (K - 1) + i);
        tentative[i] = u_at(T - (K - 1) + i);
    }
#pragma unroll
    for (int i = 0; i < K - 1; ++i) rg[i * D] = committed[i];
    if (scratch_ring) {
        float* sg = scratch_ring + b * (K - 1) * D + d;
#pragma unroll
        for (int i = 0; i < K - 1; ++i) sg[i * D] = tentative[i];
    }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Launch with programmatic stream serialization (each kernel here waits for
// its predecessor with griddepcontrol.wait before touching memory).
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, cudaStream_t stream,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

template <int K>
cudaError_t launch_conv(const ShortConvArgs& a, float* proj, __nv_bfloat16* y,
                        cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>((a.D + 255) / 256),
                    static_cast<unsigned>((a.T + kConvTile - 1) / kConvTile),
                    static_cast<unsigned>(a.B));
    if (a.T <= kConvTile)            // one tile: the gate pass also writes the rings
        return launch_pdl(short_conv_gate_kernel<K, true>, grid, dim3(256), stream, proj,
                          a.conv_ring, a.scratch_ring, a.conv_w, y, a.B, a.T, a.D, a.n_commit);
    cudaError_t err = launch_pdl(short_conv_gate_kernel<K, false>, grid, dim3(256), stream, proj,
                                 a.conv_ring, static_cast<float*>(nullptr), a.conv_w, y, a.B,
                                 a.T, a.D, a.n_commit);
    if (err != cudaSuccess) return err;
    const int64_t n = a.B * a.D;
    return launch_pdl(short_conv_ring_kernel<K>, dim3(static_cast<unsigned>((n + 255) / 256)),
                      dim3(256), stream, static_cast<const float*>(proj), a.conv_ring,
                      a.scratch_ring, a.B, a.T, a.D, a.n_commit);
}

}  // namespace

ShortConvLayout short_conv_layout(int64_t B, int64_t T, int64_t D) {
    const int64_t BT = B * T;
    ShortConvLayout L;
    L.proj = 0;
    L.y = align256(static_cast<size_t>(BT) * 3 * D * 4);
    L.bar = align256(L.y + static_cast<size_t>(BT) * D * 2);
    L.total = L.bar + 256;
    return L;
}

cudaError_t launch_short_conv(const ShortConvArgs& a, cudaStream_t stream) {
    const int64_t BT = a.B * a.T;
    if (BT == 0) return cudaSuccess;
    const ShortConvLayout L = short_conv_layout(a.B, a.T, a.D);
    char* ws = static_cast<char*>(a.workspace);
    float* proj = reinterpret_cast<float*>(ws + L.proj);
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(ws + L.y);
    // one or two positions, at most 128 rows: the whole mixer in one kernel,
    // unless the environment turns it off (GDN_SHORT_CONV_ONE_KERNEL=0; read
    // at every call)
    cudaError_t err = cudaErrorNotSupported;
    const char* one = std::getenv("GDN_SHORT_CONV_ONE_KERNEL");
    if (GDN_SHORT_CONV_FUSED && !(one && one[0] == '0' && one[1] == '\0'))
        err = launch_short_conv_fused(a, y, reinterpret_cast<unsigned long long*>(ws + L.bar),
                                      stream);
    if (err != cudaErrorNotSupported) return err;
    // at most 128 rows: stages 1-3 in one kernel (the split-K projection with
    // the gate, conv and rings as its epilogue), then stage 4
    err = launch_short_conv_in_gate(a, y, stream);
    if (err == cudaSuccess)
        return launch_linear_bf16_split(LinearArgs{y, a.w_out, a.out, BT, a.D, a.D, a.status},
                                        stream);
    if (err != cudaErrorNotSupported) return err;
    err = launch_linear_bf16_split(LinearArgs{a.hidden, a.w_in, proj, BT, 3 * a.D, a.D,
                                                    a.status}, stream);
    if (err != cudaSuccess) return err;
    switch (a.K) {
        case 2: err = launch_conv<2>(a, proj, y, stream); break;
        case 3: err = launch_conv<3>(a, proj, y, stream); break;
        case 4: err = launch_conv<4>(a, proj, y, stream); break;
        default: return cudaErrorInvalidValue;
    }
    if (err != cudaSuccess) return err;
    return launch_linear_bf16_split(LinearArgs{y, a.w_out, a.out, BT, a.D, a.D, a.status},
                                    stream);
}

}  // namespace gdn
