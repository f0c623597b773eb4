// gdn_layer_decode.cu -- fused single-token recurrent layer:
// conv prestate -> Gated DeltaNet recurrence -> gated RMSNorm tail.
//
// Page "Red Lite dev15e -- complete recurrent DeltaNet layer composition"
// (opening list: conv/prestate path with beta/decay transforms and Q/K L2
// normalisation, the recurrent state update, gated RMSNorm with
// ssm_norm.weight and SiLU(z)); stage order from "Red Lite dev15a --
// DeltaNet projection field validation", section "Validation boundary"
// (conv-state shift, ssm_conv1d, SiLU, Q/K/V split, per-head Q/K L2
// normalisation); recurrence from "Red Lite dev15c -- Gated DeltaNet
// recurrent-state parity", section "Pinned llama.cpp semantics".
//
// Design: one CTA per (sequence b, key head g). It owns every channel that
// key head's work reads -- the q and k slices of head g and the v slices of
// the G = Hv / Hk value heads h = g, g + Hk, ... -- so the conv ring of each
// channel is read and rewritten by exactly one thread, and it owns the full
// 128 rows of those value heads, so the RMSNorm over a head's 128 outputs is
// a reduction inside the CTA. The first state rows are requested before the
// prestate runs, so their HBM latency overlaps the conv and norms. State rows
// then stream exactly as in the decode-step kernel (one 16-byte float4 per
// lane per row, read once, written once).
#include "gdn_common.cuh"
#include "gdn_internal.h"

#ifndef GDN_LAYER_ROWS
#define GDN_LAYER_ROWS 8
#endif

namespace gdn {

namespace {

constexpr int kLayerThreads = 256;
constexpr int kLayerWarps = kLayerThreads / 32;

template <int G, int R>
__global__ void __launch_bounds__(kLayerThreads)
layer_decode_kernel(const float* __restrict__ mixed_qkv, const float* __restrict__ z,
                    const float* __restrict__ a_in, const float* __restrict__ b_in,
                    float* __restrict__ conv_ring, const float* __restrict__ conv_w,
                    const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                    const float* __restrict__ norm_w, float l2_eps, float norm_eps,
                    float* __restrict__ state, float* __restrict__ out, int Hk, int Hv) {
    __shared__ __align__(16) float s_q[kDk];     // read back as float4
    __shared__ __align__(16) float s_k[kDk];
    __shared__ float s_v[G][kDv];
    __shared__ float s_o[G][kDv];
    __shared__ float s_beta[G];
    __shared__ float s_decay[G];
    __shared__ float s_inv[2];
    __shared__ float s_red[kLayerWarps];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t b = blockIdx.x / Hk;
    const int g = static_cast<int>(blockIdx.x % Hk);
    const int64_t C = static_cast<int64_t>(2 * Hk) * kDk + static_cast<int64_t>(Hv) * kDv;

    // Row tasks of this CTA: G heads x (128 / R) row groups, dealt to warps.
    constexpr int kTasksPerHead = kDv / R;
    constexpr int kTasks = G * kTasksPerHead;
    auto task_rows = [&](int task) -> float* {
        const int hh = task / kTasksPerHead;
        const int row0 = (task % kTasksPerHead) * R;
        const int h = g + hh * Hk;
        return state + ((b * Hv + h) * kDv + row0) * kDk + lane * 4;
    };
    float4 m[R];
    if (warp < kTasks) {
        const float* rows = task_rows(warp);
#pragma unroll
        for (int r = 0; r < R; ++r) m[r] = ld_stream(rows + r * kDk);
    }

    // ---- prestate: conv with ring shift, SiLU, split -------------------
    constexpr int kLocalChannels = (2 + G) * kDk;
    const float* x_row = mixed_qkv + b * C;
    float* ring = conv_ring + b * (kConvK - 1) * C;
    for (int lc = tid; lc < kLocalChannels; lc += kLayerThreads) {
        const int seg = lc / kDk;          // 0: q, 1: k, 2..: v of head g + (seg-2) Hk
        const int off = lc % kDk;
        int64_t ch;
        if (seg == 0) ch = static_cast<int64_t>(g) * kDk + off;
        else if (seg == 1) ch = static_cast<int64_t>(Hk + g) * kDk + off;
        else ch = static_cast<int64_t>(2 * Hk) * kDk + static_cast<int64_t>(g + (seg - 2) * Hk) * kDv + off;
        const float x = x_row[ch];
        const float r0 = ring[ch];
        const float r1 = ring[C + ch];
        const float r2 = ring[2 * C + ch];
        const float4 w = ld_ro4(conv_w + ch * kConvK);
        const float y = fmaf(w.w, x, fmaf(w.z, r2, fmaf(w.y, r1, w.x * r0)));
        ring[ch] = r1;
        ring[C + ch] = r2;
        ring[2 * C + ch] = x;
        const float act = siluf_acc(y);
        if (seg == 0) s_q[off] = act;
        else if (seg == 1) s_k[off] = act;
        else s_v[seg - 2][off] = act;
    }
    // ---- beta and decay ------------------------------------------------
    if (tid < G) {
        const int h = g + tid * Hk;
        const int64_t bh = b * Hv + h;
        s_beta[tid] = sigmoidf_acc(b_in[bh]);
        const float gt = -expf(A_log[h]) * softplusf_acc(a_in[bh] + dt_bias[h]);
        s_decay[tid] = expf(gt);
    }
    __syncthreads();
    // ---- per-head L2 norm of q (warp 0) and k (warp 1) ----------------
    if (warp < 2) {
        const float* src = warp == 0 ? s_q : s_k;
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < kDk / 32; ++i) {
            const float x = src[lane + 32 * i];
            ss = fmaf(x, x, ss);
        }
        ss = warp_sum(ss);
        if (lane == 0) s_inv[warp] = 1.0f / fmaxf(sqrtf(ss), l2_eps);
    }
    __syncthreads();

    // ---- recurrence ------------------------------------------------------
    const float inv_q = s_inv[0];
    const float inv_k = s_inv[1];
    float4 k4 = *reinterpret_cast<const float4*>(&s_k[lane * 4]);
    float4 q4 = *reinterpret_cast<const float4*>(&s_q[lane * 4]);
    k4.x *= inv_k; k4.y *= inv_k; k4.z *= inv_k; k4.w *= inv_k;
    q4.x *= inv_q; q4.y *= inv_q; q4.z *= inv_q; q4.w *= inv_q;
    for (int task = warp; task < kTasks; task += kLayerWarps) {
        float4 nxt[R];
        const bool more = task + kLayerWarps < kTasks;
        if (more) {
            const float* rows = task_rows(task + kLayerWarps);
#pragma unroll
            for (int r = 0; r < R; ++r) nxt[r] = ld_stream(rows + r * kDk);
        }
        const int hh = task / kTasksPerHead;
        const int row0 = (task % kTasksPerHead) * R;
        const float decay = s_decay[hh];
        const float bt = s_beta[hh];
        float* rows = task_rows(task);
        float o_lane = 0.0f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float4 x = m[r];
            x.x *= decay; x.y *= decay; x.z *= decay; x.w *= decay;        // step 1
            const float sk = warp_sum(dot4(x, k4));                        // step 2
            const float delta = (s_v[hh][row0 + r] - sk) * bt;             // step 3
            x.x = fmaf(delta, k4.x, x.x);                                  // step 4
            x.y = fmaf(delta, k4.y, x.y);
            x.z = fmaf(delta, k4.z, x.z);
            x.w = fmaf(delta, k4.w, x.w);
            const float o = warp_sum(dot4(x, q4)) * kOutScale;             // step 5
            if (lane == r) o_lane = o;
            st_stream(rows + r * kDk, x);
        }
        if (lane < R) s_o[hh][row0 + lane] = o_lane;
        if (more) {
#pragma unroll
            for (int r = 0; r < R; ++r) m[r] = nxt[r];
        }
    }
    __syncthreads();

    // ---- gated RMSNorm tail: per head, over its 128 outputs -----------
    for (int hh = 0; hh < G; ++hh) {
        float ss = 0.0f;
        if (tid < kDv) {
            const float o = s_o[hh][tid];
            ss = o * o;
        }
        ss = warp_sum(ss);
        if (lane == 0) s_red[warp] = ss;
        __syncthreads();
        if (tid < kDv) {
            float tot = 0.0f;
#pragma unroll
            for (int w = 0; w < kDv / 32; ++w) tot += s_red[w];
            const float inv_rms = 1.0f / sqrtf(tot / static_cast<float>(kDv) + norm_eps);
            const int h = g + hh * Hk;
            const int64_t idx = (b * Hv + h) * kDv + tid;
            out[idx] = s_o[hh][tid] * inv_rms * norm_w[tid] * siluf_acc(z[idx]);
        }
        __syncthreads();
    }
}

template <int G>
cudaError_t launch_g(const LayerArgs& a, cudaStream_t stream) {
    const int64_t grid = a.B * a.Hk;
    layer_decode_kernel<G, GDN_LAYER_ROWS><<<static_cast<unsigned>(grid), kLayerThreads, 0, stream>>>(
        a.mixed_qkv, a.z, a.a, a.b, a.conv_ring, a.conv_w, a.A_log, a.dt_bias, a.norm_w,
        a.l2_eps, a.norm_eps, a.state, a.out, a.Hk, a.Hv);
    return cudaGetLastError();
}

}  // namespace

// Value heads per key head supported by the fused kernel.
bool layer_decode_supports(int G) { return G == 1 || G == 2 || G == 4; }

cudaError_t launch_layer_decode(const LayerArgs& a, cudaStream_t stream) {
    if (a.B == 0) return cudaSuccess;
    switch (a.Hv / a.Hk) {
        case 1: return launch_g<1>(a, stream);
        case 2: return launch_g<2>(a, stream);
        case 4: return launch_g<4>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
