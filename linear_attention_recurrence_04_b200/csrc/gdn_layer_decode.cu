// gdn_layer_decode.cu -- fused recurrent layer for one token (gdn_layer_decode)
// or for a committed token plus a tentative draft token (gdn_layer_pair):
// conv prestate -> Gated DeltaNet recurrence -> gated RMSNorm tail.
//
// Page "Red Lite dev15e -- complete recurrent DeltaNet layer composition"
// (opening list: conv/prestate path with beta/decay transforms and Q/K L2
// normalisation, the recurrent state update, gated RMSNorm with
// ssm_norm.weight and SiLU(z)); stage order from "Red Lite dev15a --
// DeltaNet projection field validation", section "Validation boundary"
// (conv-state shift, ssm_conv1d, SiLU, Q/K/V split, per-head Q/K L2
// normalisation); recurrence from "Red Lite dev15c -- Gated DeltaNet
// recurrent-state parity", section "Pinned llama.cpp semantics"; the pair
// from "Module linear_core", entry "gdn_pair" (lane 1 commits into the
// state, lane 2 is tentative in scratch, ring and state moving together).
//
// Design: one CTA per (sequence b, key head g). It owns every channel that
// key head's work reads -- the q and k slices of head g and the v slices of
// the G = Hv / Hk value heads h = g, g + Hk, ... -- so the conv ring of each
// channel is read and rewritten by exactly one thread, and it owns the full
// 128 rows of those value heads, so the RMSNorm over a head's 128 outputs is
// a reduction inside the CTA. The first state rows are requested before the
// prestate runs, so their HBM latency overlaps the conv and norms. State rows
// then stream as in the decode-step kernel (one 16-byte float4 per lane per
// row); with two positions each row is read once and written twice (live
// state after position 0, scratch state after position 1).
//
// Precision: the tail divides each head's outputs by their RMS, which
// magnifies the rounding of everything upstream, so the kernel keeps its
// arithmetic in double while the state stays fp32 in memory. The prestate
// runs in double; each state row m (the fp32 values read from HBM, exact in
// double) is dotted in double with the q and k of every position of the
// call; steps 1-5 are then applied through the identities
//     sk_0  = e_0 (m.k_0),   delta_0 = (v_0 - sk_0) beta_0,
//     out_0 = e_0 (m.q_0) + delta_0 (k_0.q_0),
// and for the second position of a pair, expanded from the same row,
//     m_1.k_1 = e_0 (m.k_1) + delta_0 (k_0.k_1),
//     m_1.q_1 = e_0 (m.q_1) + delta_0 (k_0.q_1),
//     sk_1 = e_1 (m_1.k_1),  delta_1 = (v_1 - sk_1) beta_1,
//     out_1 = e_1 (m_1.q_1) + delta_1 (k_1.q_1),
// which are steps 1-5 rearranged (the output still sees the updated state).
// The rows stored back, m_1 = e_0 m + delta_0 k_0 and m_2 = e_1 m_1 +
// delta_1 k_1, are formed in fp32. The RMSNorm tail runs in double.
#include "gdn_common.cuh"
#include "gdn_internal.h"

#ifndef GDN_LAYER_MIN_CTAS
#define GDN_LAYER_MIN_CTAS 0       // resident CTAs per SM the register budget targets (0: per variant)
#endif
#ifndef GDN_LAYER_ROWS
#define GDN_LAYER_ROWS 4           // state rows per warp task
#endif
#ifndef GDN_LAYER_STAGES
#define GDN_LAYER_STAGES 3         // row groups in flight per warp (shared-memory ring)
#endif

namespace gdn {

namespace {

constexpr int kLayerThreads = 256;
constexpr int kLayerWarps = kLayerThreads / 32;

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
    return x;
}
__device__ __forceinline__ double silu_d(double x) { return x / (1.0 + exp(-x)); }
__device__ __forceinline__ double sigmoid_d(double x) { return 1.0 / (1.0 + exp(-x)); }
// softplus(x) = ln(1 + e^x) = max(x, 0) + ln(1 + e^-|x|)
__device__ __forceinline__ double softplus_d(double x) { return fmax(x, 0.0) + log1p(exp(-fabs(x))); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

struct D4 {
    double x, y, z, w;
};
__device__ __forceinline__ double dot_fd(float4 a, const D4& b) {
    return fma(static_cast<double>(a.w), b.w,
               fma(static_cast<double>(a.z), b.z,
                   fma(static_cast<double>(a.y), b.y, static_cast<double>(a.x) * b.x)));
}

// NPOS = 1: one token, ring and state updated in place.
// NPOS = 2: position 0 commits into conv_ring/state, position 1 continues
//           into scratch_ring/scratch_state. Activations are [B][NPOS][...].
// Resident CTAs per SM that the register budget targets. One position with
// two or more value heads per key head fits four CTAs (64 registers) without
// spilling, so more CTAs overlap their prestate / rows / tail phases (measured
// 187.5 us against 195.1 us at B = 256); the two-position verify spills at 64
// registers (462 us against 308 us), so it keeps three.
constexpr int layer_min_ctas(int g, int npos) {
    return GDN_LAYER_MIN_CTAS ? GDN_LAYER_MIN_CTAS : (npos == 1 && g >= 2) ? 4 : 3;
}

template <int G, int R, int NPOS>
__global__ void __launch_bounds__(kLayerThreads, layer_min_ctas(G, NPOS))
layer_kernel(const float* __restrict__ mixed_qkv, const float* __restrict__ z,
             const float* __restrict__ a_in, const float* __restrict__ b_in,
             float* __restrict__ conv_ring, const float* __restrict__ conv_w,
             const float* __restrict__ A_log, const float* __restrict__ dt_bias,
             const float* __restrict__ norm_w, float l2_eps, float norm_eps,
             float* __restrict__ state, float* __restrict__ scratch_ring,
             float* __restrict__ scratch_state, float* __restrict__ out, int Hk, int Hv) {
    __shared__ __align__(16) double s_q[NPOS][kDk];
    __shared__ __align__(16) double s_k[NPOS][kDk];
    __shared__ double s_v[NPOS][G][kDv];
    __shared__ double s_o[NPOS][G][kDv];
    __shared__ double s_beta[NPOS][G];
    __shared__ double s_decay[NPOS][G];
    __shared__ double s_inv[NPOS][2];
    __shared__ double s_kq[4];            // k0.q0, k0.k1, k0.q1, k1.q1
    __shared__ double s_red[kLayerWarps];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t b = blockIdx.x / Hk;
    const int g = static_cast<int>(blockIdx.x % Hk);
    const int64_t C = static_cast<int64_t>(2 * Hk) * kDk + static_cast<int64_t>(Hv) * kDv;
    const int64_t HD = static_cast<int64_t>(Hv) * kDv;

    // Row tasks of this CTA: G heads x (128 / R) row groups, dealt to warps.
    constexpr int kTasksPerHead = kDv / R;
    constexpr int kTasks = G * kTasksPerHead;
    auto row_offset = [&](int task) -> int64_t {
        const int hh = task / kTasksPerHead;
        const int row0 = (task % kTasksPerHead) * R;
        const int h = g + hh * Hk;
        return ((b * Hv + h) * kDv + row0) * kDk + lane * 4;
    };
    // Each lane stages its own 16 bytes of every row of the warp's next row
    // groups in a shared-memory ring, kStages groups ahead, and later reads
    // back exactly those bytes, so no barrier is needed between copy and use.
    constexpr int kStages = GDN_LAYER_STAGES;
    extern __shared__ float4 s_dyn[];
    auto s_rows = reinterpret_cast<float4 (*)[kStages][R][32]>(s_dyn);   // [warp][slot][row][lane]
    auto stage_rows = [&](int task, int slot) {
        const float* rows = state + row_offset(task);
#pragma unroll
        for (int r = 0; r < R; ++r) cp_async16(&s_rows[warp][slot][r][lane], rows + r * kDk);
    };
#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) {
        const int task = warp + i * kLayerWarps;
        if (task < kTasks) stage_rows(task, i);
        cp_async_commit();
    }

    // ---- prestate: conv with ring shift, SiLU, split (double) ----------
    constexpr int kLocalChannels = (2 + G) * kDk;
    float* ring = conv_ring + b * (kConvK - 1) * C;
    float* sring = (NPOS == 2) ? scratch_ring + b * (kConvK - 1) * C : nullptr;
    for (int lc = tid; lc < kLocalChannels; lc += kLayerThreads) {
        const int seg = lc / kDk;          // 0: q, 1: k, 2..: v of head g + (seg-2) Hk
        const int off = lc % kDk;
        int64_t ch;
        if (seg == 0) ch = static_cast<int64_t>(g) * kDk + off;
        else if (seg == 1) ch = static_cast<int64_t>(Hk + g) * kDk + off;
        else ch = static_cast<int64_t>(2 * Hk) * kDk + static_cast<int64_t>(g + (seg - 2) * Hk) * kDv + off;
        // window, oldest first: ring slots, then this call's positions
        float win[kConvK - 1 + NPOS];
        win[0] = ring[ch];
        win[1] = ring[C + ch];
        win[2] = ring[2 * C + ch];
#pragma unroll
        for (int ps = 0; ps < NPOS; ++ps) win[3 + ps] = mixed_qkv[(b * NPOS + ps) * C + ch];
        const float4 w = ld_ro4(conv_w + ch * kConvK);
#pragma unroll
        for (int ps = 0; ps < NPOS; ++ps) {
            double y = static_cast<double>(w.x) * win[ps];
            y = fma(static_cast<double>(w.y), static_cast<double>(win[ps + 1]), y);
            y = fma(static_cast<double>(w.z), static_cast<double>(win[ps + 2]), y);
            y = fma(static_cast<double>(w.w), static_cast<double>(win[ps + 3]), y);
            const double act = silu_d(y);
            if (seg == 0) s_q[ps][off] = act;
            else if (seg == 1) s_k[ps][off] = act;
            else s_v[ps][seg - 2][off] = act;
        }
        // ring after position 0 (committed), and after position 1 (scratch)
        ring[ch] = win[1];
        ring[C + ch] = win[2];
        ring[2 * C + ch] = win[3];
        if (NPOS == 2) {
            sring[ch] = win[2];
            sring[C + ch] = win[3];
            sring[2 * C + ch] = win[NPOS == 2 ? 4 : 3];
        }
    }
    // ---- beta and decay ------------------------------------------------
    if (tid < G * NPOS) {
        const int hh = tid % G;
        const int ps = tid / G;
        const int h = g + hh * Hk;
        const int64_t bh = (b * NPOS + ps) * Hv + h;
        s_beta[ps][hh] = sigmoid_d(b_in[bh]);
        const double gt = -exp(static_cast<double>(A_log[h])) *
                          softplus_d(static_cast<double>(a_in[bh]) + dt_bias[h]);
        s_decay[ps][hh] = exp(gt);
    }
    __syncthreads();
    // ---- per-head L2 norm of q and k (one warp per vector) -------------
    if (warp < 2 * NPOS) {
        const int ps = warp >> 1;
        const double* src = (warp & 1) ? s_k[ps] : s_q[ps];
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < kDk / 32; ++i) {
            const double x = src[lane + 32 * i];
            ss = fma(x, x, ss);
        }
        ss = warp_sum_d(ss);
        if (lane == 0) s_inv[ps][warp & 1] = 1.0 / fmax(sqrt(ss), static_cast<double>(l2_eps));
    }
    __syncthreads();
    // normalise in place (thread tid < 128 NPOS handles column tid % 128)
    if (tid < kDk * NPOS) {
        const int ps = tid / kDk, col = tid % kDk;
        s_q[ps][col] *= s_inv[ps][0];
        s_k[ps][col] *= s_inv[ps][1];
    }
    __syncthreads();
    // key-query products the identities need (one warp each)
    if (warp < (NPOS == 2 ? 4 : 1)) {
        const double* x = (warp == 3) ? s_k[NPOS - 1] : s_k[0];
        const double* y = (warp == 0) ? s_q[0] : (warp == 1) ? s_k[NPOS - 1] : s_q[NPOS - 1];
        double acc = 0.0;
#pragma unroll
        for (int i = 0; i < kDk / 32; ++i) acc = fma(x[lane + 32 * i], y[lane + 32 * i], acc);
        acc = warp_sum_d(acc);
        if (lane == 0) s_kq[warp] = acc;
    }
    __syncthreads();

    // ---- recurrence ------------------------------------------------------
    D4 kd[NPOS], qd[NPOS];
    float4 kf0, kf1;
#pragma unroll
    for (int ps = 0; ps < NPOS; ++ps) {
        kd[ps] = *reinterpret_cast<const D4*>(&s_k[ps][lane * 4]);
        qd[ps] = *reinterpret_cast<const D4*>(&s_q[ps][lane * 4]);
    }
    kf0 = make_float4(static_cast<float>(kd[0].x), static_cast<float>(kd[0].y),
                      static_cast<float>(kd[0].z), static_cast<float>(kd[0].w));
    kf1 = make_float4(static_cast<float>(kd[NPOS - 1].x), static_cast<float>(kd[NPOS - 1].y),
                      static_cast<float>(kd[NPOS - 1].z), static_cast<float>(kd[NPOS - 1].w));
    const double kq00 = s_kq[0];
    const double kk01 = (NPOS == 2) ? s_kq[1] : 0.0;
    const double kq01 = (NPOS == 2) ? s_kq[2] : 0.0;
    const double kq11 = (NPOS == 2) ? s_kq[3] : 0.0;
    for (int i = 0, task = warp; task < kTasks; ++i, task += kLayerWarps) {
        cp_async_wait<kStages - 2>();              // this lane's copies of group i landed
        {
            const int ahead = task + (kStages - 1) * kLayerWarps;
            if (ahead < kTasks) stage_rows(ahead, (i + kStages - 1) % kStages);
            cp_async_commit();
        }
        const float4* m = s_rows[warp][i % kStages][0] + lane;   // m[r * 32]
        const int hh = task / kTasksPerHead;
        const int row0 = (task % kTasksPerHead) * R;
        const int64_t off = row_offset(task);
        const double e0 = s_decay[0][hh], b0 = s_beta[0][hh];
        const float e0f = static_cast<float>(e0);
        double o_lane[NPOS];
#pragma unroll
        for (int ps = 0; ps < NPOS; ++ps) o_lane[ps] = 0.0;
        // dot products of the task's input rows with k and q of every
        // position, in double, reduced over the warp RG rows at a time (value
        // (rr * NPOS + ps) * 2 + {0: m.k, 1: m.q})
        constexpr int RG = (NPOS == 2 && R % 2 == 0) ? 2 : R;   // rows reduced together
        constexpr int kVals = RG * NPOS * 2;
#pragma unroll
        for (int rg = 0; rg < R; rg += RG) {
            float4 xs[RG];
            double dots[kVals];
#pragma unroll
            for (int rr = 0; rr < RG; ++rr) {
                xs[rr] = m[(rg + rr) * 32];
#pragma unroll
                for (int ps = 0; ps < NPOS; ++ps) {
                    dots[(rr * NPOS + ps) * 2] = dot_fd(xs[rr], kd[ps]);
                    dots[(rr * NPOS + ps) * 2 + 1] = dot_fd(xs[rr], qd[ps]);
                }
            }
            const double tot = warp_sum_many<kVals>(dots, lane);
            auto dot_of = [&](int rr, int ps, int which) -> double {
                return __shfl_sync(kFull, tot, sum_many_lane<kVals>((rr * NPOS + ps) * 2 + which));
            };
#pragma unroll
            for (int rr = 0; rr < RG; ++rr) {
                const int r = rg + rr;
                const float4 x = xs[rr];
                const double mk0 = dot_of(rr, 0, 0);
                const double mq0 = dot_of(rr, 0, 1);
                const double d0 = (s_v[0][hh][row0 + r] - e0 * mk0) * b0;      // steps 1-3
                const double out0 = (e0 * mq0 + d0 * kq00) * static_cast<double>(kOutScale);
                if (lane == r) o_lane[0] = out0;
                // step 4 for position 0, stored to the live state
                const float d0f = static_cast<float>(d0);
                float4 m1;
                m1.x = fmaf(d0f, kf0.x, e0f * x.x);
                m1.y = fmaf(d0f, kf0.y, e0f * x.y);
                m1.z = fmaf(d0f, kf0.z, e0f * x.z);
                m1.w = fmaf(d0f, kf0.w, e0f * x.w);
                st_stream(state + off + r * kDk, m1);
                if (NPOS == 2) {
                    const double e1 = s_decay[NPOS - 1][hh], b1 = s_beta[NPOS - 1][hh];
                    const double mk1 = dot_of(rr, NPOS - 1, 0);
                    const double mq1 = dot_of(rr, NPOS - 1, 1);
                    const double m1k1 = e0 * mk1 + d0 * kk01;
                    const double m1q1 = e0 * mq1 + d0 * kq01;
                    const double d1 = (s_v[NPOS - 1][hh][row0 + r] - e1 * m1k1) * b1;
                    const double out1 = (e1 * m1q1 + d1 * kq11) * static_cast<double>(kOutScale);
                    if (lane == r) o_lane[NPOS - 1] = out1;
                    const float e1f = static_cast<float>(e1), d1f = static_cast<float>(d1);
                    float4 m2;
                    m2.x = fmaf(d1f, kf1.x, e1f * m1.x);
                    m2.y = fmaf(d1f, kf1.y, e1f * m1.y);
                    m2.z = fmaf(d1f, kf1.z, e1f * m1.z);
                    m2.w = fmaf(d1f, kf1.w, e1f * m1.w);
                    st_stream(scratch_state + off + r * kDk, m2);
                }
            }
        }
        if (lane < R) {
#pragma unroll
            for (int ps = 0; ps < NPOS; ++ps) s_o[ps][hh][row0 + lane] = o_lane[ps];
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- gated RMSNorm tail (double): per position and head ------------
    for (int ps = 0; ps < NPOS; ++ps) {
        for (int hh = 0; hh < G; ++hh) {
            double ss = 0.0;
            if (tid < kDv) {
                const double o = s_o[ps][hh][tid];
                ss = o * o;
            }
            ss = warp_sum_d(ss);
            if (lane == 0) s_red[warp] = ss;
            __syncthreads();
            if (tid < kDv) {
                double tot = 0.0;
#pragma unroll
                for (int w = 0; w < kDv / 32; ++w) tot += s_red[w];
                const double inv_rms = 1.0 / sqrt(tot / static_cast<double>(kDv) +
                                                  static_cast<double>(norm_eps));
                const int h = g + hh * Hk;
                const int64_t idx = (b * NPOS + ps) * HD + static_cast<int64_t>(h) * kDv + tid;
                out[idx] = static_cast<float>(s_o[ps][hh][tid] * inv_rms *
                                              static_cast<double>(norm_w[tid]) * silu_d(z[idx]));
            }
            __syncthreads();
        }
    }
}

template <int G, int NPOS>
cudaError_t launch_g(const LayerArgs& a, cudaStream_t stream) {
    const int64_t grid = a.B * a.Hk;
    const size_t smem = sizeof(float4) * kLayerWarps * GDN_LAYER_STAGES * GDN_LAYER_ROWS * 32;
    cudaError_t err = cudaFuncSetAttribute(layer_kernel<G, GDN_LAYER_ROWS, NPOS>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    layer_kernel<G, GDN_LAYER_ROWS, NPOS><<<static_cast<unsigned>(grid), kLayerThreads, smem, stream>>>(
        a.mixed_qkv, a.z, a.a, a.b, a.conv_ring, a.conv_w, a.A_log, a.dt_bias, a.norm_w,
        a.l2_eps, a.norm_eps, a.state, a.scratch_ring, a.scratch_state, a.out, a.Hk, a.Hv);
    return cudaGetLastError();
}

template <int NPOS>
cudaError_t launch_npos(const LayerArgs& a, cudaStream_t stream) {
    if (a.B == 0) return cudaSuccess;
    switch (a.Hv / a.Hk) {
        case 1: return launch_g<1, NPOS>(a, stream);
        case 2: return launch_g<2, NPOS>(a, stream);
        case 4: return launch_g<4, NPOS>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// Value heads per key head supported by the fused kernels.
bool layer_decode_supports(int G) { return G == 1 || G == 2 || G == 4; }

cudaError_t launch_layer_decode(const LayerArgs& a, cudaStream_t stream) {
    return launch_npos<1>(a, stream);
}

cudaError_t launch_layer_pair(const LayerArgs& a, cudaStream_t stream) {
    return launch_npos<2>(a, stream);
}

}  // namespace gdn
