// gdn_prefill.cu -- sequential multi-position Gated DeltaNet prefill.
//
// Page "Module linear_core", entry "gdn_forward_batch": the recurrence runs
// sequentially over positions and is elementwise identical to the
// one-position path; the per-position steps are those of "Red Lite dev15c --
// Gated DeltaNet recurrent-state parity", section "Pinned llama.cpp
// semantics".
//
// Design: the state never leaves the chip between positions. Row j of a head
// only needs k, q, v[j], beta and gate of each position, so the 128 x 128
// state of a head splits into independent rows. A warp owns 8 rows of NH
// value heads that share one key head (h, h + Hk, ...): lane l holds a
// 32-column slice of each of its NH rows in registers (4 lanes per row), so
// every k/q value a lane loads serves NH rows. The per-position dot products
// reduce over the 4 lanes of a row with two shuffles.
//
// Algebra used in place of step 1 (same result up to rounding): the state of
// head h is kept as s * W with a per-head scalar s, so the decay is s *= e
// (one multiply per head, not per element). With W held:
//   sk = s (W.k),  delta = (v - sk) beta,  W += (delta / s) k,
//   out = s (W_new.q) / sqrt(128).
// That is three fused multiply-adds per element and position instead of
// four. When s leaves [2^-40, 2^40] it is folded back into W (W *= s, s = 1);
// an exactly zero decay folds to W = 0 as step 1 would. At the end W * s is
// written back, so the stored state has the ordinary meaning.
#include "gdn_common.cuh"
#include "gdn_internal.h"

#ifndef GDN_PREFILL_WARPS
#define GDN_PREFILL_WARPS 1      // warps per CTA
#endif

namespace gdn {

namespace {

constexpr int kRowsPerWarp = 8;         // 8 rows x 4 lanes = 32 lanes
constexpr int kChunks = 8;              // float4 chunks per lane per row (32 columns)
constexpr float kScaleLo = 0x1p-40f;
constexpr float kScaleHi = 0x1p40f;

// Lane l covers row p = l / 4 of the warp's 8 rows and the float4 chunks
// {4 i + c : i < 8} with c = l % 4, so one warp-wide 16-byte load of k or q
// touches 64 contiguous bytes.
__device__ __forceinline__ int chunk_col(int i, int c) { return 16 * i + 4 * c; }

template <int NH>
__global__ void __launch_bounds__(32 * GDN_PREFILL_WARPS)
prefill_kernel(float* __restrict__ state, const float* __restrict__ q,
               const float* __restrict__ k, const float* __restrict__ v,
               const float* __restrict__ beta, const float* __restrict__ gate,
               float* __restrict__ out, int64_t T, int Hk, int Hv, int64_t n_units) {
    const int64_t unit = static_cast<int64_t>(blockIdx.x) * GDN_PREFILL_WARPS + (threadIdx.x >> 5);
    if (unit >= n_units) return;
    const int lane = threadIdx.x & 31;
    const int p = lane >> 2;
    const int c = lane & 3;

    // unit -> (b, g, head group, row block of 8)
    constexpr int kBlocksPerHead = kDv / kRowsPerWarp;
    const int groups = (Hv / Hk) / NH;
    int64_t rest = unit;
    const int rb = static_cast<int>(rest % kBlocksPerHead);
    rest /= kBlocksPerHead;
    const int grp = static_cast<int>(rest % groups);
    rest /= groups;
    const int g = static_cast<int>(rest % Hk);
    const int64_t b = rest / Hk;
    const int j = rb * kRowsPerWarp + p;
    int hidx[NH];
#pragma unroll
    for (int n = 0; n < NH; ++n) hidx[n] = g + (grp * NH + n) * Hk;

    // Load the NH state rows (row j of each head) into registers.
    float4 w[NH][kChunks];
    float s[NH];
#pragma unroll
    for (int n = 0; n < NH; ++n) {
        const float* row = state + ((b * Hv + hidx[n]) * kDv + j) * kDk;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) w[n][i] = ld_stream(row + chunk_col(i, c));
        s[n] = 1.0f;
    }

    // Per-position inputs, prefetched one position ahead.
    float4 kk[kChunks], qq[kChunks];
    float vv[NH], be[NH], ga[NH];
    auto load_pos = [&](int64_t t, float4 (&kd)[kChunks], float4 (&qd)[kChunks], float (&vd)[NH],
                        float (&bd)[NH], float (&gd)[NH]) {
        const int64_t bt = b * T + t;
        const float* kr = k + (bt * Hk + g) * kDk;
        const float* qr = q + (bt * Hk + g) * kDk;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            kd[i] = ld_ro4(kr + chunk_col(i, c));
            qd[i] = ld_ro4(qr + chunk_col(i, c));
        }
#pragma unroll
        for (int n = 0; n < NH; ++n) {
            const int64_t bh = bt * Hv + hidx[n];
            vd[n] = __ldg(v + bh * kDv + j);
            bd[n] = __ldg(beta + bh);
            gd[n] = __ldg(gate + bh);
        }
    };
    if (T > 0) load_pos(0, kk, qq, vv, be, ga);

    for (int64_t t = 0; t < T; ++t) {
        float4 kn[kChunks], qn[kChunks];
        float vn[NH], bn[NH], gn[NH];
        const bool more = t + 1 < T;
        if (more) load_pos(t + 1, kn, qn, vn, bn, gn);

        const int64_t bt = b * T + t;
#pragma unroll
        for (int n = 0; n < NH; ++n) {
            // step 1 as a scale update; fold the scale into W when it drifts.
            const float s_new = s[n] * expf(ga[n]);
            if (!(s_new >= kScaleLo && s_new <= kScaleHi)) {
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    w[n][i].x *= s_new; w[n][i].y *= s_new;
                    w[n][i].z *= s_new; w[n][i].w *= s_new;
                }
                s[n] = 1.0f;
            } else {
                s[n] = s_new;
            }
            // step 2: sk = s (W.k)
            float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int i = 0; i < kChunks; i += 2) {
                a0 += dot4(w[n][i], kk[i]);
                a1 += dot4(w[n][i + 1], kk[i + 1]);
            }
            const float sk = s[n] * group_sum<4>(a0 + a1);
            // step 3
            const float delta = (vv[n] - sk) * be[n];
            // step 4: W += (delta / s) k
            const float cf = delta / s[n];
#pragma unroll
            for (int i = 0; i < kChunks; ++i) {
                w[n][i].x = fmaf(cf, kk[i].x, w[n][i].x);
                w[n][i].y = fmaf(cf, kk[i].y, w[n][i].y);
                w[n][i].z = fmaf(cf, kk[i].z, w[n][i].z);
                w[n][i].w = fmaf(cf, kk[i].w, w[n][i].w);
            }
            // step 5: out = s (W_new.q) / sqrt(128)
            float o0 = 0.0f, o1 = 0.0f;
#pragma unroll
            for (int i = 0; i < kChunks; i += 2) {
                o0 += dot4(w[n][i], qq[i]);
                o1 += dot4(w[n][i + 1], qq[i + 1]);
            }
            const float o = s[n] * group_sum<4>(o0 + o1) * kOutScale;
            if (c == (n & 3)) out[(bt * Hv + hidx[n]) * kDv + j] = o;
        }

        if (more) {
#pragma unroll
            for (int i = 0; i < kChunks; ++i) { kk[i] = kn[i]; qq[i] = qn[i]; }
#pragma unroll
            for (int n = 0; n < NH; ++n) { vv[n] = vn[n]; be[n] = bn[n]; ga[n] = gn[n]; }
        }
    }

    // Write the final state back with the scale folded in.
#pragma unroll
    for (int n = 0; n < NH; ++n) {
        float* row = state + ((b * Hv + hidx[n]) * kDv + j) * kDk;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            float4 x = w[n][i];
            x.x *= s[n]; x.y *= s[n]; x.z *= s[n]; x.w *= s[n];
            st_stream(row + chunk_col(i, c), x);
        }
    }
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const int G = a.Hv / a.Hk;
    const int nh = (G % 2 == 0) ? 2 : 1;
    const int64_t n_units = a.B * a.Hk * (G / nh) * (kDv / kRowsPerWarp);
    if (n_units == 0) return cudaSuccess;
    const int64_t grid = (n_units + GDN_PREFILL_WARPS - 1) / GDN_PREFILL_WARPS;
    if (nh == 2) {
        prefill_kernel<2><<<static_cast<unsigned>(grid), 32 * GDN_PREFILL_WARPS, 0, stream>>>(
            a.state, a.q, a.k, a.v, a.beta, a.gate, a.out, a.T, a.Hk, a.Hv, n_units);
    } else {
        prefill_kernel<1><<<static_cast<unsigned>(grid), 32 * GDN_PREFILL_WARPS, 0, stream>>>(
            a.state, a.q, a.k, a.v, a.beta, a.gate, a.out, a.T, a.Hk, a.Hv, n_units);
    }
    return cudaGetLastError();
}

}  // namespace gdn
