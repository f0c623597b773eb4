// gdn_prefill.cu -- sequential multi-position Gated DeltaNet prefill.
//
// Page "Module linear_core", entry "gdn_forward_batch": the recurrence runs
// sequentially over positions and is elementwise identical to the
// one-position path; the per-position steps are those of "Red Lite dev15c --
// Gated DeltaNet recurrent-state parity", section "Pinned llama.cpp
// semantics".
//
// Design
//  * The state never leaves the chip between positions. Row j of a head only
//    needs k, q, v[j], beta and gate of each position, so a head's 128 x 128
//    state splits into independent rows. A warp owns 8 rows of NH value heads
//    that share one key head (h, h + Hk, ...): lane l holds a 32-column slice
//    of each of its NH rows in registers (4 lanes per row), so each k/q value
//    it reads serves NH rows; a row's dot products reduce over its 4 lanes
//    with two shuffles.
//  * Work balance: the warps ("units") are dealt to one CTA per SM in
//    contiguous runs whose lengths differ by at most one, so every SM carries
//    the same number of rows. A run covers at most two (sequence, key head,
//    head group) groups.
//  * Inputs are staged in shared memory S stages of TS positions ahead with
//    16-byte asynchronous copies (cp.async), shared by all warps of the CTA:
//    k and q rows once per group and position, each warp's v rows, beta and
//    gate. The copy of stage s + S - 1 overlaps the arithmetic of stage s.
//  * Algebra in place of step 1 (same result up to rounding): head h's state
//    is held as s * W with a per-head scalar s, so the decay is s *= e (one
//    multiply per head, not per element). With W held:
//       sk = s (W.k),  delta = (v - sk) beta,  W += (delta / s) k,
//       out = s (W_new.q) / sqrt(128),
//    three fused multiply-adds per element and position (issued two at a time
//    as packed f32x2 FMAs) instead of four. When s leaves [2^-40, 2^40] it is
//    folded back into W (W *= s, s = 1); a decay that underflows to zero
//    folds to W = 0 exactly as step 1 would. W * s is written back at the
//    end, so the stored state has its ordinary meaning.
#include "gdn_common.cuh"
#include "gdn_internal.h"

#ifndef GDN_PREFILL_TS
#define GDN_PREFILL_TS 16          // positions per stage
#endif
#ifndef GDN_PREFILL_STAGES
#define GDN_PREFILL_STAGES 3       // stages in flight
#endif
#ifndef GDN_PREFILL_MAX_WARPS
#define GDN_PREFILL_MAX_WARPS 8    // units (warps) per CTA at most
#endif
#ifndef GDN_PREFILL_FMA2
#define GDN_PREFILL_FMA2 1         // packed f32x2 FMAs for the per-element work
#endif

namespace gdn {

namespace {

constexpr int kTS = GDN_PREFILL_TS;
constexpr int kStages = GDN_PREFILL_STAGES;
constexpr int kMaxWarps = GDN_PREFILL_MAX_WARPS;
constexpr int kRowsPerUnit = 8;                 // 8 rows x 4 lanes = one warp
constexpr int kUnitsPerHead = kDv / kRowsPerUnit;
constexpr int kChunks = 8;                      // float4 chunks per lane per row
constexpr int kMaxGroups = 2;                   // groups one CTA's run can touch
constexpr int kMaxRows = kMaxWarps * kRowsPerUnit;
constexpr float kScaleLo = 0x1p-40f;
constexpr float kScaleHi = 0x1p40f;
static_assert(kMaxWarps <= kUnitsPerHead, "a run must span at most two groups");
static_assert((kTS & (kTS - 1)) == 0, "positions per stage must be a power of two");

// Shared-memory image of one stage.
template <int NH>
struct Stage {
    float kq[kMaxGroups][kTS][2][kDk];          // [group][pos][k|q][col]
    float v[kMaxGroups][kTS][NH][kMaxRows];     // rows [row_lo, row_hi) of the group
    float bg[kMaxGroups][kTS][NH][2];           // beta, gate
};

// One group of the CTA's run: (sequence b, key head g, head group grp) and the
// rows of it that the run covers.
struct Group {
    int64_t b;
    int g;
    int grp;
    int row_lo;
    int rows;
};

__device__ __forceinline__ int chunk_col(int i, int c) { return 16 * i + 4 * c; }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// d = a * b + c on two lanes of packed floats.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
#if GDN_PREFILL_FMA2
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
#else
    return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
#endif
}

__device__ __forceinline__ float2 lo2(float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(float4 v) { return make_float2(v.z, v.w); }

template <int NH>
__global__ void __launch_bounds__(32 * kMaxWarps, 1)
prefill_kernel(float* __restrict__ state, const float* __restrict__ q,
               const float* __restrict__ k, const float* __restrict__ v,
               const float* __restrict__ beta, const float* __restrict__ gate,
               float* __restrict__ out, int64_t T, int Hk, int Hv, int units_lo, int n_big) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Stage<NH>* stages = reinterpret_cast<Stage<NH>*>(smem_raw);

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int p = lane >> 2;
    const int c = lane & 3;

    // This CTA's run of units: [u0, u0 + count).
    const int cta = blockIdx.x;
    const int64_t u0 = static_cast<int64_t>(cta) * units_lo + (cta < n_big ? cta : n_big);
    const int count = units_lo + (cta < n_big ? 1 : 0);
    const int groups_per_key = (Hv / Hk) / NH;

    // The (at most two) groups the run touches.
    Group grp_of[kMaxGroups];
    const int64_t gid0 = u0 / kUnitsPerHead;
    const int64_t gid1 = (u0 + count - 1) / kUnitsPerHead;
    const int n_groups = static_cast<int>(gid1 - gid0) + 1;
#pragma unroll
    for (int gi = 0; gi < kMaxGroups; ++gi) {
        const int64_t gid = gid0 + gi;
        int64_t rest = gid;
        Group G;
        G.grp = static_cast<int>(rest % groups_per_key);
        rest /= groups_per_key;
        G.g = static_cast<int>(rest % Hk);
        G.b = rest / Hk;
        const int64_t first = gid * kUnitsPerHead > u0 ? gid * kUnitsPerHead : u0;
        const int64_t last = (gid + 1) * kUnitsPerHead < u0 + count ? (gid + 1) * kUnitsPerHead
                                                                   : u0 + count;
        G.row_lo = static_cast<int>(first - gid * kUnitsPerHead) * kRowsPerUnit;
        G.rows = static_cast<int>(last - first) * kRowsPerUnit;
        grp_of[gi] = G;
    }

    // ---- stage loader: every thread issues a share of the copies --------
    auto load_stage = [&](int64_t t0, Stage<NH>& st) {
#pragma unroll
        for (int gi = 0; gi < kMaxGroups; ++gi) {
            if (gi >= n_groups) break;
            const Group G = grp_of[gi];
            // k and q rows: TS positions x 2 x 32 chunks of 16 bytes
            for (int idx = tid; idx < kTS * 64; idx += nthreads) {
                const int chunk = idx & 31;
                const int which = (idx >> 5) & 1;
                const int tp = idx >> 6;
                const int64_t t = t0 + tp;
                if (t < T) {
                    const float* src = (which ? q : k) + ((G.b * T + t) * Hk + G.g) * kDk + chunk * 4;
                    cp_async16(&st.kq[gi][tp][which][chunk * 4], src);
                }
            }
            // v rows of the run, for each of the NH heads
            const int vchunks = G.rows / 4;
            for (int idx = tid; idx < kTS * NH * vchunks; idx += nthreads) {
                const int chunk = idx % vchunks;
                const int n = (idx / vchunks) % NH;
                const int tp = idx / (vchunks * NH);
                const int64_t t = t0 + tp;
                if (t < T) {
                    const int h = G.g + (G.grp * NH + n) * Hk;
                    const float* src = v + ((G.b * T + t) * Hv + h) * kDv + G.row_lo + chunk * 4;
                    cp_async16(&st.v[gi][tp][n][chunk * 4], src);
                }
            }
            // beta and gate
            for (int idx = tid; idx < kTS * NH * 2; idx += nthreads) {
                const int which = idx & 1;
                const int n = (idx >> 1) % NH;
                const int tp = (idx >> 1) / NH;
                const int64_t t = t0 + tp;
                if (t < T) {
                    const int h = G.g + (G.grp * NH + n) * Hk;
                    cp_async4(&st.bg[gi][tp][n][which], (which ? gate : beta) + (G.b * T + t) * Hv + h);
                }
            }
        }
    };

    // ---- this warp's unit ------------------------------------------------
    const bool active = warp < count;
    const int64_t unit = u0 + warp;
    const int gi = active ? static_cast<int>(unit / kUnitsPerHead - gid0) : 0;
    const Group G = gi == 0 ? grp_of[0] : grp_of[1];
    const int rb = static_cast<int>(unit % kUnitsPerHead);
    const int j = rb * kRowsPerUnit + p;                 // row within the head
    const int vrow = j - G.row_lo;                       // row within the staged v
    int hidx[NH];
#pragma unroll
    for (int n = 0; n < NH; ++n) hidx[n] = G.g + (G.grp * NH + n) * Hk;

    // Prologue: request the first S - 1 stages, then load the state rows.
    const int64_t n_stages_total = (T + kTS - 1) / kTS;
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < n_stages_total) load_stage(static_cast<int64_t>(s) * kTS, stages[s]);
        cp_async_commit();
    }

    float4 w[NH][kChunks];
    float sc[NH];
    if (active) {
#pragma unroll
        for (int n = 0; n < NH; ++n) {
            const float* row = state + ((G.b * Hv + hidx[n]) * kDv + j) * kDk;
#pragma unroll
            for (int i = 0; i < kChunks; ++i) w[n][i] = ld_stream(row + chunk_col(i, c));
            sc[n] = 1.0f;
        }
    }

    for (int64_t s = 0; s < n_stages_total; ++s) {
        cp_async_wait<kStages - 2>();       // this thread's copies of stage s landed
        __syncthreads();                     // ... and everyone's; stage s-1 is free
        {
            const int64_t nxt = s + kStages - 1;
            if (nxt < n_stages_total) load_stage(nxt * kTS, stages[nxt % kStages]);
            cp_async_commit();
        }
        const Stage<NH>& st = stages[s % kStages];
        const int64_t t0 = s * kTS;
        const int tp_end = (T - t0) < kTS ? static_cast<int>(T - t0) : kTS;
        if (active) {
            for (int tp = 0; tp < tp_end; ++tp) {
                float4 kk[kChunks], qq[kChunks];
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    kk[i] = *reinterpret_cast<const float4*>(&st.kq[gi][tp][0][chunk_col(i, c)]);
                    qq[i] = *reinterpret_cast<const float4*>(&st.kq[gi][tp][1][chunk_col(i, c)]);
                }
                const int64_t bt = G.b * T + t0 + tp;
                // The NH heads are independent: each phase below runs for all
                // of them before the next, so their dependency chains overlap.
                float s_new[NH], sk[NH], vj[NH], bn[NH];
                float2 a0[NH], a1[NH];
#pragma unroll
                for (int n = 0; n < NH; ++n) {
                    vj[n] = st.v[gi][tp][n][vrow];
                    bn[n] = st.bg[gi][tp][n][0];
                    // step 1 as a scale update
                    s_new[n] = sc[n] * expf(st.bg[gi][tp][n][1]);
                    // step 2: W.k (the scale enters below)
                    a0[n] = make_float2(0.f, 0.f);
                    a1[n] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int i = 0; i < kChunks; ++i) {
                        a0[n] = fma2(lo2(w[n][i]), lo2(kk[i]), a0[n]);
                        a1[n] = fma2(hi2(w[n][i]), hi2(kk[i]), a1[n]);
                    }
                }
                float delta[NH];
                bool fold = false;
#pragma unroll
                for (int n = 0; n < NH; ++n) {
                    // sk = s_new (W.k) whether or not the scale is folded below
                    sk[n] = s_new[n] * group_sum<4>((a0[n].x + a0[n].y) + (a1[n].x + a1[n].y));
                    delta[n] = (vj[n] - sk[n]) * bn[n];                  // step 3
                    fold |= !(s_new[n] >= kScaleLo && s_new[n] <= kScaleHi);
                }
                if (fold) {          // rare, and uniform across the warp
#pragma unroll
                    for (int n = 0; n < NH; ++n) {
                        if (!(s_new[n] >= kScaleLo && s_new[n] <= kScaleHi)) {
#pragma unroll
                            for (int i = 0; i < kChunks; ++i) {
                                w[n][i].x *= s_new[n]; w[n][i].y *= s_new[n];
                                w[n][i].z *= s_new[n]; w[n][i].w *= s_new[n];
                            }
                            s_new[n] = 1.0f;
                        }
                    }
                }
                float2 o0[NH], o1[NH];
#pragma unroll
                for (int n = 0; n < NH; ++n) {
                    sc[n] = s_new[n];
                    // step 4: W += (delta / s) k
                    const float cf = delta[n] * __frcp_rn(sc[n]);
                    const float2 cf2 = make_float2(cf, cf);
#pragma unroll
                    for (int i = 0; i < kChunks; ++i) {
                        const float2 lo = fma2(cf2, lo2(kk[i]), lo2(w[n][i]));
                        const float2 hi = fma2(cf2, hi2(kk[i]), hi2(w[n][i]));
                        w[n][i] = make_float4(lo.x, lo.y, hi.x, hi.y);
                    }
                    // step 5: W_new.q
                    o0[n] = make_float2(0.f, 0.f);
                    o1[n] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int i = 0; i < kChunks; ++i) {
                        o0[n] = fma2(lo2(w[n][i]), lo2(qq[i]), o0[n]);
                        o1[n] = fma2(hi2(w[n][i]), hi2(qq[i]), o1[n]);
                    }
                }
#pragma unroll
                for (int n = 0; n < NH; ++n) {
                    const float o = sc[n] * group_sum<4>((o0[n].x + o0[n].y) + (o1[n].x + o1[n].y)) * kOutScale;
                    if (c == (n & 3)) out[(bt * Hv + hidx[n]) * kDv + j] = o;
                }
            }
        }
    }
    cp_async_wait<0>();

    // Write the final state back with the scale folded in.
    if (active) {
#pragma unroll
        for (int n = 0; n < NH; ++n) {
            float* row = state + ((G.b * Hv + hidx[n]) * kDv + j) * kDk;
#pragma unroll
            for (int i = 0; i < kChunks; ++i) {
                float4 x = w[n][i];
                x.x *= sc[n]; x.y *= sc[n]; x.z *= sc[n]; x.w *= sc[n];
                st_stream(row + chunk_col(i, c), x);
            }
        }
    }
}

template <int NH>
cudaError_t launch_nh(const PrefillArgs& a, cudaStream_t stream) {
    const int G = a.Hv / a.Hk;
    const int64_t n_units = a.B * a.Hk * (G / NH) * kUnitsPerHead;
    if (n_units == 0) return cudaSuccess;
    const int64_t sms = device_sm_count();
    int64_t grid = n_units < sms ? n_units : sms;
    const int64_t min_grid = (n_units + kMaxWarps - 1) / kMaxWarps;
    if (grid < min_grid) grid = min_grid;
    const int units_lo = static_cast<int>(n_units / grid);
    const int n_big = static_cast<int>(n_units % grid);
    const int warps = units_lo + (n_big > 0 ? 1 : 0);
    const size_t smem = sizeof(Stage<NH>) * kStages;
    cudaError_t err = cudaFuncSetAttribute(prefill_kernel<NH>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    prefill_kernel<NH><<<static_cast<unsigned>(grid), 32 * warps, smem, stream>>>(
        a.state, a.q, a.k, a.v, a.beta, a.gate, a.out, a.T, a.Hk, a.Hv, units_lo, n_big);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const int G = a.Hv / a.Hk;
    return (G % 2 == 0) ? launch_nh<2>(a, stream) : launch_nh<1>(a, stream);
}

}  // namespace gdn
