// gdn_step.cu -- batched single-token Gated DeltaNet decode.
//
// Page "Red Lite dev15c -- Gated DeltaNet recurrent-state parity", section
// "Pinned llama.cpp semantics": per value head h (q/k of key head h % Hk),
// with M[j][i] = S[i][j],
//   1. M *= exp(gate)   2. sk[j] = M[j].k   3. delta[j] = (v[j] - sk[j]) beta
//   4. M[j] += delta[j] k   5. out[j] = M_new[j].q / sqrt(128).
//
// Design: every row j of M is independent once k, q, v[j], beta and gate are
// known, so the kernel streams rows. A warp owns R = 4 consecutive rows of one
// head; lane l holds columns [4l, 4l+4) of each row as one float4, so a row
// is one coalesced 512-byte access. All R row loads are issued before any
// arithmetic, the five steps run in registers (the R rows' key dots share one
// warp reduction, and so do their output dots), and each row is written back
// once: the state crosses HBM exactly
// once in each direction per token. Warps walk row groups with a grid-stride
// loop over a persistent grid of (SMs x resident CTAs), prefetching the next
// group's rows while the current group computes.
//
// The same kernel with a decay per key channel is the KDA core ("Module
// linear_core", entry "kda_forward"; the published Kimi Delta Attention
// update): step 1 becomes M[j][i] *= exp(g[i]), g [.., Hv, dk], so each lane
// scales its four columns by their own factors; steps 2-5 are unchanged.
#include "gdn_common.cuh"
#include "gdn_internal.h"

#ifndef GDN_STEP_ROWS
#define GDN_STEP_ROWS 4          // rows per warp task
#endif
#ifndef GDN_STEP_THREADS
#define GDN_STEP_THREADS 256     // threads per CTA
#endif
#ifndef GDN_STEP_PREFETCH
#define GDN_STEP_PREFETCH 1      // load the next task's rows before computing
#endif
#ifndef GDN_STEP_PDL
#define GDN_STEP_PDL 1           // programmatic dependent launch for grids below the persistent size
#endif


namespace gdn {

namespace {

template <int R>
struct RowTask {
    int64_t head;   // flat (layer, sequence, value head)
    int row0;       // first row j of the task
};

template <int R>
__device__ __forceinline__ RowTask<R> decode_task(int64_t task) {
    constexpr int kTasksPerHead = kDv / R;
    RowTask<R> t;
    t.head = task / kTasksPerHead;
    t.row0 = static_cast<int>(task - t.head * kTasksPerHead) * R;
    return t;
}

template <int R>
__device__ __forceinline__ void load_rows(float4 (&m)[R], const float* state, RowTask<R> t,
                                          int lane) {
    const float* rows = state + (t.head * kDv + t.row0) * kDk + lane * 4;
#pragma unroll
    for (int r = 0; r < R; ++r) m[r] = ld_stream(rows + r * kDk);
}

// Steps 1-5 on R rows held in registers; writes the rows and R outputs.
// kChannelDecay: gate holds a log-decay per key channel ([head][dk]) instead
// of one per head.
template <int R, bool kChannelDecay>
__device__ __forceinline__ void update_rows(float4 (&m)[R], float* __restrict__ state,
                                            const float* __restrict__ q,
                                            const float* __restrict__ k,
                                            const float* __restrict__ v,
                                            const float* __restrict__ beta,
                                            const float* __restrict__ gate,
                                            float* __restrict__ out, RowTask<R> t, int Hk,
                                            int Hv, int lane) {
    const int64_t lb = t.head / Hv;
    const int h = static_cast<int>(t.head - lb * Hv);
    const int64_t key = (lb * Hk + (h % Hk)) * kDk + lane * 4;
    const float4 k4 = ld_ro4(k + key);
    const float4 q4 = ld_ro4(q + key);
    float4 decay;
    if constexpr (kChannelDecay) {
        const float4 g4 = ld_ro4(gate + t.head * kDk + lane * 4);
        decay = make_float4(expf(g4.x), expf(g4.y), expf(g4.z), expf(g4.w));
    } else {
        const float e = expf(gate[t.head]);
        decay = make_float4(e, e, e, e);
    }
    const float bt = beta[t.head];
    const int64_t vrow = t.head * kDv + t.row0;
    float* rows = state + vrow * kDk + lane * 4;
    // step 1 on every row, then step 2 for all R rows in one reduction:
    // lane sum_many_lane<R>(r) receives sk of row r and forms its delta
    float part[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        m[r].x *= decay.x; m[r].y *= decay.y; m[r].z *= decay.z; m[r].w *= decay.w;
        part[r] = dot4(m[r], k4);
    }
    const float sk_lane = warp_sum_many<R>(part, lane);
    const int my_row = lane / (32 / R);                     // the row whose totals this lane holds
    const float delta_lane = (v[vrow + my_row] - sk_lane) * bt;          // step 3
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float delta = __shfl_sync(kFull, delta_lane, sum_many_lane<R>(r));
        // step 4: rank-1 update
        m[r].x = fmaf(delta, k4.x, m[r].x);
        m[r].y = fmaf(delta, k4.y, m[r].y);
        m[r].z = fmaf(delta, k4.z, m[r].z);
        m[r].w = fmaf(delta, k4.w, m[r].w);
        part[r] = dot4(m[r], q4);
        st_stream(rows + r * kDk, m[r]);
    }
    // step 5: the outputs of the updated rows, again in one reduction
    const float o_lane = warp_sum_many<R>(part, lane) * kOutScale;
    if (lane % (32 / R) == 0) out[vrow + my_row] = o_lane;
}

template <int R, bool kChannelDecay>
__global__ void __launch_bounds__(GDN_STEP_THREADS)
step_kernel(float* __restrict__ state, const float* __restrict__ q, const float* __restrict__ k,
            const float* __restrict__ v, const float* __restrict__ beta,
            const float* __restrict__ gate, float* __restrict__ out, int64_t n_tasks, int Hk,
            int Hv) {
    const int lane = threadIdx.x & 31;
    const int64_t warps_per_cta = blockDim.x >> 5;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * warps_per_cta;
    int64_t task = static_cast<int64_t>(blockIdx.x) * warps_per_cta + (threadIdx.x >> 5);
#if GDN_STEP_PDL
    // When launched with programmatic stream serialization: wait until the
    // previous grid on the stream has completed and its writes are visible,
    // then let the next one be scheduled while this one runs. Without that
    // launch attribute both are no-ops.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
    if (task >= n_tasks) return;
    float4 m[R];
    load_rows<R>(m, state, decode_task<R>(task), lane);
    for (; task < n_tasks; task += stride) {
        const RowTask<R> cur = decode_task<R>(task);
#if GDN_STEP_PREFETCH
        float4 nxt[R];
        const bool more = task + stride < n_tasks;
        if (more) load_rows<R>(nxt, state, decode_task<R>(task + stride), lane);
        update_rows<R, kChannelDecay>(m, state, q, k, v, beta, gate, out, cur, Hk, Hv, lane);
        if (more) {
#pragma unroll
            for (int r = 0; r < R; ++r) m[r] = nxt[r];
        }
#else
        update_rows<R, kChannelDecay>(m, state, q, k, v, beta, gate, out, cur, Hk, Hv, lane);
        if (task + stride < n_tasks) load_rows<R>(m, state, decode_task<R>(task + stride), lane);
#endif
    }
}

// Two positions on R rows held in registers ("Module linear_core", entry
// "gdn_pair"): position 0 as in update_rows, its rows written to `state`;
// position 1 continues from them, its rows written to `scratch`. Inputs are
// [L][B][2][..], so position p of head (lb, h) sits at row lb * 2 + p. Every
// value is formed by the same operations, in the same order, as two
// update_rows calls: the batched reduction below (position 0's output dots
// with position 1's key dots) sums each value over the same butterfly tree as
// warp_sum_many<R>, so the pair equals two gdn_step calls bit for bit.
template <int R>
__device__ __forceinline__ void pair_rows(float4 (&m)[R], float* __restrict__ state,
                                          float* __restrict__ scratch,
                                          const float* __restrict__ q,
                                          const float* __restrict__ k,
                                          const float* __restrict__ v,
                                          const float* __restrict__ beta,
                                          const float* __restrict__ gate,
                                          float* __restrict__ out, RowTask<R> t, int Hk, int Hv,
                                          int lane) {
    constexpr int kLanesPerRow = 32 / R;          // lanes holding one row's totals
    constexpr int kLanesPerVal2 = 32 / (2 * R);   // ... in the batch of 2 R values
    const int64_t lb = t.head / Hv;
    const int h = static_cast<int>(t.head - lb * Hv);
    const int64_t p0 = lb * 2;                    // (l, b, position 0); position 1 is p0 + 1
    const int g = h % Hk;
    const float4 k0 = ld_ro4(k + (p0 * Hk + g) * kDk + lane * 4);
    const float4 q0 = ld_ro4(q + (p0 * Hk + g) * kDk + lane * 4);
    const float4 k1 = ld_ro4(k + ((p0 + 1) * Hk + g) * kDk + lane * 4);
    const float4 q1 = ld_ro4(q + ((p0 + 1) * Hk + g) * kDk + lane * 4);
    const float e0 = expf(gate[p0 * Hv + h]);
    const float e1 = expf(gate[(p0 + 1) * Hv + h]);
    const float bt0 = beta[p0 * Hv + h];
    const float bt1 = beta[(p0 + 1) * Hv + h];
    const int64_t vrow0 = (p0 * Hv + h) * kDv + t.row0;
    const int64_t vrow1 = ((p0 + 1) * Hv + h) * kDv + t.row0;
    const int64_t srow = (t.head * kDv + t.row0) * kDk + lane * 4;
    float* rows = state + srow;
    float* srows = scratch + srow;

    // position 0, steps 1-2: one reduction of the R key dots
    float part[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        m[r].x *= e0; m[r].y *= e0; m[r].z *= e0; m[r].w *= e0;
        part[r] = dot4(m[r], k0);
    }
    const float sk0 = warp_sum_many<R>(part, lane);
    const int my_row = lane / kLanesPerRow;
    const float delta0_lane = (v[vrow0 + my_row] - sk0) * bt0;
    // position 0, step 4 (rows committed to `state`) and step 5's dots;
    // position 1, steps 1-2: values r < R are the output dots of row r,
    // values R + r the key dots of row r
    float part2[2 * R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float delta = __shfl_sync(kFull, delta0_lane, sum_many_lane<R>(r));
        m[r].x = fmaf(delta, k0.x, m[r].x);
        m[r].y = fmaf(delta, k0.y, m[r].y);
        m[r].z = fmaf(delta, k0.z, m[r].z);
        m[r].w = fmaf(delta, k0.w, m[r].w);
        st_stream(rows + r * kDk, m[r]);
        part2[r] = dot4(m[r], q0);
        m[r].x *= e1; m[r].y *= e1; m[r].z *= e1; m[r].w *= e1;
        part2[R + r] = dot4(m[r], k1);
    }
    const float tot = warp_sum_many<2 * R>(part2, lane);
    const int my_val = lane / kLanesPerVal2;
    if (my_val < R && lane % kLanesPerVal2 == 0) out[vrow0 + my_val] = tot * kOutScale;
    const int v1_row = my_val >= R ? my_val - R : 0;    // lanes holding an output dot read row 0
    const float delta1_lane = (v[vrow1 + v1_row] - tot) * bt1;
    // position 1, step 4 (rows to `scratch`) and step 5
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float delta = __shfl_sync(kFull, delta1_lane, sum_many_lane<2 * R>(R + r));
        m[r].x = fmaf(delta, k1.x, m[r].x);
        m[r].y = fmaf(delta, k1.y, m[r].y);
        m[r].z = fmaf(delta, k1.z, m[r].z);
        m[r].w = fmaf(delta, k1.w, m[r].w);
        st_stream(srows + r * kDk, m[r]);
        part[r] = dot4(m[r], q1);
    }
    const float o1 = warp_sum_many<R>(part, lane) * kOutScale;
    if (lane % kLanesPerRow == 0) out[vrow1 + my_row] = o1;
}

template <int R>
__global__ void __launch_bounds__(GDN_STEP_THREADS)
pair_kernel(float* __restrict__ state, float* __restrict__ scratch, const float* __restrict__ q,
            const float* __restrict__ k, const float* __restrict__ v,
            const float* __restrict__ beta, const float* __restrict__ gate,
            float* __restrict__ out, int64_t n_tasks, int Hk, int Hv) {
    const int lane = threadIdx.x & 31;
    const int64_t warps_per_cta = blockDim.x >> 5;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * warps_per_cta;
    int64_t task = static_cast<int64_t>(blockIdx.x) * warps_per_cta + (threadIdx.x >> 5);
    if (task >= n_tasks) return;
    float4 m[R];
    load_rows<R>(m, state, decode_task<R>(task), lane);
    for (; task < n_tasks; task += stride) {
        const RowTask<R> cur = decode_task<R>(task);
        float4 nxt[R];
        const bool more = task + stride < n_tasks;
        if (more) load_rows<R>(nxt, state, decode_task<R>(task + stride), lane);
        pair_rows<R>(m, state, scratch, q, k, v, beta, gate, out, cur, Hk, Hv, lane);
        if (more) {
#pragma unroll
            for (int r = 0; r < R; ++r) m[r] = nxt[r];
        }
    }
}

template <bool kChannelDecay>
cudaError_t launch_rows(const StepArgs& a, cudaStream_t stream) {
    constexpr int R = GDN_STEP_ROWS;
    static_assert(kDv % R == 0 && R <= 32, "rows per task must divide dv");
    const int64_t n_tasks = a.n_heads * (kDv / R);
    if (n_tasks == 0) return cudaSuccess;
    constexpr int threads = GDN_STEP_THREADS;
    constexpr int warps_per_cta = threads / 32;
    const int64_t needed = (n_tasks + warps_per_cta - 1) / warps_per_cta;
    int per_sm = 0;
    cudaError_t err = resident_ctas_per_sm(
        reinterpret_cast<const void*>(&step_kernel<R, kChannelDecay>), threads, &per_sm);
    if (err != cudaSuccess) return err;
    const int64_t resident = static_cast<int64_t>(device_sm_count()) * per_sm;
    const int grid = static_cast<int>(needed < resident ? needed : resident);
#if GDN_STEP_PDL
    // A grid below the persistent size (a few sequences, e.g. B = 1) is bound
    // by launch latency, and overlapping its launch with the previous grid's
    // tail measured 3.75 us against 4.05 us at B = 1. A persistent grid gains
    // nothing (B = 64) or loses a little (36 layers, 382 us against 376 us),
    // so it is launched plainly.
    if (needed > resident) {
        step_kernel<R, kChannelDecay><<<grid, threads, 0, stream>>>(
            a.state, a.q, a.k, a.v, a.beta, a.gate, a.out, n_tasks, a.Hk, a.Hv);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, step_kernel<R, kChannelDecay>, a.state, a.q, a.k, a.v,
                              a.beta, a.gate, a.out, n_tasks, a.Hk, a.Hv);
#else
    step_kernel<R, kChannelDecay><<<grid, threads, 0, stream>>>(a.state, a.q, a.k, a.v, a.beta,
                                                                a.gate, a.out, n_tasks, a.Hk,
                                                                a.Hv);
    return cudaGetLastError();
#endif
}

}  // namespace

cudaError_t launch_step(const StepArgs& a, cudaStream_t stream) {
    return launch_rows<false>(a, stream);
}

cudaError_t launch_kda_step(const StepArgs& a, cudaStream_t stream) {
    return launch_rows<true>(a, stream);
}

cudaError_t launch_pair(const StepArgs& a, float* scratch, cudaStream_t stream) {
    constexpr int R = GDN_STEP_ROWS;
    static_assert(2 * R <= 32, "the batched reduction holds 2 R values");
    const int64_t n_tasks = a.n_heads * (kDv / R);
    if (n_tasks == 0) return cudaSuccess;
    constexpr int threads = GDN_STEP_THREADS;
    constexpr int warps_per_cta = threads / 32;
    const int64_t needed = (n_tasks + warps_per_cta - 1) / warps_per_cta;
    int per_sm = 0;
    cudaError_t err = resident_ctas_per_sm(reinterpret_cast<const void*>(&pair_kernel<R>),
                                           threads, &per_sm);
    if (err != cudaSuccess) return err;
    const int64_t resident = static_cast<int64_t>(device_sm_count()) * per_sm;
    const int grid = static_cast<int>(needed < resident ? needed : resident);
    pair_kernel<R><<<grid, threads, 0, stream>>>(a.state, scratch, a.q, a.k, a.v, a.beta,
                                                 a.gate, a.out, n_tasks, a.Hk, a.Hv);
    return cudaGetLastError();
}

}  // namespace gdn
