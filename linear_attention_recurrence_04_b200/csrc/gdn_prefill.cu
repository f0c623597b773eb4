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
//    that share one key head (h, h + Hk, ...), held in registers: with the
//    scalar decay 4 lanes share a row and each holds a 32-column slice of
//    each of its NH rows, so each k/q value a lane reads serves NH rows; a
//    row's dot products reduce over its 4 lanes with two shuffles. (Eight
//    lanes per row, 16 columns each, doubles the resident warps but measured
//    slower.) The per-channel decay uses the layout of struct Layout below.
//  * Work balance: the warps ("units") are dealt to one CTA per SM in
//    contiguous runs whose lengths differ by at most one, so every SM carries
//    the same number of rows. A run covers at most two (sequence, key head,
//    head group) groups.
//  * Inputs are staged in shared memory S stages of TS positions ahead with
//    16-byte asynchronous copies (cp.async), shared by all warps of the CTA:
//    k and q rows once per group and position, each warp's v rows, beta and
//    gate. The decays exp(gate) of a stage are computed once per warp (one
//    per lane) and broadcast by shuffle. Scalar decay: one loader warp (the
//    CTA's last) issues every copy, and stages pass to the warps with rows
//    through per-stage full/empty mbarriers with bounded waits, with no block
//    barrier in the loop; positions past T are never consumed and are left
//    unwritten. Per-channel decay: every thread issues a share of the copies,
//    positions past T are zero-filled, and block barriers bracket each
//    stage's conversion.
//  * Software pipeline across positions: after the rank-1 update of position
//    t, one pass over the register-resident rows makes both the output dot
//    W.q_t and the next position's key dot W.k_{t+1} (both read the same
//    updated row), and the 4-lane reductions of out_t and sk_{t+1} run as one
//    batch at the top of the next iteration. The dependency chain per
//    position is then: reduce -> scalar delta -> one fused pass. With the
//    scalar decay the next key read by pass t stays in registers as pass
//    t + 1's update vector, so each position reads two staged vectors (its q
//    and the next k) instead of three: the pass is bound by register-operand
//    bandwidth and shared-memory delivery to the lanes, not by the chain.
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
//  * KDA ("Module linear_core", entry "kda_forward_batch"; the published Kimi
//    Delta Attention update) is the same pipeline with a log-decay per key
//    channel, g [B][T][Hv][dk], applied element by element as step 1 reads:
//    the registers hold D = alpha_t (.) M_{t-1}, the state already decayed
//    for the coming position, and pass t runs
//       M = D + delta_t k_t,  o += M.q_t,  D = alpha_{t+1} (.) M,  a += D.k_{t+1},
//    four packed operations per element pair and position. k and q are
//    shared by the two value heads of a warp and k_t is kept in registers
//    from the previous pass, so each position reads q_t, k_{t+1} and each
//    head's alpha_{t+1} from shared memory. The loader warp turns each
//    staged g into alpha = exp(g) once its copies have landed (alpha = 1 past
//    the last position, so the final registers hold M_{T-1}).
#include <type_traits>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_tc.cuh"

#ifndef GDN_PREFILL_STAGES
#define GDN_PREFILL_STAGES 2       // stages in flight (at least 2)
#endif
#ifndef GDN_PREFILL_GDN_LPR
#define GDN_PREFILL_GDN_LPR 4      // scalar decay: lanes per state row (4 or 8)
#endif
#ifndef GDN_PREFILL_EARLY_DECAY
#define GDN_PREFILL_EARLY_DECAY 1  // scalar decay, 4 lanes per row: broadcast each position's
                                   // decays before its reductions (1.553 against 1.586 ms)
#endif
#ifndef GDN_PREFILL_STAGE_FOLD_CHECK
#define GDN_PREFILL_STAGE_FOLD_CHECK 0  // scalar decay, 1: one check per stage of whether the
                                        // running scale can leave its range, the per-position
                                        // check skipped when it cannot (measured slower: the
                                        // branch splits the unrolled positions)
#endif
#ifndef GDN_PREFILL_GDN_HALVING
#define GDN_PREFILL_GDN_HALVING 0  // scalar decay, 4 lanes per row: one halving reduction of
                                   // the A and O values with the deltas broadcast
#endif
#ifndef GDN_PREFILL_GDN_RPL
#define GDN_PREFILL_GDN_RPL 1      // scalar decay: state rows per lane (2 needs 8 lanes per row)
#endif
#ifndef GDN_PREFILL_KREUSE
#define GDN_PREFILL_KREUSE 1       // scalar decay: the next key read by a pass is kept in
                                   // registers as the following pass's update vector
#endif
#ifndef GDN_PREFILL_FMA2
#define GDN_PREFILL_FMA2 1         // packed f32x2 FMAs for the per-element work
#endif
#ifndef GDN_PREFILL_NH
#define GDN_PREFILL_NH 0           // value heads per warp: 0 = 2 when Hv/Hk is even, else 1
#endif
#ifndef GDN_PREFILL_LOADER_WARP
#define GDN_PREFILL_LOADER_WARP 1  // scalar decay: one extra warp issues every stage copy
#endif
#ifndef GDN_PREFILL_MBAR
#define GDN_PREFILL_MBAR 1         // scalar decay: stage handoff through mbarriers, no block barrier
#endif
#ifndef GDN_PREFILL_UNROLL
#define GDN_PREFILL_UNROLL 4       // scalar decay: positions per unrolled block of a stage
#endif
#ifndef GDN_PREFILL_BULK
#define GDN_PREFILL_BULK 1         // scalar decay: the loader's rows as bulk copies
#endif
#ifndef GDN_PREFILL_KDA_LPR
#define GDN_PREFILL_KDA_LPR 8      // per-channel decay: lanes per state row (4 or 8)
#endif
#ifndef GDN_PREFILL_KDA_RPL
#define GDN_PREFILL_KDA_RPL 2      // per-channel decay: state rows per lane (2 needs 8 lanes)
#endif
#ifndef GDN_PREFILL_KDA_UNROLL
#define GDN_PREFILL_KDA_UNROLL 4   // per-channel decay: positions per unrolled block
#endif

namespace gdn {

namespace {

#ifndef GDN_PREFILL_TS
#define GDN_PREFILL_TS 32          // positions per stage (scalar decay)
#endif
constexpr int kTS = GDN_PREFILL_TS;             // positions per stage (scalar decay)
#ifndef GDN_PREFILL_KDA_TS
#define GDN_PREFILL_KDA_TS 20      // positions per stage (per-channel decay)
#endif
#ifndef GDN_PREFILL_KDA_CONVERTER
#define GDN_PREFILL_KDA_CONVERTER 1  // per-channel decay: a second warp shares the alpha conversion
#endif
#ifndef GDN_PREFILL_KDA_LOADER_SHARE
#define GDN_PREFILL_KDA_LOADER_SHARE 0  // per-channel decay: eighths of the alpha conversion
                                        // the loader takes (the converter warp the rest)
#endif
#ifndef GDN_PREFILL_KDA_FASTEXP
#define GDN_PREFILL_KDA_FASTEXP 0  // per-channel decay: alpha by the fast exponential intrinsic
#endif
#ifndef GDN_PREFILL_KDA_STAGES
#define GDN_PREFILL_KDA_STAGES 2   // stages in flight (per-channel decay)
#endif
constexpr int kTSChannel = GDN_PREFILL_KDA_TS;  // positions per stage (per-channel decay)
constexpr int kStages = GDN_PREFILL_STAGES;
template <bool kCh>
constexpr int unroll_for() { return kCh ? GDN_PREFILL_KDA_UNROLL : GDN_PREFILL_UNROLL; }
constexpr int kMaxGroups = 2;                   // groups one CTA's run can touch
constexpr int kMaxRows = 64;                    // rows of one group a CTA holds at most
constexpr float kScaleLo = 0x1p-40f;           // scalar decay: fold-back bounds of the scale
constexpr float kScaleHi = 0x1p40f;
static_assert(kStages >= 2, "at least double buffering");

// Lane layout of a warp's 8 rows. Scalar decay: 4 lanes per row and one row
// per lane, 32 columns each. Per-channel decay: 8 lanes per row group and two
// rows per lane, 16 columns each, so that every staged vector value a lane
// loads serves two rows of each head; that kernel reads a decay vector per
// head besides q and k, and a 16-byte shared load is served a quarter warp
// per wavefront, whatever its broadcast.
template <bool kCh>
struct Layout {
    static constexpr int LPR = kCh ? GDN_PREFILL_KDA_LPR : GDN_PREFILL_GDN_LPR;   // lanes per row
    static constexpr int RPL = kCh ? GDN_PREFILL_KDA_RPL : GDN_PREFILL_GDN_RPL;   // rows per lane
    static constexpr int Chunks = kDk / 4 / LPR;                // float4 chunks per lane and row
    static constexpr int RowsPerUnit = 32 / LPR * RPL;          // rows of a head per warp
    static constexpr int UnitsPerHead = kDv / RowsPerUnit;
    // One more warp, the CTA's last, issues every stage copy. Per-channel
    // decay: a converter warp (the one before it) turns each landed stage's
    // g into alpha. Warps issue on sub-partition warp % 4, so with 7 warps
    // with rows the converter (warp 7) shares the sub-partition that holds
    // only one of them, and the loader (warp 8, bulk copies only) one that
    // holds two (build options: GDN_PREFILL_KDA_LOADER_SHARE, the eighths of
    // the conversion the loader takes; GDN_PREFILL_KDA_CONVERTER=0, the
    // loader alone).
    static constexpr bool Loader = kCh || GDN_PREFILL_LOADER_WARP;
    static constexpr bool Converter = kCh && GDN_PREFILL_KDA_CONVERTER;
    static constexpr int Helpers = (Loader ? 1 : 0) + (Converter ? 1 : 0);   // warps without rows
    static constexpr int MaxWarps = kMaxRows / RowsPerUnit - (Loader ? 1 : 0);  // units per CTA
    static constexpr int Threads = 32 * (MaxWarps + Helpers);
    // One halving reduction of all key and output dots with the deltas
    // broadcast, rather than a full reduction of each on every lane.
    static constexpr bool Halving = LPR == 8 || (!kCh && GDN_PREFILL_GDN_HALVING);
    static_assert(LPR == 4 || LPR == 8, "4 or 8 lanes per row");
    static_assert(Halving || RPL == 1, "two rows per lane use the halving reduction");
    // The key of position t + 1, read by pass t for the next key dot, is the
    // update vector of pass t + 1: kept in registers, it is read from shared
    // memory once instead of twice.
    static constexpr bool KReuse = kCh || GDN_PREFILL_KREUSE;
    static_assert(MaxWarps <= UnitsPerHead, "a run must span at most two groups");
};

// Shared-memory image of one stage. Slot TS of kq (k only) holds the first
// position of the next stage, so a pass always reads the next key from its
// own stage. kCh (per-channel decay) adds al, per value head and position the
// decay alpha = exp(g) (g as copied, then converted in place), with slot TS
// as well; without kCh it is a stub.
template <int NH, bool kCh>
struct alignas(16) Stage {    // stages sit back to back: each starts 16-byte aligned
    static constexpr int TS = kCh ? kTSChannel : kTS;   // positions per stage
    static constexpr int CG = kCh ? kMaxGroups : 1;
    static constexpr int CT = kCh ? TS : 0;
    static constexpr int CD = kCh ? kDk : 4;
    float kq[kMaxGroups][TS + 1][2][kDk];      // [group][pos][k|q][col]
    float v[kMaxGroups][TS][NH][kMaxRows];     // rows [row_lo, row_lo + rows) of the group
    float bg[kMaxGroups][TS][NH][2];           // beta, gate
    float al[CG][CT + 1][NH][CD];              // kCh: alpha of positions t0 .. t0 + TS
};

// Stages in flight.
template <bool kCh>
constexpr int stages_for() { return kCh ? GDN_PREFILL_KDA_STAGES : kStages; }

// One group of the CTA's run: (sequence b, key head g, head group grp) and the
// rows of it that the run covers.
struct Group {
    int64_t b;
    int g;
    int grp;
    int row_lo;
    int rows;
};

// Lane c of a row holds the float4 chunks {LPR i + c}, so one warp-wide
// 16-byte load of k or q touches 16 LPR contiguous bytes.
template <int LPR>
__device__ __forceinline__ int chunk_col(int i, int c) { return 4 * (LPR * i + c); }

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

// d = a * b + c on two lanes of packed floats (one packed f32x2 FMA).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
#if GDN_PREFILL_FMA2
    return __ffma2_rn(a, b, c);
#else
    return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
#endif
}

__device__ __forceinline__ float2 lo2(float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(float4 v) { return make_float2(v.z, v.w); }
__device__ __forceinline__ float4 ld_s4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
#if GDN_PREFILL_FMA2
    return __fmul2_rn(a, b);
#else
    return make_float2(a.x * b.x, a.y * b.y);
#endif
}
// (a.x + b.x) + (a.y + b.y): one packed add and one scalar add.
__device__ __forceinline__ float sum4(float2 a, float2 b) {
#if GDN_PREFILL_FMA2
    const float2 t = __fadd2_rn(a, b);
    return t.x + t.y;
#else
    return (a.x + b.x) + (a.y + b.y);
#endif
}
// 1 / x to within one unit in the last place (PTX rcp.approx.ftz.f32). Used
// for running scales in [2^-40, 2^40], where x and 1 / x are normal.
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

template <int NH, bool kCh>
__global__ void __launch_bounds__(Layout<kCh>::Threads, 1)
prefill_kernel(float* __restrict__ state, const float* __restrict__ q,
               const float* __restrict__ k, const float* __restrict__ v,
               const float* __restrict__ beta, const float* __restrict__ gate,
               float* __restrict__ out, int64_t T, int Hk, int Hv, int units_lo, int n_big,
               int64_t qk_stride, int64_t v_stride, int64_t bg_stride, uint32_t* status) {
    constexpr int S = stages_for<kCh>();
    constexpr int TS = kCh ? kTSChannel : kTS;      // positions per stage
    using StageT = Stage<NH, kCh>;
    constexpr int kLPR = Layout<kCh>::LPR;
    constexpr int kRPL = Layout<kCh>::RPL;
    constexpr int kChunks = Layout<kCh>::Chunks;
    constexpr int kRowsPerUnit = Layout<kCh>::RowsPerUnit;
    constexpr int kUnitsPerHead = Layout<kCh>::UnitsPerHead;
    constexpr bool kHalving = Layout<kCh>::Halving;
    static_assert(sizeof(StageT) % 16 == 0, "16-byte copies and loads need aligned stages");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StageT* stages = reinterpret_cast<StageT*>(smem_raw);
    __shared__ Group grp_of[kMaxGroups];
    // kPipe (a loader warp): stage s is full once the loader's copies of it
    // have landed (and, kCh, its g has become alpha; one arrival per loader
    // lane), and empty again once every warp with rows has finished it.
    constexpr bool kPipe = Layout<kCh>::Loader && (kCh || GDN_PREFILL_MBAR);
    static_assert(!kCh || kPipe, "the per-channel decay runs on the loader-warp pipeline");
    constexpr bool kConverter = Layout<kCh>::Converter;
    __shared__ __align__(8) uint64_t pipe_full[kPipe ? S : 1], pipe_empty[kPipe ? S : 1];
    // kCh: the loader's copies of stage s have landed (one arrival per loader
    // lane); the loader and the converter then each convert half of it and
    // arrive on pipe_full (one arrival per warp).
    __shared__ __align__(8) uint64_t pipe_landed[kCh ? S : 1];

    const int tid = threadIdx.x;
    const int nthreads = blockDim.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int p = lane / kLPR;                  // row group within the warp
    const int c = lane % kLPR;                  // column slice

    // This CTA's run of units: [u0, u0 + count).
    const int cta = blockIdx.x;
    const int64_t u0 = static_cast<int64_t>(cta) * units_lo + (cta < n_big ? cta : n_big);
    const int count = units_lo + (cta < n_big ? 1 : 0);
    const int groups_per_key = (Hv / Hk) / NH;
    const int64_t gid0 = u0 / kUnitsPerHead;
    const int n_groups = static_cast<int>((u0 + count - 1) / kUnitsPerHead - gid0) + 1;
    if (tid < kMaxGroups) {
        const int64_t gid = gid0 + tid;
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
        grp_of[tid] = G;
    }
    if constexpr (kPipe) {
        if (tid == 0) {
            for (int i = 0; i < S; ++i) {
                tc::mbar_init(tc::smem_u32(&pipe_full[i]),
                              kCh ? (kConverter ? 2 : 1) : (GDN_PREFILL_BULK ? 64 : 32));
                // kCh: each loader lane arrives twice, once with the bytes of
                // its bulk copies and once when its 4-byte copies land
                if (kCh) tc::mbar_init(tc::smem_u32(&pipe_landed[i]), 64);
                tc::mbar_init(tc::smem_u32(&pipe_empty[i]), static_cast<uint32_t>(count));
            }
            tc::fence_mbar_init();
        }
    }
    __syncthreads();

    // ---- stage loader: every thread issues a share of the copies; positions
    //      at or past T are zero-filled ------------------------------------
    // With a loader warp (the CTA's last warp), it alone issues the copies.
    constexpr bool kLoaderWarp = Layout<kCh>::Loader;
    const bool is_loader = kLoaderWarp && warp == static_cast<int>(blockDim.x >> 5) - 1;
    const bool is_converter = kConverter && warp == static_cast<int>(blockDim.x >> 5) - 2;
    const int ltid = kLoaderWarp ? lane : tid;
    const int lstride = kLoaderWarp ? 32 : nthreads;
    // The stage's rows (512-byte k and q rows, kCh: g rows, the v rows of the
    // run) as bulk copies that complete on `landed`, beta (and the scalar
    // gate) as 4-byte copies; kCh: alpha slots past the last position get
    // g = 0. The lane then arrives on `landed` twice (with the bytes of its
    // bulk copies, and when its 4-byte copies have landed).
    auto load_stage_bulk = [&](int64_t t0, StageT& st, uint32_t landed) {
        uint32_t bytes = 0;
        for (int gi = 0; gi < n_groups; ++gi) {
            const Group G = grp_of[gi];
            const int kq_items = 2 * TS + 1;              // k of t0 .. t0+TS, q of t0 .. t0+TS-1
            const int g_items = kCh ? (TS + 1) * NH : 0;
            const int v_items = TS * NH;
            const int n_items = kq_items + g_items + v_items;
            for (int it = lane; it < n_items; it += 32) {
                const float* src = nullptr;
                float* dst = nullptr;
                uint32_t size = 0;
                int64_t t = 0;
                if (it < kq_items) {
                    const int tp = it >> 1, which = it & 1;
                    t = t0 + tp;
                    src = (which ? q : k) + (G.b * T + t) * qk_stride + G.g * kDk;
                    dst = &st.kq[gi][tp][which][0];
                    size = kDk * 4;
                } else if (it < kq_items + g_items) {
                    const int j = it - kq_items;
                    const int tp = j / NH, n = j - (j / NH) * NH;
                    t = t0 + tp;
                    const int h = G.g + (G.grp * NH + n) * Hk;
                    src = gate + ((G.b * T + t) * Hv + h) * kDk;
                    dst = &st.al[gi][tp][n][0];
                    size = kDk * 4;
                    if (t >= T) {                         // g = 0: alpha = 1 past the end
                        float4* z = reinterpret_cast<float4*>(dst);
                        for (int c4 = 0; c4 < kDk / 4; ++c4) z[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                } else {
                    const int j = it - kq_items - g_items;
                    const int tp = j / NH, n = j - (j / NH) * NH;
                    t = t0 + tp;
                    const int h = G.g + (G.grp * NH + n) * Hk;
                    src = v + (G.b * T + t) * v_stride + h * kDv + G.row_lo;
                    dst = &st.v[gi][tp][n][0];
                    size = static_cast<uint32_t>(G.rows) * 4;
                }
                if (t < T) {
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
                        "[%0], [%1], %2, [%3];"
                        ::"r"(tc::smem_u32(dst)), "l"(src), "r"(size), "r"(landed) : "memory");
                    bytes += size;
                }
            }
            constexpr int kScalars = kCh ? 1 : 2;                       // beta (, gate)
            for (int idx = lane; idx < TS * NH * kScalars; idx += 32) {
                const int which = idx % kScalars;
                const int n = (idx / kScalars) % NH, tp = idx / (kScalars * NH);
                const int64_t t = t0 + tp;
                if (t < T) {
                    const int h = G.g + (G.grp * NH + n) * Hk;
                    cp_async4(&st.bg[gi][tp][n][which],
                              (which ? gate : beta) + (G.b * T + t) * bg_stride + h);
                }
            }
        }
        tc::mbar_arrive_expect_tx(landed, bytes);
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(landed) : "memory");
    };
    auto load_stage = [&](int64_t t0, StageT& st) {
        if (kLoaderWarp && !is_loader) return;
#pragma unroll
        for (int gi = 0; gi < kMaxGroups; ++gi) {
            if (gi >= n_groups) break;
            const Group G = grp_of[gi];
            for (int idx = ltid; idx < TS * 64 + 32; idx += lstride) {   // k, q rows; k of t0 + TS
                const int chunk = idx & 31;
                const int which = (idx >> 5) & 1;     // the extra slot gets k only
                const int tp = idx >> 6;
                const int64_t t = t0 + tp;
                float* dst = &st.kq[gi][tp][which][chunk * 4];
                if (t < T) {
                    cp_async16(dst, (which ? q : k) + (G.b * T + t) * qk_stride + G.g * kDk + chunk * 4);
                } else if (!kPipe) {
                    *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            const int vchunks = G.rows / 4;                              // v rows
            for (int idx = ltid; idx < TS * NH * vchunks; idx += lstride) {
                const int chunk = idx % vchunks;
                const int n = (idx / vchunks) % NH;
                const int tp = idx / (vchunks * NH);
                const int64_t t = t0 + tp;
                float* dst = &st.v[gi][tp][n][chunk * 4];
                if (t < T) {
                    const int h = G.g + (G.grp * NH + n) * Hk;
                    cp_async16(dst, v + (G.b * T + t) * v_stride + h * kDv + G.row_lo + chunk * 4);
                } else if (!kPipe) {
                    *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            for (int idx = ltid; idx < TS * NH * 2; idx += lstride) {    // beta, gate
                const int which = idx & 1;
                const int n = (idx >> 1) % NH;
                const int tp = (idx >> 1) / NH;
                const int64_t t = t0 + tp;
                float* dst = &st.bg[gi][tp][n][which];
                if (t < T && !(kCh && which)) {
                    const int h = G.g + (G.grp * NH + n) * Hk;
                    cp_async4(dst, (which ? gate : beta) + (G.b * T + t) * bg_stride + h);
                } else if (!kPipe) {
                    *dst = 0.0f;
                }
            }
            if constexpr (kCh) {                                         // g rows
                for (int idx = ltid; idx < (TS + 1) * NH * 32; idx += lstride) {
                    const int chunk = idx & 31;
                    const int n = (idx >> 5) % NH;
                    const int tp = (idx >> 5) / NH;
                    const int64_t t = t0 + tp;
                    float* dst = &st.al[gi][tp][n][chunk * 4];
                    if (t < T) {
                        const int h = G.g + (G.grp * NH + n) * Hk;
                        cp_async16(dst, gate + ((G.b * T + t) * Hv + h) * kDk + chunk * 4);
                    } else {     // g = 0: alpha = 1 past the last position
                        *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
            }
        }
    };
    // kCh: alpha = exp(g) in place, once the loader's copies of the stage have
    // landed: part 0 by the loader warp, part 1 by the converter warp
    auto alpha_stage = [&](StageT& st, int half) {
        if constexpr (kCh) {
            const int n4 = n_groups * (TS + 1) * NH * (kDk / 4);
            const int cut = n4 * GDN_PREFILL_KDA_LOADER_SHARE / 8;
            const int lo = !kConverter ? 0 : half ? cut : 0;
            const int hi = !kConverter ? n4 : half ? n4 : cut;
            float4* a4 = reinterpret_cast<float4*>(&st.al[0][0][0][0]);
            for (int idx = lo + lane; idx < hi; idx += 32) {
                float4 g4 = a4[idx];
#if GDN_PREFILL_KDA_FASTEXP
                g4.x = __expf(g4.x); g4.y = __expf(g4.y); g4.z = __expf(g4.z); g4.w = __expf(g4.w);
#else
                g4.x = expf(g4.x); g4.y = expf(g4.y); g4.z = expf(g4.z); g4.w = expf(g4.w);
#endif
                a4[idx] = g4;
            }
        }
    };

    // ---- this warp's unit ------------------------------------------------
    // Lane (p, c) holds rows j0 + r = rb * 8 + p * kRPL + r (r < kRPL) of
    // the warp's NH value heads, columns chunk_col(i, c). Each position
    // reduces the key dots A and output dots O of its (head, row) pairs over
    // the row group's kLPR lanes.
    //  * Four lanes per row (scalar decay): every lane gets both heads' A and
    //    O (two shuffles each) and forms both deltas; lane c < NH stores head
    //    c's output.
    //  * Eight lanes per row group (kHalving): one halving reduction of all
    //    2 NH kRPL values leaves lane c with the total of value c >> kShift
    //    (values below NH kRPL are the A of pair n kRPL + r, the rest the O of
    //    the same pairs). A lane holding an A forms that pair's delta and the
    //    group broadcasts it; a lane holding an O stores that output.
    const bool active = warp < count;
    const int64_t unit = u0 + warp;
    const int gi = active ? static_cast<int>(unit / kUnitsPerHead - gid0) : 0;
    const Group G = grp_of[gi];
    const int rb = static_cast<int>(unit % kUnitsPerHead);
    const int j0 = rb * kRowsPerUnit + p * kRPL;         // first row within the head
    int hidx[NH];
#pragma unroll
    for (int n = 0; n < NH; ++n) hidx[n] = G.g + (G.grp * NH + n) * Hk;
    constexpr int kPairs = NH * kRPL;                    // (head, row) pairs per lane
    constexpr int kVals = 2 * kPairs;                    // their A and O
    static_assert(!kHalving || kVals <= kLPR, "one reduced value per lane at least");
    constexpr int kShift = (kLPR == 8 ? 3 : 2) - (kVals == 8 ? 3 : kVals == 4 ? 2 : 1);
    const int grp_lane0 = lane & ~(kLPR - 1);
    int my_n = c < NH ? c : 0, my_r = 0;                 // the pair this lane stores
    bool my_store = c < NH;
    if constexpr (kHalving) {
        const int my_val = c >> kShift;
        const int my_pair = my_val < kPairs ? my_val : my_val - kPairs;
        my_n = my_pair / kRPL;
        my_r = my_pair % kRPL;
        my_store = my_val >= kPairs && (c & ((1 << kShift) - 1)) == 0;
    }
    // staged v and beta: kHalving, this lane's pair; otherwise row j0, head 0
    const int my_v_off = kHalving ? my_n * kMaxRows + (j0 + my_r - G.row_lo) : j0 - G.row_lo;
    const int my_b_off = kHalving ? 2 * my_n : 0;
    // The pointer of this lane's output walks the positions (out_next: the
    // coming position, out_prev: the pending one).
    const int64_t out_stride = static_cast<int64_t>(Hv) * kDv;
    float* out_next = out + (G.b * T * Hv + G.g + (G.grp * NH + my_n) * Hk) * kDv + j0 + my_r;
    float* out_prev = out_next;

    // Prologue: request the first S - 1 stages (kPipe: the loader's loop
    // does), then load the state rows.
    const int64_t n_stages = (T + TS - 1) / TS;
    if constexpr (!kPipe) {
#pragma unroll
        for (int s2 = 0; s2 < S - 1; ++s2) {
            if (s2 < n_stages) load_stage(static_cast<int64_t>(s2) * TS, stages[s2]);
            cp_async_commit();
        }
    }

    float4 w[NH][kRPL][kChunks];
    float sc[NH];
    if (active) {
#pragma unroll
        for (int n = 0; n < NH; ++n) {
#pragma unroll
            for (int r = 0; r < kRPL; ++r) {
                const float* row = state + ((G.b * Hv + hidx[n]) * kDv + j0 + r) * kDk;
#pragma unroll
                for (int i = 0; i < kChunks; ++i) w[n][r][i] = ld_stream(row + chunk_col<kLPR>(i, c));
            }
            sc[n] = 1.0f;
        }
    }

    // Loop-carried partial sums: a = W.k of the coming position, o = W.q of
    // the previous position (its store is pending), s_out = its scale.
    float2 a_lo[NH][kRPL], a_hi[NH][kRPL], o_lo[NH][kRPL], o_hi[NH][kRPL];
    float s_out[NH];
#pragma unroll
    for (int n = 0; n < NH; ++n) {
#pragma unroll
        for (int r = 0; r < kRPL; ++r)
            a_lo[n][r] = a_hi[n][r] = o_lo[n][r] = o_hi[n][r] = make_float2(0.f, 0.f);
        s_out[n] = 1.0f;
    }
    bool out_pending = false;
    constexpr bool kKReuse = Layout<kCh>::KReuse;
    float4 kreg[kKReuse ? kChunks : 1];      // kKReuse: this lane's chunks of the coming key

    // One stage's positions for a warp with rows (the stage has landed).
    auto stage_body = [&](int64_t s) {
        const StageT& st = stages[s % S];
        const int64_t t0 = s * TS;
        const int tp_end = (T - t0) < TS ? static_cast<int>(T - t0) : TS;

        // This lane's view of the stage; position tp sits at tp * (stride).
        constexpr int kqP = 2 * kDk;            // k and q of one position
        constexpr int vP = NH * kMaxRows;       // v of one position
        constexpr int bgP = 2 * NH;             // beta, gate of one position
        constexpr int alP = NH * kDk;           // kCh: alpha of one position
        constexpr int kStep = 4 * kLPR;         // columns between a lane's chunks
        const int ccol = kCh ? chunk_col<kLPR>(0, c) : 0;
        const float* kq_s = &st.kq[gi][0][0][chunk_col<kLPR>(0, c)];    // k; q at + kDk
        const float* v_s = &st.v[gi][0][0][0] + my_v_off;      // see my_v_off
        const float* bg_s = &st.bg[gi][0][0][0] + my_b_off;
        const float* al_s = &st.al[gi * kCh][0][0][ccol];     // kCh only

        // decays of this stage: lane tp holds exp(gate) of position tp for
        // each head (stages of at most 32 positions)
        static_assert(kCh || TS <= 32, "one lane per position of a stage");
        float e_lane[NH];
#pragma unroll
        for (int n = 0; n < NH; ++n)
            e_lane[n] = (!kCh && lane < TS) ? expf(st.bg[gi][lane % TS][n][1]) : 1.0f;
        // Scalar decay: whether the running scale can leave its range within
        // this stage. Without a fold every prefix product of the stage's
        // decays lies between the product of their parts below 1 and the
        // product of their parts above 1; with a factor-2 margin for rounding,
        // a stage whose bounds stay inside needs no per-position check (and
        // no position of it would fold: the results are the same).
        bool may_fold = true;
        if constexpr (!kCh && GDN_PREFILL_STAGE_FOLD_CHECK) {
            may_fold = false;
#pragma unroll
            for (int n = 0; n < NH; ++n) {
                float lo = fminf(e_lane[n], 1.0f), hi = fmaxf(e_lane[n], 1.0f);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    lo *= __shfl_xor_sync(kFull, lo, off);
                    hi *= __shfl_xor_sync(kFull, hi, off);
                }
                may_fold |= !(sc[n] * lo >= 2.0f * kScaleLo && sc[n] * hi <= 0.5f * kScaleHi);
            }
        }

        if (s == 0) {
            // first key dot: a = W.k_0 (kCh: first the decay of position 0,
            // D = alpha_0 (.) M, then a = D.k_0)
#pragma unroll
            for (int i = 0; i < kChunks; ++i) {
                const float4 kv = ld_s4(kq_s + kStep * i);
                if constexpr (kKReuse) kreg[i] = kv;
#pragma unroll
                for (int n = 0; n < NH; ++n) {
                    if constexpr (kCh) {
                        const float4 al = ld_s4(al_s + n * kDk + kStep * i);
#pragma unroll
                        for (int r = 0; r < kRPL; ++r) {
                            const float2 l = mul2(lo2(w[n][r][i]), lo2(al));
                            const float2 h = mul2(hi2(w[n][r][i]), hi2(al));
                            w[n][r][i] = make_float4(l.x, l.y, h.x, h.y);
                        }
                    }
#pragma unroll
                    for (int r = 0; r < kRPL; ++r) {
                        a_lo[n][r] = fma2(lo2(w[n][r][i]), lo2(kv), a_lo[n][r]);
                        a_hi[n][r] = fma2(hi2(w[n][r][i]), hi2(kv), a_hi[n][r]);
                    }
                }
            }
        }

        // The positions of the stage.
        auto positions = [&]() {
#pragma unroll(unroll_for<kCh>())
            for (int tp = 0; tp < TS; ++tp) {
                if (tp >= tp_end) break;
                float cf[NH][kRPL];
                if constexpr (!kHalving) {
                    // this position's decays, broadcast first (their shuffles
                    // overlap the reductions' below)
                    [[maybe_unused]] float e_t[NH];
#if GDN_PREFILL_EARLY_DECAY
                    if constexpr (!kCh) {
#pragma unroll
                        for (int n = 0; n < NH; ++n) e_t[n] = __shfl_sync(kFull, e_lane[n], tp);
                    }
#endif
                    // (a) batched reductions: sk of t, and out of t-1
                    float A[NH], O[NH];
#pragma unroll
                    for (int n = 0; n < NH; ++n) {
                        A[n] = sum4(a_lo[n][0], a_hi[n][0]);
                        O[n] = sum4(o_lo[n][0], o_hi[n][0]);
                    }
#pragma unroll
                    for (int n = 0; n < NH; ++n) {
                        A[n] = group_sum<kLPR>(A[n]);
                        O[n] = group_sum<kLPR>(O[n]);
                    }
                    {   // lane c < NH stores head c's output of t - 1
                        float ov = O[0], so = s_out[0];
#pragma unroll
                        for (int n = 1; n < NH; ++n)
                            if (c == n) { ov = O[n]; so = s_out[n]; }
                        if (out_pending && my_store) *out_prev = so * ov * kOutScale;
                    }
                    if constexpr (kCh) {     // the state is held unscaled: A is sk
#pragma unroll
                        for (int n = 0; n < NH; ++n)
                            cf[n][0] = (v_s[tp * vP + n * kMaxRows] - A[n]) * bg_s[tp * bgP + 2 * n];
                    } else {
                    // (b) step 1 as a scale update s *= e; then, with
                    // r = 1 / s, delta / s = (v r - W.k) beta (steps 2-3)
                    float s_new[NH];
                    bool fold = false;
#pragma unroll
                    for (int n = 0; n < NH; ++n)
#if GDN_PREFILL_EARLY_DECAY
                        s_new[n] = sc[n] * e_t[n];
#else
                        s_new[n] = sc[n] * __shfl_sync(kFull, e_lane[n], tp);
#endif
                    if (may_fold) {      // uniform across the warp
#pragma unroll
                        for (int n = 0; n < NH; ++n)
                            fold |= !(s_new[n] >= kScaleLo && s_new[n] <= kScaleHi);
                    }
                    if (fold) {          // rare, and uniform across the warp
#pragma unroll
                        for (int n = 0; n < NH; ++n) {
                            if (!(s_new[n] >= kScaleLo && s_new[n] <= kScaleHi)) {
#pragma unroll
                                for (int i = 0; i < kChunks; ++i) {
                                    w[n][0][i].x *= s_new[n]; w[n][0][i].y *= s_new[n];
                                    w[n][0][i].z *= s_new[n]; w[n][0][i].w *= s_new[n];
                                }
                                A[n] *= s_new[n];
                                s_new[n] = 1.0f;
                            }
                        }
                    }
#pragma unroll
                    for (int n = 0; n < NH; ++n) {
                        sc[n] = s_new[n];
                        s_out[n] = s_new[n];
                        cf[n][0] = fmaf(v_s[tp * vP + n * kMaxRows], rcp_approx(s_new[n]), -A[n]) *
                                   bg_s[tp * bgP + 2 * n];
                    }
                    }
                } else {
                    // (a) one halving reduction: sk of t and out of t-1 for
                    // every pair
                    float vals[kVals];
#pragma unroll
                    for (int n = 0; n < NH; ++n) {
#pragma unroll
                        for (int r = 0; r < kRPL; ++r) {
                            vals[n * kRPL + r] = sum4(a_lo[n][r], a_hi[n][r]);
                            vals[kPairs + n * kRPL + r] = sum4(o_lo[n][r], o_hi[n][r]);
                        }
                    }
                    float tot = group_sum_many<kVals, kLPR>(vals, lane);
                    float so = s_out[0];
#pragma unroll
                    for (int n = 1; n < NH; ++n)
                        if (my_n == n) so = s_out[n];
                    if (out_pending && my_store) *out_prev = so * tot * kOutScale;
                    // (b) this lane's pair's delta, then the broadcast
                    float cf_mine;
                    if constexpr (kCh) {
                        // the state is held unscaled: tot is sk
                        cf_mine = (v_s[tp * vP] - tot) * bg_s[tp * bgP];
                    } else {
                        // step 1 as a scale update s *= e (every lane keeps
                        // both heads' scales); then, with r = 1 / s,
                        // delta / s = (v r - W.k) beta (steps 2-3)
                        float s_new[NH];
                        bool fold = false;
#pragma unroll
                        for (int n = 0; n < NH; ++n)
                            s_new[n] = sc[n] * __shfl_sync(kFull, e_lane[n], tp);
                        if (may_fold) {  // uniform across the warp
#pragma unroll
                            for (int n = 0; n < NH; ++n)
                                fold |= !(s_new[n] >= kScaleLo && s_new[n] <= kScaleHi);
                        }
                        if (fold) {      // rare, and uniform across the warp
#pragma unroll
                            for (int n = 0; n < NH; ++n) {
                                if (!(s_new[n] >= kScaleLo && s_new[n] <= kScaleHi)) {
#pragma unroll
                                    for (int r = 0; r < kRPL; ++r) {
#pragma unroll
                                        for (int i = 0; i < kChunks; ++i) {
                                            w[n][r][i].x *= s_new[n]; w[n][r][i].y *= s_new[n];
                                            w[n][r][i].z *= s_new[n]; w[n][r][i].w *= s_new[n];
                                        }
                                    }
                                    if (my_n == n) tot *= s_new[n];
                                    s_new[n] = 1.0f;
                                }
                            }
                        }
                        float s_mine = s_new[0];
#pragma unroll
                        for (int n = 0; n < NH; ++n) {
                            sc[n] = s_new[n];
                            s_out[n] = s_new[n];
                            if (my_n == n) s_mine = s_new[n];
                        }
                        cf_mine = fmaf(v_s[tp * vP], rcp_approx(s_mine), -tot) * bg_s[tp * bgP];
                    }
#pragma unroll
                    for (int n = 0; n < NH; ++n) {
#pragma unroll
                        for (int r = 0; r < kRPL; ++r)
                            cf[n][r] = __shfl_sync(kFull, cf_mine,
                                                   grp_lane0 + ((n * kRPL + r) << kShift));
                    }
                }
                // (c) one pass: step 4 for t, then W.q_t (step 5) and the next
                // position's key dot; kCh: the next position's decay (step 1)
                // between the two, D = alpha_{t+1} (.) M. Slot tp + 1 always
                // exists (kCh: alpha = 1 past the last position).
                const float* kp = kq_s + tp * kqP;
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    float4 kv_sh;
                    if constexpr (kKReuse) kv_sh = kreg[i];
                    else kv_sh = ld_s4(kp + kStep * i);
                    const float4 qv = ld_s4(kp + kDk + kStep * i);
                    const float4 nv = ld_s4(kp + kqP + kStep * i);
                    if constexpr (kKReuse) kreg[i] = nv;
#pragma unroll
                    for (int n = 0; n < NH; ++n) {
                        [[maybe_unused]] float4 al;
                        if constexpr (kCh) al = ld_s4(al_s + (tp + 1) * alP + n * kDk + kStep * i);
#pragma unroll
                        for (int r = 0; r < kRPL; ++r) {
                            const float4 wv = w[n][r][i];
                            const float2 cf2 = make_float2(cf[n][r], cf[n][r]);
                            const float2 lo = fma2(cf2, lo2(kv_sh), lo2(wv));
                            const float2 hi = fma2(cf2, hi2(kv_sh), hi2(wv));
                            float2 dlo = lo, dhi = hi;
                            if constexpr (kCh) {
                                dlo = mul2(lo, lo2(al));
                                dhi = mul2(hi, hi2(al));
                            }
                            w[n][r][i] = make_float4(dlo.x, dlo.y, dhi.x, dhi.y);
                            if (i == 0) {
                                o_lo[n][r] = mul2(lo, lo2(qv));
                                o_hi[n][r] = mul2(hi, hi2(qv));
                                a_lo[n][r] = mul2(dlo, lo2(nv));
                                a_hi[n][r] = mul2(dhi, hi2(nv));
                            } else {
                                o_lo[n][r] = fma2(lo, lo2(qv), o_lo[n][r]);
                                o_hi[n][r] = fma2(hi, hi2(qv), o_hi[n][r]);
                                a_lo[n][r] = fma2(dlo, lo2(nv), a_lo[n][r]);
                                a_hi[n][r] = fma2(dhi, hi2(nv), a_hi[n][r]);
                            }
                        }
                    }
                }
                out_pending = true;
                out_prev = out_next;
                out_next += out_stride;
            }
        };
        positions();
    };

    if constexpr (kPipe) {
        // The loader fills stage si once its slot is empty; each warp with
        // rows waits for its stage to fill and frees it after its positions.
        // Every wait is bounded: on a timeout the warp stops and reports.
        bool timed_out = false;
        if (is_loader) {
            for (int64_t si = 0; si < n_stages; ++si) {
                const int slot = static_cast<int>(si % S);
                if (si >= S && !tc::mbar_wait(tc::smem_u32(&pipe_empty[slot]),
                                              static_cast<uint32_t>((si / S - 1) & 1))) {
                    timed_out = true;
                    break;
                }
                if constexpr (kCh) {
                    // the copies land on pipe_landed; then this warp converts
                    // its part of the stage (all of it without a converter
                    // warp) and publishes it
                    load_stage_bulk(si * TS, stages[slot], tc::smem_u32(&pipe_landed[slot]));
                    __syncwarp();                  // the zero-filled alpha slots
                    if (!tc::mbar_wait(tc::smem_u32(&pipe_landed[slot]),
                                       static_cast<uint32_t>((si / S) & 1))) {
                        // give the copies in flight one more bounded wait
                        // before this CTA can leave
                        tc::mbar_wait(tc::smem_u32(&pipe_landed[slot]),
                                      static_cast<uint32_t>((si / S) & 1));
                        timed_out = true;
                        break;
                    }
                    alpha_stage(stages[slot], 0);
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(tc::smem_u32(&pipe_full[slot]));
                } else if constexpr (GDN_PREFILL_BULK != 0) {
                    load_stage_bulk(si * TS, stages[slot], tc::smem_u32(&pipe_full[slot]));
                } else {
                    load_stage(si * TS, stages[slot]);
                    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];"
                                 ::"r"(tc::smem_u32(&pipe_full[slot])) : "memory");
                }
            }
            asm volatile("cp.async.wait_all;" ::: "memory");   // nothing left in flight
        } else if (is_converter) {
            // kCh: the converter's part of every stage, once its copies have landed
            for (int64_t si = 0; si < n_stages; ++si) {
                const int slot = static_cast<int>(si % S);
                if (!tc::mbar_wait(tc::smem_u32(&pipe_landed[slot]),
                                   static_cast<uint32_t>((si / S) & 1))) {
                    timed_out = true;
                    break;
                }
                alpha_stage(stages[slot], 1);
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(tc::smem_u32(&pipe_full[slot]));
            }
        } else if (active) {
            for (int64_t s = 0; s < n_stages; ++s) {
                const int slot = static_cast<int>(s % S);
                if (!tc::mbar_wait(tc::smem_u32(&pipe_full[slot]),
                                   static_cast<uint32_t>((s / S) & 1))) {
                    timed_out = true;
                    break;
                }
                stage_body(s);
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(tc::smem_u32(&pipe_empty[slot]));
            }
        }
        if (timed_out && status != nullptr && lane == 0) atomicOr(status, tc::kTimeoutPrefill);
    } else {
        for (int64_t s = 0; s < n_stages; ++s) {
            cp_async_wait<S - 2>();             // this thread's copies of stage s landed
            __syncthreads();                     // ... and everyone's; stage s-1 is consumed
            {
                const int64_t nxt = s + S - 1;
                if (nxt < n_stages) load_stage(nxt * TS, stages[nxt % S]);
                cp_async_commit();
            }
            if (!active) continue;
            stage_body(s);
        }
        cp_async_wait<0>();
    }

    if (active) {
        // the last position's output
        if (out_pending) {
            if constexpr (!kHalving) {
                float ov = 0.0f, so = s_out[0];
#pragma unroll
                for (int n = 0; n < NH; ++n) {
                    const float O = group_sum<kLPR>(sum4(o_lo[n][0], o_hi[n][0]));
                    if (c == n) { ov = O; so = s_out[n]; }
                }
                if (my_store) *out_prev = so * ov * kOutScale;
            } else {
                float vals[kVals];
#pragma unroll
                for (int n = 0; n < NH; ++n) {
#pragma unroll
                    for (int r = 0; r < kRPL; ++r) {
                        vals[n * kRPL + r] = 0.0f;
                        vals[kPairs + n * kRPL + r] = sum4(o_lo[n][r], o_hi[n][r]);
                    }
                }
                const float tot = group_sum_many<kVals, kLPR>(vals, lane);
                float so = s_out[0];
#pragma unroll
                for (int n = 1; n < NH; ++n)
                    if (my_n == n) so = s_out[n];
                if (my_store) *out_prev = so * tot * kOutScale;
            }
        }
        // the final state (scalar decay: with the scale folded in; kCh: the
        // registers hold M_{T-1}, decayed by alpha = 1)
#pragma unroll
        for (int n = 0; n < NH; ++n) {
#pragma unroll
            for (int r = 0; r < kRPL; ++r) {
                float* row = state + ((G.b * Hv + hidx[n]) * kDv + j0 + r) * kDk;
#pragma unroll
                for (int i = 0; i < kChunks; ++i) {
                    float4 x = w[n][r][i];
                    if constexpr (!kCh) {
                        x.x *= sc[n]; x.y *= sc[n]; x.z *= sc[n]; x.w *= sc[n];
                    }
                    st_stream(row + chunk_col<kLPR>(i, c), x);
                }
            }
        }
    }
}

template <int NH, bool kCh>
cudaError_t launch_nh(const PrefillArgs& a, cudaStream_t stream) {
    const int G = a.Hv / a.Hk;
    using L = Layout<kCh>;
    const int64_t n_units = a.B * a.Hk * (G / NH) * L::UnitsPerHead;
    if (n_units == 0) return cudaSuccess;
    const int64_t sms = device_sm_count();
    int64_t grid = n_units < sms ? n_units : sms;
    const int64_t min_grid = (n_units + L::MaxWarps - 1) / L::MaxWarps;
    if (grid < min_grid) grid = min_grid;
    const int units_lo = static_cast<int>(n_units / grid);
    const int n_big = static_cast<int>(n_units % grid);
    const int warps = units_lo + (n_big > 0 ? 1 : 0) + L::Helpers;
    const size_t smem = sizeof(Stage<NH, kCh>) * stages_for<kCh>();
    cudaError_t err = cudaFuncSetAttribute(prefill_kernel<NH, kCh>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int64_t qk_stride = a.qk_stride ? a.qk_stride : static_cast<int64_t>(a.Hk) * kDk;
    const int64_t v_stride = a.v_stride ? a.v_stride : static_cast<int64_t>(a.Hv) * kDv;
    const int64_t bg_stride = a.bg_stride ? a.bg_stride : a.Hv;
    prefill_kernel<NH, kCh><<<static_cast<unsigned>(grid), 32 * warps, smem, stream>>>(
        a.state, a.q, a.k, a.v, a.beta, a.gate, a.out, a.T, a.Hk, a.Hv, units_lo, n_big,
        qk_stride, v_stride, bg_stride, a.status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const int G = a.Hv / a.Hk;
    const bool two = GDN_PREFILL_NH == 0 ? (G % 2 == 0) : (GDN_PREFILL_NH == 2 && G % 2 == 0);
    return two ? launch_nh<2, false>(a, stream) : launch_nh<1, false>(a, stream);
}

cudaError_t launch_kda_prefill(const PrefillArgs& a, cudaStream_t stream) {
    const int G = a.Hv / a.Hk;
    return (G % 2 == 0) ? launch_nh<2, true>(a, stream) : launch_nh<1, true>(a, stream);
}

}  // namespace gdn
