// gdn_linear.cu -- dense projection y[M][N] (fp32) = x[M][K] (bf16) . W[N][K]^T
// (bf16) on the sm_100a tensor cores.
//
// These are the layer's input and output projections ("Red Lite dev15e --
// complete recurrent DeltaNet layer composition", opening list: attn_qkv
// 2048 -> 8192, attn_gate 2048 -> 4096, ssm_ba 2048 -> 64, ssm_out 4096 ->
// 2048), here with dense bf16 weights; "Module linear_core", entry
// "gdn_forward_batch", runs them as matrix-matrix products over a batch of
// positions.
//
// Design (persistent: one CTA per SM walks BM x BN output tiles, 192
// threads). The tile is the widest of 256 x 256, 128 x 256, 128 x 128 and
// 128 x 64 whose count still covers every SM once: wide tiles take in fewer
// bytes per MMA through TMA (which bounds this kernel), narrow ones let a
// decode-sized product spread its weight stream over more SMs.
//   warp 0      one thread issues TMA loads of BM x 64 tiles of x and BN x 64
//               tiles of W (128-byte swizzle) into an S-stage shared-memory
//               ring that runs on across tiles;
//   warp 1      owns the TMEM accumulators -- two sets of BN fp32 columns for
//               128-row tiles, one set of 2 x 256 for 256-row tiles (TMEM
//               holds 512 columns); one thread issues tcgen05.mma (bf16,
//               M = 128, N = BN, K = 16) per 32-byte K step, one per 128-row
//               half of the tile; a tcgen05.commit per stage frees the slot
//               back to the producer, one per tile hands the set to the
//               epilogue;
//   warps 2-5   read an accumulator set with tcgen05.ld (warp w its TMEM lane
//               quarter w % 4), store fp32 rows and release the set: with two
//               sets, tile i drains while the MMAs of tile i+1 fill the other.
// Tiles past M, N or K are zero-filled by TMA and masked on store. An
// element's K order never depends on the tile width, the tile's place or M,
// so a row's result is the same in any batch.
//
// Two more forms follow the persistent kernel: the pair-CTA kernel
// (cta_group::2, one 256 x 256 tile per pair of SMs) that products with
// enough such tiles take -- same K order, same rows -- and the split-K
// cluster kernel for calls of at most 128 rows (its own fixed K grouping). Every mbarrier wait gives up
// after 2 s, ORs an error bit into the caller's status word (if given), lets
// in-flight copies land and frees TMEM.
//
// Both kernels are launched with programmatic stream serialization: barrier
// setup, TMEM allocation and an L2 prefetch of the weight boxes overlap the
// tail of the previous kernel on the stream; every thread waits for that
// kernel (griddepcontrol.wait) before its first global read or write or
// bounded wait, and each CTA releases the next kernel once set up.
#include <cuda.h>
#include <cuda_bf16.h>

#include <unistd.h>

#include <algorithm>
#include <atomic>
#include <chrono>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_tc.cuh"

// Tile shape: 0 chooses per launch; 64, 128 or 256 force 128 x that width;
// 512 forces 256 x 256.
#ifndef GDN_LINEAR_BN
#define GDN_LINEAR_BN 0
#endif
// Split-K form: k-steps of each CTA's weight stripe prefetched into L2 before
// the dependency wait (-1: all of them). The first two measured best: the
// whole stripe of every CTA at once queues the first stages behind it
// (short-conv decode 22.2 against 21.2 us).
#ifndef GDN_SPLIT_PREFETCH
#define GDN_SPLIT_PREFETCH 2
#endif
// 1: products with enough 256 x 256 tiles take the pair-CTA (cta_group::2) form.
#ifndef GDN_LINEAR_PAIR
#define GDN_LINEAR_PAIR 1
#endif

namespace gdn {

namespace {

constexpr int kMmaM = 128;               // rows of one tcgen05.mma (cta_group::1)
constexpr int kBK = 64;                  // 64 bf16 = one 128-byte swizzle row
constexpr int kEpilogueWarps = 4;        // one per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpilogueWarps;

// Shared-memory ring for a BM x BN tile: as many stages of (BM + BN) rows of
// 128 bytes as fit 192 KB, at most 8 -- 3 of 64 KB (256 x 256), 4 of 48 KB
// (128 x 256), 6 of 32 KB (128 x 128), 8 of 24 KB (128 x 64).
template <int BN, int BM>
struct LinearSmem {
    static constexpr uint32_t kA = BM * kBK * 2;
    static constexpr uint32_t kB = BN * kBK * 2;
    static constexpr uint32_t kStage = kA + kB;
    static constexpr int kStages = (196608 / kStage) < 8 ? static_cast<int>(196608 / kStage) : 8;
    static constexpr size_t kDynamic = static_cast<size_t>(kStage) * kStages + 1024;
};

// A tile of BM = 128 or 256 rows: with 256, two M = 128 MMAs per K step share
// each B tile, so every byte the SM takes in through TMA feeds more MMA work
// (the per-SM TMA intake, not the tensor pipe, bounds this kernel).
template <int BN, int BM>
__global__ void __launch_bounds__(kThreads, 1)
linear_bf16_kernel(const __grid_constant__ CUtensorMap tmap_x,
                   const __grid_constant__ CUtensorMap tmap_w, float* __restrict__ y, int M,
                   int N, int K, uint32_t* __restrict__ status) {
    using L = LinearSmem<BN, BM>;
    constexpr int kStages = L::kStages;
    constexpr int kHalves = BM / kMmaM;                     // MMAs per K step
    constexpr uint32_t kAccCols = kHalves * BN;             // one tile's accumulators
    constexpr int kNumAcc = 2 * kAccCols <= 512 ? 2 : 1;    // tiles in flight in TMEM
    static_assert(BM == 128 || BM == 256, "tile rows");
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages];
    __shared__ __align__(8) uint64_t empty[kStages];
    __shared__ __align__(8) uint64_t acc_full[2];      // MMA -> epilogue, per accumulator
    __shared__ __align__(8) uint64_t acc_empty[2];     // epilogue -> MMA
    __shared__ uint32_t tmem_slot;
    __shared__ int64_t issued, consumed;
    __shared__ int failed;

    // 1024-byte aligned base for the swizzled tiles
    const uint32_t raw = tc::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_kt = (K + kBK - 1) / kBK;
    const int tiles_n = (N + BN - 1) / BN;
    const int n_tiles = tiles_n * ((M + BM - 1) / BM);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(tc::smem_u32(&full[s]), 1);
            tc::mbar_init(tc::smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(tc::smem_u32(&acc_full[a]), 1);
            tc::mbar_init(tc::smem_u32(&acc_empty[a]), kEpilogueWarps);   // one per epilogue warp
        }
        tc::fence_mbar_init();
        issued = 0;
        consumed = 0;
        failed = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_u32(&tmem_slot), kNumAcc * kAccCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    volatile int* vfailed = &failed;
    tc::grid_dep_launch();

    if (warp == 0 && lane == 0) {
        // ---- producer: k-steps of every tile, through the stage ring --------
        tc::prefetch_tmap(&tmap_x);
        tc::prefetch_tmap(&tmap_w);
        // the first tile's weight boxes head for L2 while the previous kernel
        // on the stream finishes
        if (static_cast<int>(blockIdx.x) < n_tiles) {
            const int n0 = (static_cast<int>(blockIdx.x) % tiles_n) * BN;
            for (int kt = 0; kt < n_kt && kt < kStages; ++kt)
                tc::tma_prefetch_l2_2d(&tmap_w, kt * kBK, n0);
        }
        tc::grid_dep_wait();
        int64_t g = 0;                                     // k-steps issued so far
        for (int tile = blockIdx.x; tile < n_tiles && !*vfailed; tile += gridDim.x) {
            const int m0 = (tile / tiles_n) * BM;
            const int n0 = (tile % tiles_n) * BN;
            for (int kt = 0; kt < n_kt; ++kt, ++g) {
                const int s = static_cast<int>(g % kStages);
                const uint32_t ph = static_cast<uint32_t>(g / kStages) & 1u;
                if (!tc::mbar_wait(tc::smem_u32(&empty[s]), ph ^ 1)) {
                    if (status) atomicOr(status, tc::kTimeoutProducer);
                    atomicExch(&failed, 1);
                    break;
                }
                if (*vfailed) break;
                const uint32_t a = base + s * L::kStage;
                tc::mbar_arrive_expect_tx(tc::smem_u32(&full[s]), L::kStage);
                tc::tma_load_2d(a, &tmap_x, tc::smem_u32(&full[s]), kt * kBK, m0);
                tc::tma_load_2d(a + L::kA, &tmap_w, tc::smem_u32(&full[s]), kt * kBK, n0);
                issued = g + 1;
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer: tile li accumulates into accumulator set li % kNumAcc
        tc::grid_dep_wait();                       // bounded waits start from here
        const uint32_t idesc = tc::idesc_bf16_f32(kMmaM, BN);
        int64_t g = 0;
        bool ok = true;
        int li = 0;
        for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++li) {
            const int acc = li % kNumAcc;
            const int use = li / kNumAcc;                  // this set's earlier uses
            const uint32_t d = tmem + static_cast<uint32_t>(acc) * kAccCols;
            if (!tc::mbar_wait(tc::smem_u32(&acc_empty[acc]), (use & 1) ^ 1) || *vfailed) {
                if (status) atomicOr(status, tc::kTimeoutMma);
                atomicExch(&failed, 1);
                break;
            }
            tc::tc_fence_after();
            for (int kt = 0; kt < n_kt; ++kt, ++g) {
                const int s = static_cast<int>(g % kStages);
                const uint32_t ph = static_cast<uint32_t>(g / kStages) & 1u;
                if (!tc::mbar_wait(tc::smem_u32(&full[s]), ph) || *vfailed) {
                    if (status) atomicOr(status, tc::kTimeoutMma);
                    atomicExch(&failed, 1);
                    ok = false;
                    break;
                }
                consumed = g + 1;
                tc::tc_fence_after();
                const uint32_t a = base + s * L::kStage;
                const uint32_t b = a + L::kA;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
                    for (int hf = 0; hf < kHalves; ++hf) {   // rows [128 hf, 128 hf + 128)
                        tc::mma_bf16(d + hf * BN,
                                     tc::desc_k_sw128(a + hf * (kMmaM * kBK * 2) + kk * 32),
                                     tc::desc_k_sw128(b + kk * 32), idesc,
                                     (kt > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc::mma_commit(tc::smem_u32(&empty[s]));   // slot free once these MMAs finish
            }
            if (ok) tc::mma_commit(tc::smem_u32(&acc_full[acc]));   // accumulator complete
        }
    } else if (warp >= 2) {
        // ---- epilogue: TMEM -> registers -> global, then release ------------
        tc::grid_dep_wait();
        const int quarter = warp & 3;                      // TMEM lanes 32 q .. 32 q + 31
        int li = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++li) {
            const int acc = li % kNumAcc;
            if (!tc::mbar_wait(tc::smem_u32(&acc_full[acc]), (li / kNumAcc) & 1) || *vfailed) {
                if (status) atomicOr(status, tc::kTimeoutEpilogue);
                atomicExch(&failed, 1);
                break;
            }
            tc::tc_fence_after();
            const int m0 = (tile / tiles_n) * BM;
            const int n0 = (tile % tiles_n) * BN;
#pragma unroll 1
            for (int hf = 0; hf < kHalves; ++hf) {
                const int row = m0 + hf * kMmaM + quarter * 32 + lane;
                const bool row_ok = row < M;
                float* yrow = y + static_cast<int64_t>(row) * N;
                const uint32_t src = tmem + static_cast<uint32_t>(acc) * kAccCols + hf * BN +
                                     (static_cast<uint32_t>(quarter * 32) << 16);
    #pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    uint32_t r[32];
                    tc::tmem_ld_32x32b_x32(src + c0, r);
                    tc::tmem_ld_wait();
                    const int col = n0 + c0;
                    if (!row_ok || col >= N) continue;
                    if (col + 32 <= N && (N & 3) == 0) {
    #pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            *reinterpret_cast<float4*>(yrow + col + j) =
                                make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                            __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                        }
                    } else {
    #pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (col + j < N) yrow[col + j] = __uint_as_float(r[j]);
                    }
                }
            }
            // every read of this accumulator set has completed: hand it back
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tc::smem_u32(&acc_empty[acc]));
        }
    }

    // On failure, let copies that were issued but never consumed land before
    // the shared memory goes away (bounded like every other wait).
    __syncthreads();
    if (threadIdx.x == 0 && failed) {
        for (int64_t g = consumed; g < issued; ++g)
            tc::mbar_wait(tc::smem_u32(&full[g % kStages]),
                          static_cast<uint32_t>(g / kStages) & 1u);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 1) tc::tmem_dealloc(tmem, kNumAcc * kAccCols);
}

// Split-K form for products of at most 128 rows (decode-sized calls).
//
// With few rows the persistent kernel's cost is one CTA's K/16 MMA
// instructions (32 k-steps x 4 for K = 2048), each about 87 ns of issue
// whatever the tile's width or rows (interleaved accumulators do not shorten
// it), and only N / BN SMs stream the weights. Here a cluster of `splits` CTAs shares
// one 128 x BN output tile: CTA r runs k-steps [r n_kt / S, (r+1) n_kt / S)
// into its own TMEM accumulator, parks the fp32 partial tile in its (then
// idle) stage ring, and after a cluster barrier every CTA sums a 1/S slice of
// the tile over the S partials through distributed shared memory, always in
// rank order 0, 1, .., S-1, and stores it. The split depends on (N, K) and the
// device alone, so a row's result is the same in any call of at most 128
// rows; it differs from the persistent kernel's by the fp32 rounding of the
// grouped sum.
//
// kGate = 2, 3 or 4 (conv taps): the short-conv mixer's input projection with
// its gate and conv as the epilogue. A tile is 64 channels d0.. of the three
// row blocks of W_in (bg | cg | xv), loaded as three 64-row boxes into one
// 192-row B tile (N = 192, M = rows of the call). After the cluster barrier
// CTA r takes the channel quads [16 r / S, 16 (r+1) / S) of the tile: it sums
// bg, cg, xv over the S partials (rank order), forms u = bg * xv in fp32 and
// keeps u and cg in its own shared memory; after a second cluster barrier one
// thread per (sequence, channel) walks the call's positions through the conv
// window -- the ring before position 0, u after -- exactly as the mixer's
// gate kernel does (window sum and output gate in double, y rounded to bf16
// once) and writes y and both rings.
// Gate mode: the ring entries and conv taps of the CTA's channels are read
// into shared memory past the stage ring while the main loop runs (they do not
// depend on the product), so the conv walk after the reduction reads no
// global memory. Used when the CTA's share fits kRingCache bytes.
constexpr size_t kRingCache = 16384;
constexpr size_t kTapCache = 32 * 4 * 4;          // at most 32 channels x 4 taps

//
// kFuse (gate mode, one or two positions, every channel tile's conv ring in
// shared memory): the whole mixer in one kernel. The output projection
// out = y W_out^T is split exactly as the split-K form splits it on its own
// (64-column tiles, the same K chunks, the same rank-order reduction), so
// its bits are those of the two-kernel path: CTA r of cluster c owns output
// columns [64 c, 64 c + 64) and y channels of the k-steps it owned in the
// input projection. Its W_out chunks stream into shared memory as soon as
// the input projection's MMAs are done (into the freed stage ring and a
// region past the ring cache), while the partials are reduced and the conv
// walked. Every CTA's y (all channels of every sequence) is written before
// any CTA reads it: after the walk one thread per CTA passes a grid-wide
// barrier (a tagged counter in the caller's workspace, every wait bounded),
// then loads the CTA's y chunks with TMA into the freed ring; the MMAs run
// as each chunk lands, and the partial tiles are reduced over the cluster
// like any split-K product and stored as out.
constexpr int split_threads(bool fuse) { return fuse ? kThreads + 64 : kThreads; }
constexpr uint32_t kWoChunk = 64 * kBK * 2;       // 64 W_out rows of one k-step
constexpr int kFuseMaxSteps = 8;                  // k-steps per CTA the fused form holds
// W_out chunks 4..7 past the caches, on a 1024-byte boundary (the swizzle atom)
constexpr size_t kWoSpare = 4 * static_cast<size_t>(kWoChunk) + 1024;

template <int BN, int kGate, bool kFuse = false>
constexpr size_t split_smem_bytes() {
    return LinearSmem<BN, kMmaM>::kDynamic + (kGate ? kRingCache + kTapCache : 0) +
           (kFuse ? kWoSpare : 0);
}

struct GateEpi {
    float* ring;            // [B][K-1][D]
    float* scratch_ring;    // [B][K-1][D] or null
    const float* conv_w;    // [D][K]
    __nv_bfloat16* y;       // [B][T][D]
    int B, T, D, n_commit;
};

// The fused form's output projection: y as the A operand (128-row boxes of
// 64 channels; rows past B*T read as zero), W_out as the B operand (64-row
// boxes), out [B*T][D] fp32, the barrier word and this call's tag.
struct alignas(64) FuseMaps {
    CUtensorMap y;
    CUtensorMap wo;
};
struct FuseOut {
    float* out;
    unsigned long long* bar;
    uint64_t tag;
};

template <int BN, int kGate, bool kFuse = false>
__global__ void __launch_bounds__(split_threads(kFuse), 1)
linear_bf16_splitk_kernel(const __grid_constant__ CUtensorMap tmap_x,
                          const __grid_constant__ CUtensorMap tmap_w, float* __restrict__ y,
                          int M, int N, int K, int splits, uint32_t* __restrict__ status,
                          GateEpi ge, const __grid_constant__ FuseMaps fm, FuseOut fo) {
    using L = LinearSmem<BN, kMmaM>;
    // the fused form has two more warps, for the walk and the reductions
    constexpr int kThr = split_threads(kFuse);
    constexpr int kStages = L::kStages;
    constexpr int kPitch = BN + 4;        // floats per parked row: 16-byte shift per row
    constexpr int kQuads = BN / 4;        // float4 columns of a row
    constexpr uint32_t kTmemCols = BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
    static_assert(kGate == 0 || BN == 192, "the gate tile is three 64-row blocks");
    static_assert(!kFuse || (kGate > 0 && kStages * L::kStage >= 16 * 8192 + 4 * kWoChunk),
                  "the fused form's y chunks and W_out chunks 0..3 fit the stage ring");
    // gate mode: u and cg of at most 8 channel quads per row after the parked tile
    constexpr size_t kGateOff = static_cast<size_t>(kMmaM) * kPitch * 4;
    constexpr size_t kGateBytes = kGate ? 2 * static_cast<size_t>(kMmaM) * 8 * 16 : 0;
    static_assert(kGateOff + kGateBytes + 1024 <= L::kDynamic,
                  "the partial tile fits the stage ring");
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages];
    __shared__ __align__(8) uint64_t empty[kStages];
    __shared__ __align__(8) uint64_t acc_full;
    // fused form: W_out chunks landed, each y chunk landed, output MMAs done
    __shared__ __align__(8) uint64_t wo_full;
    __shared__ __align__(8) uint64_t y_full[kFuseMaxSteps];
    __shared__ __align__(8) uint64_t out_full;
    __shared__ uint32_t tmem_slot;
    __shared__ int issued, consumed;
    __shared__ int failed;
    __shared__ int wo_issued, y_issued;

    const uint32_t raw = tc::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    float* part = reinterpret_cast<float*>(smem_raw + (base - raw));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = static_cast<int>(tc::cluster_ctarank());
    const int n0 = static_cast<int>(blockIdx.x / splits) * (kGate ? 64 : BN);   // column / channel base
    const int n_kt = (K + kBK - 1) / kBK;
    const int kb = static_cast<int>(static_cast<int64_t>(rank) * n_kt / splits);
    const int ke = static_cast<int>(static_cast<int64_t>(rank + 1) * n_kt / splits);
    // gate mode: this CTA's channel quads [q_lo, q_lo + nq) of the tile, and
    // the shared-memory copies of their ring entries and taps (past the ring)
    constexpr int KT = kGate > 0 ? kGate : 2;
    const int q_lo = rank * 16 / splits;
    const int nq = (rank + 1) * 16 / splits - q_lo;      // at most 8
    const int nch = 4 * nq;
    const bool ring_cached =
        kGate > 0 && static_cast<size_t>(ge.B) * (KT - 1) * nch * 4 <= kRingCache;
    float* ring_c = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(part) +
                                             static_cast<size_t>(kStages) * L::kStage);
    float* taps_c = ring_c + kRingCache / 4;
    // fused form: y chunk g at base + g * 16 KB (after the grid barrier);
    // W_out chunks 0..3 in the ring's last 32 KB, 4..7 past the caches
    const uint32_t wo_lo = base + kFuseMaxSteps * L::kA;
    const uint32_t wo_hi =
        (base + static_cast<uint32_t>(kStages * L::kStage + kRingCache + kTapCache) + 1023u) &
        ~1023u;
    auto wo_addr = [&](int g) -> uint32_t {
        return g < 4 ? wo_lo + g * kWoChunk : wo_hi + (g - 4) * kWoChunk;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(tc::smem_u32(&full[s]), 1);
            tc::mbar_init(tc::smem_u32(&empty[s]), 1);
        }
        tc::mbar_init(tc::smem_u32(&acc_full), 1);
        if constexpr (kFuse) {
            tc::mbar_init(tc::smem_u32(&wo_full), 1);
            for (int j = 0; j < kFuseMaxSteps; ++j) tc::mbar_init(tc::smem_u32(&y_full[j]), 1);
            tc::mbar_init(tc::smem_u32(&out_full), 1);
        }
        tc::fence_mbar_init();
        issued = 0;
        consumed = 0;
        failed = 0;
        wo_issued = 0;
        y_issued = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_u32(&tmem_slot), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    volatile int* vfailed = &failed;
    tc::grid_dep_launch();

    if (warp == 0 && lane == 0) {
        // ---- producer: this rank's k-steps through the stage ring ----------
        tc::prefetch_tmap(&tmap_x);
        tc::prefetch_tmap(&tmap_w);
        // the rank's x boxes, then the weight stripe, into L2 early (x
        // first: its few boxes would otherwise queue behind the stripe)
        for (int kt = kb; kt < ke; ++kt) tc::tma_prefetch_l2_2d(&tmap_x, kt * kBK, 0);
        const int pf_end = GDN_SPLIT_PREFETCH < 0 ? ke : min(ke, kb + GDN_SPLIT_PREFETCH);
        for (int kt = kb; kt < pf_end; ++kt) {
            if constexpr (kGate) {
                for (int blk = 0; blk < 3; ++blk)
                    tc::tma_prefetch_l2_2d(&tmap_w, kt * kBK, blk * ge.D + n0);
            } else {
                tc::tma_prefetch_l2_2d(&tmap_w, kt * kBK, n0);
            }
        }
        tc::grid_dep_wait();
        for (int kt = kb, g = 0; kt < ke; ++kt, ++g) {
            const int s = g % kStages;
            const uint32_t ph = static_cast<uint32_t>(g / kStages) & 1u;
            if (!tc::mbar_wait(tc::smem_u32(&empty[s]), ph ^ 1)) {
                if (status) atomicOr(status, tc::kTimeoutProducer);
                atomicExch(&failed, 1);
                break;
            }
            if (*vfailed) break;
            const uint32_t a = base + s * L::kStage;
            tc::mbar_arrive_expect_tx(tc::smem_u32(&full[s]), L::kStage);
            tc::tma_load_2d(a, &tmap_x, tc::smem_u32(&full[s]), kt * kBK, 0);
            if constexpr (kGate) {       // bg, cg, xv rows of the tile's channels
                for (int blk = 0; blk < 3; ++blk)
                    tc::tma_load_2d(a + L::kA + blk * 64 * kBK * 2, &tmap_w,
                                    tc::smem_u32(&full[s]), kt * kBK, blk * ge.D + n0);
            } else {
                tc::tma_load_2d(a + L::kA, &tmap_w, tc::smem_u32(&full[s]), kt * kBK, n0);
            }
            issued = g + 1;
        }
        if constexpr (kFuse) {
            // this call's tag into the barrier word (the previous kernel on
            // the stream is complete, so no launch still polls it)
            tc::grid_barrier_install(fo.bar, fo.tag, gridDim.x);
            // the input projection's MMAs are done, so its stages are free:
            // this CTA's W_out chunks (rows n0.., its k-steps), while the
            // partials are parked and reduced
            if (!*vfailed) {
                if (!tc::mbar_wait(tc::smem_u32(&acc_full), 0)) {
                    atomicExch(&failed, 1);
                } else if (!*vfailed) {
                    tc::mbar_arrive_expect_tx(tc::smem_u32(&wo_full),
                                              static_cast<uint32_t>(ke - kb) * kWoChunk);
                    for (int kt = kb, g = 0; kt < ke; ++kt, ++g)
                        tc::tma_load_2d(wo_addr(g), &fm.wo, tc::smem_u32(&wo_full), kt * kBK, n0);
                    wo_issued = 1;
                }
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer: one accumulator, the rank's k-steps in order ------
        tc::grid_dep_wait();
        const uint32_t idesc = tc::idesc_bf16_f32(kMmaM, BN);
        bool ok = true;
        for (int kt = kb, g = 0; kt < ke; ++kt, ++g) {
            const int s = g % kStages;
            const uint32_t ph = static_cast<uint32_t>(g / kStages) & 1u;
            if (!tc::mbar_wait(tc::smem_u32(&full[s]), ph) || *vfailed) {
                if (status) atomicOr(status, tc::kTimeoutMma);
                atomicExch(&failed, 1);
                ok = false;
                break;
            }
            consumed = g + 1;
            tc::tc_fence_after();
            const uint32_t a = base + s * L::kStage;
            const uint32_t b = a + L::kA;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
                tc::mma_bf16(tmem, tc::desc_k_sw128(a + kk * 32), tc::desc_k_sw128(b + kk * 32),
                             idesc, (g > 0 || kk > 0) ? 1u : 0u);
            tc::mma_commit(tc::smem_u32(&empty[s]));
        }
        // every MMA done (so every stage read and every copy landed): the
        // ring is free for the partial tile
        if (ok) tc::mma_commit(tc::smem_u32(&acc_full));
    } else if (warp >= 2 && warp < 2 + kEpilogueWarps) {
        tc::grid_dep_wait();
        if (kGate > 0 && ring_cached) {
            // ---- gate mode, while the MMAs run: the ring entries and taps of
            //      this CTA's channels into shared memory (the ring was
            //      written by earlier kernels on the stream: after the wait)
            const int et = static_cast<int>(threadIdx.x) - 64;
            const int n4 = ge.B * (KT - 1) * nq;
            for (int it = et; it < n4; it += 32 * kEpilogueWarps) {
                const int bt = it / nq;                        // b (K-1) + slot
                const int ql = it - bt * nq;
                const int d = n0 + 4 * (q_lo + ql);
                if (d < ge.D)
                    reinterpret_cast<float4*>(ring_c)[it] = *reinterpret_cast<const float4*>(
                        ge.ring + static_cast<int64_t>(bt) * ge.D + d);
            }
            for (int it = et; it < nch * KT; it += 32 * kEpilogueWarps) {
                const int d = n0 + 4 * q_lo + it / KT;
                if (d < ge.D) taps_c[it] = ge.conv_w[static_cast<int64_t>(d) * KT + it % KT];
            }
        }
        // ---- park the partial tile: TMEM -> registers -> this CTA's ring ---
        const int row = (warp & 3) * 32 + lane;            // TMEM lane quarter warp % 4
        if (!tc::mbar_wait(tc::smem_u32(&acc_full), 0) || *vfailed) {
            if (status) atomicOr(status, tc::kTimeoutEpilogue);
            atomicExch(&failed, 1);
        } else {
            tc::tc_fence_after();
            const uint32_t src = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
            static_assert(BN % 64 == 0, "the partial is parked 64 columns at a time");
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 64) {
                uint32_t r[64];
                tc::tmem_ld_32x32b_x64(src + c0, r);
                tc::tmem_ld_wait();
                if (row < M) {
                    float4* dst = reinterpret_cast<float4*>(part + row * kPitch + c0);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                             __uint_as_float(r[4 * j + 2]),
                                             __uint_as_float(r[4 * j + 3]));
                }
            }
        }
    }

    // Every CTA's partial is parked; each sums its slice over the cluster.
    // (On a timeout the partials are stale: the output is then undefined and
    // the status word says so, but every CTA still meets both barriers.)
    if ((warp < 2 && lane != 0) || warp >= 2 + kEpilogueWarps)
        tc::grid_dep_wait();                           // they store below too
    tc::tc_fence_before();
    __syncthreads();
    __syncwarp();
    tc::cluster_sync();
    // every rank's partial tile, addressed through its mapped base (an offset
    // into a peer's shared memory maps like the base)
    uint32_t peer[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) peer[s] = s < splits ? tc::map_shared_rank(base, s) : 0u;
    if constexpr (kGate == 0) {
        {
            const int units = M * kQuads;
            const int lo = static_cast<int>(static_cast<int64_t>(rank) * units / splits);
            const int hi = static_cast<int>(static_cast<int64_t>(rank + 1) * units / splits);
            const bool vec = (N & 3) == 0;
            // two units per pass: all 2 S remote loads are in flight together
    #pragma unroll 1
            for (int u0 = lo + static_cast<int>(threadIdx.x); u0 < hi; u0 += 2 * kThr) {
                float4 v[2][8];
    #pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int u = u0 + h * kThr;
                    const int row = u / kQuads;
                    const int c = (u - row * kQuads) * 4;
                    if (u >= hi || n0 + c >= N) continue;
                    const uint32_t off = static_cast<uint32_t>((row * kPitch + c) * 4);
    #pragma unroll
                    for (int s = 0; s < 8; ++s)
                        if (s < splits) v[h][s] = tc::ld_cluster_f4(peer[s] + off);
                }
    #pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int u = u0 + h * kThr;
                    const int row = u / kQuads;
                    const int c = (u - row * kQuads) * 4;
                    const int col = n0 + c;
                    if (u >= hi || col >= N) continue;
                    float4 acc = v[h][0];
    #pragma unroll
                    for (int s = 1; s < 8; ++s) {
                        if (s < splits) {
                            acc.x = __fadd_rn(acc.x, v[h][s].x);
                            acc.y = __fadd_rn(acc.y, v[h][s].y);
                            acc.z = __fadd_rn(acc.z, v[h][s].z);
                            acc.w = __fadd_rn(acc.w, v[h][s].w);
                        }
                    }
                    float* yrow = y + static_cast<int64_t>(row) * N;
                    if (vec && col + 4 <= N) {
                        *reinterpret_cast<float4*>(yrow + col) = acc;
                    } else {
                        const float e[4] = {acc.x, acc.y, acc.z, acc.w};
    #pragma unroll
                        for (int j = 0; j < 4; ++j)
                            if (col + j < N) yrow[col + j] = e[j];
                    }
                }
            }
        }
        // no CTA leaves (releasing its shared memory) while a peer still reads it
        __syncwarp();
        tc::cluster_sync();
    } else if (ge.T <= 2 && ring_cached) {
        // ---- gate mode, calls of one or two positions (decode, verify): one
        //      thread per (sequence, channel quad) sums bg, cg and xv over the
        //      S partials (rank order), forms u = bg * xv, walks its four
        //      channels' conv windows through the positions (the ring from the
        //      shared copy) and writes y and both rings. The arithmetic, and so
        //      every bit of y and the rings, is that of the general path below.
#pragma unroll 1
        for (int it = static_cast<int>(threadIdx.x); it < ge.B * nq; it += kThr) {
            const int b = it / nq;
            const int ql = it - b * nq;
            const int c = 4 * (q_lo + ql);
            const int d = n0 + c;
            if (d >= ge.D) continue;
            double wt[4][KT];
            float win[4][KT - 1], committed[4][KT - 1];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int tau = 0; tau < KT; ++tau) wt[j][tau] = taps_c[(4 * ql + j) * KT + tau];
#pragma unroll
                for (int i = 0; i < KT - 1; ++i)
                    committed[j][i] = win[j][i] = ring_c[(b * (KT - 1) + i) * nch + 4 * ql + j];
            }
            for (int t = 0; t < ge.T; ++t) {
                const int row = b * ge.T + t;
                const uint32_t off = static_cast<uint32_t>((row * kPitch + c) * 4);
                float4 v[3][8];
#pragma unroll
                for (int s2 = 0; s2 < 8; ++s2) {
                    if (s2 < splits) {
#pragma unroll
                        for (int blk = 0; blk < 3; ++blk)
                            v[blk][s2] = tc::ld_cluster_f4(peer[s2] + off + blk * 64 * 4);
                    }
                }
                float4 t3[3];
#pragma unroll
                for (int blk = 0; blk < 3; ++blk) {
                    t3[blk] = v[blk][0];
#pragma unroll
                    for (int s2 = 1; s2 < 8; ++s2) {
                        if (s2 < splits) {
                            t3[blk].x = __fadd_rn(t3[blk].x, v[blk][s2].x);
                            t3[blk].y = __fadd_rn(t3[blk].y, v[blk][s2].y);
                            t3[blk].z = __fadd_rn(t3[blk].z, v[blk][s2].z);
                            t3[blk].w = __fadd_rn(t3[blk].w, v[blk][s2].w);
                        }
                    }
                }
                const float uu[4] = {__fmul_rn(t3[0].x, t3[2].x), __fmul_rn(t3[0].y, t3[2].y),
                                     __fmul_rn(t3[0].z, t3[2].z), __fmul_rn(t3[0].w, t3[2].w)};
                const float cgv[4] = {t3[1].x, t3[1].y, t3[1].z, t3[1].w};
                __nv_bfloat16 yv[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    double conv = 0.0;
#pragma unroll
                    for (int tau = 0; tau < KT - 1; ++tau)
                        conv = fma(wt[j][tau], static_cast<double>(win[j][tau]), conv);
                    conv = fma(wt[j][KT - 1], static_cast<double>(uu[j]), conv);
                    yv[j] = __double2bfloat16(static_cast<double>(cgv[j]) * conv);
#pragma unroll
                    for (int tau = 0; tau < KT - 2; ++tau) win[j][tau] = win[j][tau + 1];
                    win[j][KT - 2] = uu[j];
                    if (t == ge.n_commit - 1) {
#pragma unroll
                        for (int tau = 0; tau < KT - 1; ++tau) committed[j][tau] = win[j][tau];
                    }
                }
                uint2 packed;
                packed.x = static_cast<uint32_t>(__bfloat16_as_ushort(yv[0])) |
                           (static_cast<uint32_t>(__bfloat16_as_ushort(yv[1])) << 16);
                packed.y = static_cast<uint32_t>(__bfloat16_as_ushort(yv[2])) |
                           (static_cast<uint32_t>(__bfloat16_as_ushort(yv[3])) << 16);
                *reinterpret_cast<uint2*>(ge.y + static_cast<int64_t>(row) * ge.D + d) = packed;
            }
            float* rg = ge.ring + static_cast<int64_t>(b) * (KT - 1) * ge.D + d;
#pragma unroll
            for (int tau = 0; tau < KT - 1; ++tau)
                *reinterpret_cast<float4*>(rg + static_cast<int64_t>(tau) * ge.D) =
                    make_float4(committed[0][tau], committed[1][tau], committed[2][tau],
                                committed[3][tau]);
            if (ge.scratch_ring) {
                float* sg = ge.scratch_ring + static_cast<int64_t>(b) * (KT - 1) * ge.D + d;
#pragma unroll
                for (int tau = 0; tau < KT - 1; ++tau)
                    *reinterpret_cast<float4*>(sg + static_cast<int64_t>(tau) * ge.D) =
                        make_float4(win[0][tau], win[1][tau], win[2][tau], win[3][tau]);
            }
        }
        if constexpr (kFuse) {
            // ---- the output projection ------------------------------------
            // This CTA's y is stored (generic proxy); every CTA's must be
            // before any is loaded (async proxy). Passing the grid barrier
            // also means every peer has finished reading this CTA's parked
            // partial, so TMA may overwrite the ring (the proxy fences order
            // the parked partial's generic stores before those writes).
            tc::fence_proxy_async();
            __syncthreads();
            const int nk = ke - kb;
            if (threadIdx.x == 0) {
                if (!tc::grid_barrier_wait(fo.bar, fo.tag, gridDim.x)) {
                    if (status) atomicOr(status, tc::kTimeoutGrid);
                    atomicExch(&failed, 1);
                } else if (!*vfailed) {
                    tc::fence_proxy_async();
                    for (int kt = kb, g = 0; kt < ke; ++kt, ++g) {
                        tc::mbar_arrive_expect_tx(tc::smem_u32(&y_full[g]), L::kA);
                        tc::tma_load_2d(base + g * L::kA, &fm.y, tc::smem_u32(&y_full[g]),
                                        kt * kBK, 0);
                    }
                    y_issued = nk;
                }
            }
            __syncthreads();
            const bool run_out = y_issued > 0;
            if (run_out && warp == 1 && lane == 0) {
                // y chunk g (A, 128 rows) times W_out chunk g (B, 64 rows)
                // into TMEM columns [0, 64), in k order, as each chunk lands
                bool ok = tc::mbar_wait(tc::smem_u32(&wo_full), 0) && !*vfailed;
                const uint32_t idesc = tc::idesc_bf16_f32(kMmaM, 64);
                for (int g = 0; ok && g < nk; ++g) {
                    if (!tc::mbar_wait(tc::smem_u32(&y_full[g]), 0)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t a = base + g * L::kA;
                    const uint32_t b = wo_addr(g);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc::mma_bf16(tmem, tc::desc_k_sw128(a + kk * 32),
                                     tc::desc_k_sw128(b + kk * 32), idesc,
                                     (g > 0 || kk > 0) ? 1u : 0u);
                }
                if (ok) {
                    tc::mma_commit(tc::smem_u32(&out_full));
                } else {
                    if (status) atomicOr(status, tc::kTimeoutMma);
                    atomicExch(&failed, 1);
                }
            } else if (run_out && warp >= 2 && warp < 2 + kEpilogueWarps) {
                // park the output partial (rows < M, 64 columns, rows padded
                // by 16 bytes) at the ring's start: every y chunk was read
                constexpr int kPitchO = 64 + 4;
                const int row = (warp & 3) * 32 + lane;
                if (!tc::mbar_wait(tc::smem_u32(&out_full), 0) || *vfailed) {
                    if (status) atomicOr(status, tc::kTimeoutEpilogue);
                    atomicExch(&failed, 1);
                } else {
                    tc::tc_fence_after();
                    const uint32_t src = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
                    uint32_t r[64];
                    tc::tmem_ld_32x32b_x64(src, r);
                    tc::tmem_ld_wait();
                    if (row < M) {
                        float4* dst = reinterpret_cast<float4*>(part + row * kPitchO);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            dst[j] = make_float4(
                                __uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                    }
                }
            }
            tc::tc_fence_before();
            __syncthreads();
            __syncwarp();
            tc::cluster_sync();
            // every CTA sums a 1/S slice of the 64-column tile over the S
            // partials in rank order and stores it: the split-K form's sum
            {
                constexpr int kPitchO = 64 + 4;
                constexpr int kQuadsO = 16;
                const int units = run_out ? M * kQuadsO : 0;
                const int lo = static_cast<int>(static_cast<int64_t>(rank) * units / splits);
                const int hi = static_cast<int>(static_cast<int64_t>(rank + 1) * units / splits);
#pragma unroll 1
                for (int u0 = lo + static_cast<int>(threadIdx.x); u0 < hi; u0 += 2 * kThr) {
                    float4 v[2][8];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int u = u0 + h * kThr;
                        if (u >= hi) continue;
                        const int row = u / kQuadsO;
                        const int c = (u - row * kQuadsO) * 4;
                        const uint32_t off = static_cast<uint32_t>((row * kPitchO + c) * 4);
#pragma unroll
                        for (int s2 = 0; s2 < 8; ++s2)
                            if (s2 < splits) v[h][s2] = tc::ld_cluster_f4(peer[s2] + off);
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int u = u0 + h * kThr;
                        if (u >= hi) continue;
                        const int row = u / kQuadsO;
                        const int c = (u - row * kQuadsO) * 4;
                        float4 acc = v[h][0];
#pragma unroll
                        for (int s2 = 1; s2 < 8; ++s2) {
                            if (s2 < splits) {
                                acc.x = __fadd_rn(acc.x, v[h][s2].x);
                                acc.y = __fadd_rn(acc.y, v[h][s2].y);
                                acc.z = __fadd_rn(acc.z, v[h][s2].z);
                                acc.w = __fadd_rn(acc.w, v[h][s2].w);
                            }
                        }
                        *reinterpret_cast<float4*>(fo.out + static_cast<int64_t>(row) * ge.D + n0 +
                                                   c) = acc;
                    }
                }
            }
        }
        // no CTA leaves (releasing its shared memory) while a peer still reads it
        __syncwarp();
        tc::cluster_sync();
    } else {
        // ---- gate mode: u = bg * xv and cg for this CTA's channel quads ----
        float4* u_s = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(part) + kGateOff);
        float4* cg_s = u_s + kMmaM * 8;
#pragma unroll 1
        for (int it = static_cast<int>(threadIdx.x); it < M * nq; it += kThr) {
            const int row = it / nq;
            const int ql = it - row * nq;
            const int c = 4 * (q_lo + ql);
            if (n0 + c >= ge.D) continue;
            const uint32_t off = static_cast<uint32_t>((row * kPitch + c) * 4);
            float4 v[3][8];
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
                if (s2 < splits) {
#pragma unroll
                    for (int blk = 0; blk < 3; ++blk)
                        v[blk][s2] = tc::ld_cluster_f4(peer[s2] + off + blk * 64 * 4);
                }
            }
            float4 t3[3];
#pragma unroll
            for (int blk = 0; blk < 3; ++blk) {
                t3[blk] = v[blk][0];
#pragma unroll
                for (int s2 = 1; s2 < 8; ++s2) {
                    if (s2 < splits) {
                        t3[blk].x = __fadd_rn(t3[blk].x, v[blk][s2].x);
                        t3[blk].y = __fadd_rn(t3[blk].y, v[blk][s2].y);
                        t3[blk].z = __fadd_rn(t3[blk].z, v[blk][s2].z);
                        t3[blk].w = __fadd_rn(t3[blk].w, v[blk][s2].w);
                    }
                }
            }
            u_s[row * 8 + ql] = make_float4(__fmul_rn(t3[0].x, t3[2].x), __fmul_rn(t3[0].y, t3[2].y),
                                            __fmul_rn(t3[0].z, t3[2].z), __fmul_rn(t3[0].w, t3[2].w));
            cg_s[row * 8 + ql] = t3[1];
        }
        // no CTA leaves (releasing its shared memory) while a peer still
        // reads it; u and cg are complete in this CTA
        __syncwarp();
        tc::cluster_sync();
        // ---- the conv walk: one thread per (sequence, channel) -------------
        // (two items per pass, so that the two independent chains of shared
        // loads, double-precision window sums and stores overlap)
        auto walk = [&](int it) {
            const int b = it / nch;
            const int cl = it - b * nch;
            const int d = n0 + 4 * q_lo + cl;
            if (d >= ge.D) return;
            const float* u_f = reinterpret_cast<const float*>(u_s) + (cl >> 2) * 4 + (cl & 3);
            const float* cg_f = reinterpret_cast<const float*>(cg_s) + (cl >> 2) * 4 + (cl & 3);
            double wt[KT];
#pragma unroll
            for (int tau = 0; tau < KT; ++tau)
                wt[tau] = ring_cached ? taps_c[cl * KT + tau]
                                      : ge.conv_w[static_cast<int64_t>(d) * KT + tau];
            float* rg = ge.ring + static_cast<int64_t>(b) * (KT - 1) * ge.D + d;
            float win[KT - 1], committed[KT - 1];
#pragma unroll
            for (int i = 0; i < KT - 1; ++i)
                committed[i] = win[i] = ring_cached ? ring_c[(b * (KT - 1) + i) * nch + cl]
                                                    : rg[static_cast<int64_t>(i) * ge.D];
            for (int t = 0; t < ge.T; ++t) {
                const int row = b * ge.T + t;
                const float u = u_f[row * 32];
                double conv = 0.0;
#pragma unroll
                for (int tau = 0; tau < KT - 1; ++tau)
                    conv = fma(wt[tau], static_cast<double>(win[tau]), conv);
                conv = fma(wt[KT - 1], static_cast<double>(u), conv);
                ge.y[static_cast<int64_t>(row) * ge.D + d] =
                    __double2bfloat16(static_cast<double>(cg_f[row * 32]) * conv);
#pragma unroll
                for (int tau = 0; tau < KT - 2; ++tau) win[tau] = win[tau + 1];
                win[KT - 2] = u;
                if (t == ge.n_commit - 1) {
#pragma unroll
                    for (int tau = 0; tau < KT - 1; ++tau) committed[tau] = win[tau];
                }
            }
#pragma unroll
            for (int tau = 0; tau < KT - 1; ++tau) rg[static_cast<int64_t>(tau) * ge.D] = committed[tau];
            if (ge.scratch_ring) {
                float* sg = ge.scratch_ring + static_cast<int64_t>(b) * (KT - 1) * ge.D + d;
#pragma unroll
                for (int tau = 0; tau < KT - 1; ++tau) sg[static_cast<int64_t>(tau) * ge.D] = win[tau];
            }
        };
        const int n_items = ge.B * nch;
#pragma unroll 1
        for (int it = static_cast<int>(threadIdx.x); it < n_items; it += 2 * kThr) {
            walk(it);
            if (it + kThr < n_items) walk(it + kThr);
        }
    }

    if (threadIdx.x == 0 && failed) {
        for (int g = consumed; g < issued; ++g)
            tc::mbar_wait(tc::smem_u32(&full[g % kStages]), static_cast<uint32_t>(g / kStages) & 1u);
        if constexpr (kFuse) {      // the fused form's copies in flight land first
            if (wo_issued) tc::mbar_wait(tc::smem_u32(&wo_full), 0);
            for (int g = 0; g < y_issued; ++g) tc::mbar_wait(tc::smem_u32(&y_full[g]), 0);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

// Pair-CTA form for large products: a cluster of two CTAs on two SMs owns a
// 256 x 256 output tile and runs it as M = 256 tcgen05.mma (cta_group::2)
// issued by the leader (rank 0). Each CTA stages its own 128 rows of x and its
// own 128 rows of W per k-step (32 KB), so each SM takes in half the bytes of
// a single-CTA 256 x 256 tile, and holds only its 128 x 256 quarter of the
// accumulator: two accumulator sets fit in TMEM and a tile's epilogue runs
// while the next tile's MMAs fill the other set.
//   full[s]     leader only: one arrival (the leader's expect-tx of both
//               CTAs' bytes); both CTAs' TMA loads complete on it;
//   empty[s]    both CTAs: the leader's per-stage commit, sent to both;
//   acc_full    both CTAs: the leader's per-tile commit, sent to both;
//   acc_empty   leader only: the four epilogue warps of both CTAs (the
//               peer's arrive remotely).
// Rows of a tile accumulate over K in the same order as the other forms.
// Every wait is bounded (2 s); every path meets the cluster barriers at the
// end, after which the leader lets copies addressed to its barriers land.
#ifndef GDN_LINEAR_PAIR_STAGES
#define GDN_LINEAR_PAIR_STAGES 6
#endif
constexpr int kPairStages = GDN_LINEAR_PAIR_STAGES;
constexpr uint32_t kPairHalf = 128 * kBK * 2;                 // 128 rows x 64 bf16
constexpr uint32_t kPairStage = 2 * kPairHalf;                // x half + W half
constexpr size_t kPairDynamic = static_cast<size_t>(kPairStage) * kPairStages + 1024;
static_assert(kPairDynamic <= 232448, "the stage ring fits the shared memory of a CTA");

__global__ void __launch_bounds__(kThreads, 1)
linear_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ CUtensorMap tmap_w, float* __restrict__ y, int M,
                        int N, int K, uint32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kPairStages];
    __shared__ __align__(8) uint64_t empty[kPairStages];
    __shared__ __align__(8) uint64_t acc_full[2];
    __shared__ __align__(8) uint64_t acc_empty[2];
    __shared__ uint32_t tmem_slot;
    __shared__ int issued, consumed;
    __shared__ int failed;

    const uint32_t raw = tc::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = static_cast<int>(tc::cluster_ctarank());   // 0: leader
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int n_pairs = static_cast<int>(gridDim.x >> 1);
    const int n_kt = (K + kBK - 1) / kBK;
    const int tiles_n = (N + 255) / 256;
    const int n_tiles = tiles_n * ((M + 255) / 256);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            tc::mbar_init(tc::smem_u32(&full[s]), 1);
            tc::mbar_init(tc::smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(tc::smem_u32(&acc_full[a]), 1);
            tc::mbar_init(tc::smem_u32(&acc_empty[a]), 2 * kEpilogueWarps);
        }
        tc::fence_mbar_init();
        issued = 0;
        consumed = 0;
        failed = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc_pair(tc::smem_u32(&tmem_slot), 512);
        tc::tmem_relinquish_pair();
    }
    // both CTAs' barriers exist before either signals the other's
    tc::tc_fence_before();
    __syncthreads();
    __syncwarp();
    tc::cluster_sync();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    volatile int* vfailed = &failed;
    tc::grid_dep_launch();

    if (warp == 0 && lane == 0) {
        // ---- producer (both CTAs): this CTA's halves of every k-step -------
        tc::prefetch_tmap(&tmap_x);
        tc::prefetch_tmap(&tmap_w);
        tc::grid_dep_wait();
        int g = 0;
        for (int tile = pair; tile < n_tiles && !*vfailed; tile += n_pairs) {
            const int m0 = (tile / tiles_n) * 256 + rank * 128;
            const int n0 = (tile % tiles_n) * 256 + rank * 128;
            for (int kt = 0; kt < n_kt; ++kt, ++g) {
                const int s = g % kPairStages;
                const uint32_t ph = static_cast<uint32_t>(g / kPairStages) & 1u;
                if (!tc::mbar_wait(tc::smem_u32(&empty[s]), ph ^ 1)) {
                    if (status) atomicOr(status, tc::kTimeoutProducer);
                    atomicExch(&failed, 1);
                    break;
                }
                if (*vfailed) break;
                const uint32_t a = base + s * kPairStage;
                const uint32_t fb = tc::map_shared_rank(tc::smem_u32(&full[s]), 0);
                if (rank == 0) tc::mbar_arrive_expect_tx(tc::smem_u32(&full[s]), 2 * kPairStage);
                tc::tma_load_2d_pair(a, &tmap_x, fb, kt * kBK, m0);
                tc::tma_load_2d_pair(a + kPairHalf, &tmap_w, fb, kt * kBK, n0);
                issued = g + 1;
            }
        }
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ---- MMA issuer (leader): tile li into accumulator set li % 2 -------
        tc::grid_dep_wait();
        const uint32_t idesc = tc::idesc_bf16_f32(256, 256);
        int g = 0;
        bool ok = true;
        int li = 0;
        for (int tile = pair; ok && tile < n_tiles; tile += n_pairs, ++li) {
            const int acc = li & 1;
            const uint32_t d = tmem + static_cast<uint32_t>(acc) * 256;
            if (!tc::mbar_wait(tc::smem_u32(&acc_empty[acc]), ((li >> 1) & 1) ^ 1) || *vfailed) {
                if (status) atomicOr(status, tc::kTimeoutMma);
                atomicExch(&failed, 1);
                break;
            }
            tc::tc_fence_after();
            for (int kt = 0; kt < n_kt; ++kt, ++g) {
                const int s = g % kPairStages;
                const uint32_t ph = static_cast<uint32_t>(g / kPairStages) & 1u;
                if (!tc::mbar_wait(tc::smem_u32(&full[s]), ph) || *vfailed) {
                    if (status) atomicOr(status, tc::kTimeoutMma);
                    atomicExch(&failed, 1);
                    ok = false;
                    break;
                }
                consumed = g + 1;
                tc::tc_fence_after();
                const uint32_t a = base + s * kPairStage;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    tc::mma_bf16_pair(d, tc::desc_k_sw128(a + kk * 32),
                                      tc::desc_k_sw128(a + kPairHalf + kk * 32), idesc,
                                      (kt > 0 || kk > 0) ? 1u : 0u);
                tc::mma_commit_pair(tc::smem_u32(&empty[s]), 0x3);   // both CTAs' slots
            }
            if (ok) tc::mma_commit_pair(tc::smem_u32(&acc_full[acc]), 0x3);
        }
    } else if (warp >= 2) {
        // ---- epilogue (both CTAs): this CTA's 128 rows of each tile ---------
        tc::grid_dep_wait();
        const int quarter = warp & 3;
        const uint32_t ae0 = tc::map_shared_rank(tc::smem_u32(&acc_empty[0]), 0);
        const uint32_t ae1 = tc::map_shared_rank(tc::smem_u32(&acc_empty[1]), 0);
        int li = 0;
        for (int tile = pair; tile < n_tiles; tile += n_pairs, ++li) {
            const int acc = li & 1;
            if (!tc::mbar_wait(tc::smem_u32(&acc_full[acc]), (li >> 1) & 1) || *vfailed) {
                if (status) atomicOr(status, tc::kTimeoutEpilogue);
                atomicExch(&failed, 1);
                break;
            }
            tc::tc_fence_after();
            const int row = (tile / tiles_n) * 256 + rank * 128 + quarter * 32 + lane;
            const int n0 = (tile % tiles_n) * 256;
            const bool row_ok = row < M;
            float* yrow = y + static_cast<int64_t>(row) * N;
            const uint32_t src = tmem + static_cast<uint32_t>(acc) * 256 +
                                 (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < 256; c0 += 32) {
                uint32_t r[32];
                tc::tmem_ld_32x32b_x32(src + c0, r);
                tc::tmem_ld_wait();
                const int col = n0 + c0;
                if (!row_ok || col >= N) continue;
                if (col + 32 <= N && (N & 3) == 0) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(yrow + col + j) =
                            make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                        __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (col + j < N) yrow[col + j] = __uint_as_float(r[j]);
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive_cluster(acc ? ae1 : ae0);   // the leader's set is free
        }
    }

    // Both CTAs meet here; then the leader lets any copy still addressed to
    // its barriers land (a timeout path only), and both meet again before
    // TMEM and shared memory are released.
    if (warp < 2 && lane != 0) tc::grid_dep_wait();
    tc::tc_fence_before();
    __syncthreads();
    __syncwarp();
    tc::cluster_sync();
    if (threadIdx.x == 0 && rank == 0 && failed) {
        for (int g = consumed; g < issued; ++g)
            tc::mbar_wait(tc::smem_u32(&full[g % kPairStages]),
                          static_cast<uint32_t>(g / kPairStages) & 1u);
    }
    __syncthreads();
    __syncwarp();
    tc::cluster_sync();
    tc::tc_fence_after();
    if (warp == 1) tc::tmem_dealloc_pair(tmem, 512);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Row-major bf16 matrix [rows][K] as a 2D tensor map with box [box_rows][64].
bool make_tmap(CUtensorMap* map, const void* ptr, int64_t rows, int64_t K, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int BN, int BM>
cudaError_t launch_bn(const LinearArgs& a, cudaStream_t stream) {
    CUtensorMap tx, tw;
    if (!make_tmap(&tx, a.x, a.M, a.K, BM) || !make_tmap(&tw, a.w, a.N, a.K, BN))
        return cudaErrorInvalidValue;
    const size_t smem = LinearSmem<BN, BM>::kDynamic;
    cudaError_t err = cudaFuncSetAttribute(linear_bf16_kernel<BN, BM>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int64_t tiles = ((a.N + BN - 1) / BN) * ((a.M + BM - 1) / BM);
    if (tiles > INT32_MAX) return cudaErrorInvalidValue;
    const int64_t sms = device_sm_count();
    const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
    // programmatic serialization: the prologue overlaps the previous kernel
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, linear_bf16_kernel<BN, BM>, tx, tw, a.y, static_cast<int>(a.M),
                              static_cast<int>(a.N), static_cast<int>(a.K), a.status);
}

template <int BN, int kGate = 0, bool kFuse = false>
cudaError_t set_split_smem() {
    return cudaFuncSetAttribute(linear_bf16_splitk_kernel<BN, kGate, kFuse>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(split_smem_bytes<BN, kGate, kFuse>()));
}

// Cluster of `splits` CTAs along x, and (`pdl`) programmatic serialization
// so the prologue overlaps the previous kernel; attr holds two entries.
template <int BN, int kGate = 0, bool kFuse = false>
cudaLaunchConfig_t split_config(unsigned grid, int splits, cudaStream_t stream,
                                cudaLaunchAttribute* attr, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(split_threads(kFuse));
    cfg.dynamicSmemBytes = split_smem_bytes<BN, kGate, kFuse>();
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cfg;
}

// Clusters of `splits` CTAs of the BN-wide split kernel that the device holds
// at once (cached per device; 0 when the query fails).
template <int BN, int kGate = 0, bool kFuse = false>
int max_active_clusters(int splits) {
    constexpr int kDevs = 16;
    static std::atomic<int> cache[kDevs][9];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < kDevs) {
        const int c = cache[dev][splits].load(std::memory_order_relaxed);
        if (c > 0) return c - 1;
    }
    int n = 0;
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg = split_config<BN, kGate, kFuse>(static_cast<unsigned>(splits),
                                                           splits, nullptr, attr, false);
    if (set_split_smem<BN, kGate, kFuse>() != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, linear_bf16_splitk_kernel<BN, kGate, kFuse>, &cfg) !=
            cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (dev < kDevs) cache[dev][splits].store(n + 1, std::memory_order_relaxed);
    return n;
}

int max_active_clusters_bn(int bn, int splits) {
    if (bn == 256) return max_active_clusters<256>(splits);
    if (bn == 128) return max_active_clusters<128>(splits);
    return max_active_clusters<64>(splits);
}

struct SplitPlan {
    int bn = 0;
    int splits = 1;
};

// The split for an (N, K) product: for each tile width, as many K chunks (at
// most 8, at most one per k-step) as keep tiles x chunks within one wave of
// clusters on the device's SMs; the plan with the most CTAs wins, the wider
// tile on a tie. (Fewer k-steps per CTA through wider tiles and more chunks
// measured slower: the cluster reduction grows with the tile and the chunk
// count.) A function of (N, K) and the device, never of M.
SplitPlan split_plan(int64_t N, int64_t K) {
    const int64_t n_kt = (K + kBK - 1) / kBK;
    const int64_t sms = device_sm_count();
    SplitPlan best;
    int64_t best_ctas = 0;
    for (const int bn : {256, 128, 64}) {
        const int64_t tiles = (N + bn - 1) / bn;
        int64_t s = std::min<int64_t>(std::min<int64_t>(8, n_kt), sms / tiles);
        for (; s >= 2; --s)
            if (tiles <= max_active_clusters_bn(bn, static_cast<int>(s))) break;
        if (s < 2) continue;
        if (tiles * s > best_ctas) {
            best_ctas = tiles * s;
            best.bn = bn;
            best.splits = static_cast<int>(s);
        }
    }
    return best;
}

template <int BN>
cudaError_t launch_split_bn(const LinearArgs& a, int splits, cudaStream_t stream) {
    CUtensorMap tx, tw;
    if (!make_tmap(&tx, a.x, a.M, a.K, kMmaM) || !make_tmap(&tw, a.w, a.N, a.K, BN))
        return cudaErrorInvalidValue;
    cudaError_t err = set_split_smem<BN>();
    if (err != cudaSuccess) return err;
    const int64_t tiles = (a.N + BN - 1) / BN;
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg =
        split_config<BN>(static_cast<unsigned>(tiles * splits), splits, stream, attr, true);
    return cudaLaunchKernelEx(&cfg, linear_bf16_splitk_kernel<BN, 0>, tx, tw, a.y,
                              static_cast<int>(a.M), static_cast<int>(a.N),
                              static_cast<int>(a.K), splits, a.status, GateEpi{}, FuseMaps{},
                              FuseOut{});
}

// Pairs of the pair-CTA kernel the device holds at once (cached per device).
int max_active_pairs() {
    constexpr int kDevs = 16;
    static std::atomic<int> cache[kDevs];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < kDevs) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c - 1;
    }
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kPairDynamic;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaFuncSetAttribute(linear_bf16_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kPairDynamic)) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, linear_bf16_pair_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (dev < kDevs) cache[dev].store(n + 1, std::memory_order_relaxed);
    return n;
}

cudaError_t launch_pair_gemm(const LinearArgs& a, int64_t tiles, int pairs, cudaStream_t stream) {
    CUtensorMap tx, tw;
    if (!make_tmap(&tx, a.x, a.M, a.K, 128) || !make_tmap(&tw, a.w, a.N, a.K, 128))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(linear_bf16_pair_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kPairDynamic));
    if (err != cudaSuccess) return err;
    const int64_t n = tiles < pairs ? tiles : pairs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * n));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kPairDynamic;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, linear_bf16_pair_kernel, tx, tw, a.y, static_cast<int>(a.M),
                              static_cast<int>(a.N), static_cast<int>(a.K), a.status);
}

// The gate form's split of K for D channels: tiles of 64 channels, each split
// over K like the plain form (the most chunks that keep the clusters in one
// wave, at most 8); below 2 the form does not apply.
template <int KT, bool kFuse = false>
int64_t gate_splits(int64_t D) {
    const int64_t n_kt = (D + kBK - 1) / kBK;
    const int64_t tiles = (D + 63) / 64;
    int64_t s = std::min<int64_t>(std::min<int64_t>(8, n_kt), device_sm_count() / tiles);
    for (; s >= 2; --s)
        if (tiles <= max_active_clusters<192, KT, kFuse>(static_cast<int>(s))) break;
    return s;
}

GateEpi gate_epi(const ShortConvArgs& a, void* y) {
    GateEpi ge;
    ge.ring = a.conv_ring;
    ge.scratch_ring = a.scratch_ring;
    ge.conv_w = a.conv_w;
    ge.y = static_cast<__nv_bfloat16*>(y);
    ge.B = static_cast<int>(a.B);
    ge.T = static_cast<int>(a.T);
    ge.D = static_cast<int>(a.D);
    ge.n_commit = static_cast<int>(a.n_commit);
    return ge;
}

// The short-conv input projection with the gate and conv as its epilogue.
template <int KT>
cudaError_t launch_gate_k(const ShortConvArgs& a, void* y, cudaStream_t stream) {
    const int64_t M = a.B * a.T, D = a.D;
    const int64_t tiles = (D + 63) / 64;
    const int64_t s = gate_splits<KT>(D);
    if (s < 2) return cudaErrorNotSupported;
    CUtensorMap tx, tw;
    if (!make_tmap(&tx, a.hidden, M, D, kMmaM) || !make_tmap(&tw, a.w_in, 3 * D, D, 64))
        return cudaErrorInvalidValue;
    cudaError_t err = set_split_smem<192, KT>();
    if (err != cudaSuccess) return err;
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg = split_config<192, KT>(static_cast<unsigned>(tiles * s),
                                                         static_cast<int>(s), stream, attr, true);
    return cudaLaunchKernelEx(&cfg, linear_bf16_splitk_kernel<192, KT>, tx, tw,
                              static_cast<float*>(nullptr), static_cast<int>(M),
                              static_cast<int>(3 * D), static_cast<int>(D), static_cast<int>(s),
                              a.status, gate_epi(a, y), FuseMaps{}, FuseOut{});
}

// A 48-bit tag, never 0, for each fused launch enqueued by this process
// (SplitMix64 over a counter seeded from the clock and the process id), so
// that the barrier word of a workspace never holds a stale tag of a later
// call.
uint64_t next_call_tag() {
    static std::atomic<uint64_t> seq{0};
    static const uint64_t seed = static_cast<uint64_t>(
        std::chrono::steady_clock::now().time_since_epoch().count()) ^
        (static_cast<uint64_t>(getpid()) << 32);
    uint64_t z = seed + 0x9E3779B97F4A7C15ull * (seq.fetch_add(1, std::memory_order_relaxed) + 1);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    z &= (1ull << 48) - 1;
    return z ? z : 1;
}

// The whole mixer in one kernel (the split kernel's kFuse form), for calls of
// one or two positions whose split is the one the two-kernel path takes for
// both projections, so that its bits are that path's.
template <int KT>
cudaError_t launch_fused_k(const ShortConvArgs& a, void* y, unsigned long long* bar,
                           cudaStream_t stream) {
    const int64_t M = a.B * a.T, D = a.D;
    if (a.T > 2 || M > kMmaM || D % 64 != 0 || (reinterpret_cast<uintptr_t>(bar) & 7) != 0)
        return cudaErrorNotSupported;
    const int64_t n_kt = D / kBK, tiles = D / 64;
    const int64_t s = gate_splits<KT>(D);
    if (s < 2 || gate_splits<KT, true>(D) != s) return cudaErrorNotSupported;
    const SplitPlan p = split_plan(D, D);
    if (p.bn != 64 || p.splits != s) return cudaErrorNotSupported;
    if ((n_kt + s - 1) / s > kFuseMaxSteps) return cudaErrorNotSupported;
    // every rank's conv rings in shared memory (the walk the fused form runs)
    const int64_t nq_max = (16 + s - 1) / s;
    if (a.B * (KT - 1) * 4 * nq_max * 4 > static_cast<int64_t>(kRingCache))
        return cudaErrorNotSupported;
    CUtensorMap tx, tw;
    FuseMaps fm;
    if (!make_tmap(&tx, a.hidden, M, D, kMmaM) || !make_tmap(&tw, a.w_in, 3 * D, D, 64) ||
        !make_tmap(&fm.y, y, M, D, kMmaM) || !make_tmap(&fm.wo, a.w_out, D, D, 64))
        return cudaErrorInvalidValue;
    cudaError_t err = set_split_smem<192, KT, true>();
    if (err != cudaSuccess) return err;
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg = split_config<192, KT, true>(
        static_cast<unsigned>(tiles * s), static_cast<int>(s), stream, attr, true);
    FuseOut fo;
    fo.out = a.out;
    fo.bar = bar;
    fo.tag = next_call_tag();
    return cudaLaunchKernelEx(&cfg, linear_bf16_splitk_kernel<192, KT, true>, tx, tw,
                              static_cast<float*>(nullptr), static_cast<int>(M),
                              static_cast<int>(3 * D), static_cast<int>(D), static_cast<int>(s),
                              a.status, gate_epi(a, y), fm, fo);
}

}  // namespace

cudaError_t launch_short_conv_in_gate(const ShortConvArgs& a, void* y, cudaStream_t stream) {
    if (a.B * a.T > kMmaM) return cudaErrorNotSupported;
    switch (a.K) {
        case 2: return launch_gate_k<2>(a, y, stream);
        case 3: return launch_gate_k<3>(a, y, stream);
        case 4: return launch_gate_k<4>(a, y, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_short_conv_fused(const ShortConvArgs& a, void* y, unsigned long long* bar,
                                    cudaStream_t stream) {
    switch (a.K) {
        case 2: return launch_fused_k<2>(a, y, bar, stream);
        case 3: return launch_fused_k<3>(a, y, bar, stream);
        case 4: return launch_fused_k<4>(a, y, bar, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_linear_bf16_split(const LinearArgs& a, cudaStream_t stream) {
    if (a.M == 0 || a.N == 0) return cudaSuccess;
    if (a.M > kMmaM) return launch_linear_bf16(a, stream);
    const SplitPlan p = split_plan(a.N, a.K);
    if (p.splits < 2) return launch_linear_bf16(a, stream);
    if (p.bn == 256) return launch_split_bn<256>(a, p.splits, stream);
    if (p.bn == 128) return launch_split_bn<128>(a, p.splits, stream);
    return launch_split_bn<64>(a, p.splits, stream);
}

cudaError_t launch_linear_bf16(const LinearArgs& a, cudaStream_t stream) {
    if (a.M == 0 || a.N == 0) return cudaSuccess;
    // The widest tile whose count still covers every SM once: 256 x 256,
    // then 128 x 256, 128 x 128, 128 x 64 (decode-sized products get narrow
    // tiles so that more SMs stream the weights).
    int shape = GDN_LINEAR_BN;
    if (shape == 0) {
        const int64_t sms = device_sm_count();
        auto tiles = [&](int64_t bm, int64_t bn) {
            return ((a.M + bm - 1) / bm) * ((a.N + bn - 1) / bn);
        };
        shape = 64;
        if (tiles(256, 256) >= sms) shape = 512;
        else if (tiles(128, 256) >= sms) shape = 256;
        else if (tiles(128, 128) >= sms) shape = 128;
    }
    if (shape == 512 && GDN_LINEAR_PAIR && GDN_LINEAR_BN == 0 && a.N >= 256) {
        // 256 x 256 tiles for every pair of SMs: the pair-CTA form
        const int64_t tiles = ((a.M + 255) / 256) * ((a.N + 255) / 256);
        const int pairs = max_active_pairs();
        if (pairs > 0 && tiles >= pairs) return launch_pair_gemm(a, tiles, pairs, stream);
    }
    if (shape == 512) return launch_bn<256, 256>(a, stream);
    if (shape == 256) return launch_bn<256, 128>(a, stream);
    if (shape == 128) return launch_bn<128, 128>(a, stream);
    return launch_bn<64, 128>(a, stream);
}

}  // namespace gdn
