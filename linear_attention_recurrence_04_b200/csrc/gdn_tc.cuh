// gdn_tc.cuh -- sm_100a tensor-core building blocks: mbarriers with bounded
// waits, 2D TMA tile loads, UMMA shared-memory and instruction descriptors,
// TMEM allocation, tcgen05.mma / commit / ld.
//
// Descriptor encodings follow the sm_100 UMMA formats: a K-major operand
// tile stored with the 128-byte swizzle (TMA CU_TENSOR_MAP_SWIZZLE_128B) is
// described by start address >> 4, leading byte offset 1 (unused for swizzled
// K-major), stride byte offset 1024 B >> 4 (between 8-row groups), version 1
// and layout type 2 (128-byte swizzle). Every TMA load here fills only the
// issuing CTA's own shared memory.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace gdn {
namespace tc {

// Error bits a kernel ORs into its caller's status word.
constexpr uint32_t kTimeoutProducer = 1u;
constexpr uint32_t kTimeoutMma = 2u;
constexpr uint32_t kTimeoutEpilogue = 4u;
constexpr uint32_t kTimeoutPrefill = 8u;     // the prefill's stage pipeline
constexpr uint32_t kTimeoutGrid = 16u;       // a grid-wide barrier (one-kernel mixer)
// Every wait gives up after this long (nanoseconds of %globaltimer).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier --------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase with the given parity to complete; false once
// `limit_ns` of %globaltimer have passed without it. The timer is read once
// per kPollsPerCheck polls, so that reading it does not delay noticing the
// phase.
constexpr int kPollsPerCheck = 64;
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < kPollsPerCheck; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_timer() - t0 > limit_ns) return false;
    }
}

// ---- TMA: 2D tiled load global -> shared, completing on an mbarrier --------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(tmap), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---- UMMA descriptors --------------------------------------------------------
// K-major operand tile, 128-byte swizzle, rows of 128 bytes, 8-row groups
// 1024 bytes apart; `addr` must sit on the tile's 1024-byte-aligned base
// plus a K offset that is a multiple of 32 bytes.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);            // start address
    d |= static_cast<uint64_t>(1u) << 16;                          // leading byte offset
    d |= static_cast<uint64_t>(1024u >> 4) << 32;                  // stride byte offset
    d |= static_cast<uint64_t>(1u) << 46;                          // version (sm_100)
    d |= static_cast<uint64_t>(2u) << 61;                          // 128-byte swizzle
    return d;
}
// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4)                                  // D format: f32
         | (1u << 7)                                  // A format: bf16
         | (1u << 10)                                 // B format: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// ---- TMEM --------------------------------------------------------------------
// Whole-warp calls.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(dst_smem), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- MMA (single thread) --------------------------------------------------------
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

// ---- TMEM -> registers: 32 lanes x 32 consecutive 32-bit columns ------------
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
// 32 lanes x 64 consecutive 32-bit columns (one round trip for 64 columns).
__device__ __forceinline__ void tmem_ld_32x32b_x64(uint32_t taddr, uint32_t (&r)[64]) {
    tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- programmatic dependent launch -----------------------------------------
// A kernel launched with programmatic stream serialization may start while
// the previous kernel on the stream still runs; grid_dep_wait blocks the
// calling thread until that kernel has completed and its memory is visible.
// Every read or write of memory an earlier kernel touches comes after it.
__device__ __forceinline__ void grid_dep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Lets the next kernel on the stream begin its prologue.
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Pull one tensor-map box into L2 (a hint: no data reaches the CTA, so it may
// run before grid_dep_wait; a later load still sees every completed write).
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tmap, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
                 ::"l"(tmap), "r"(x), "r"(y) : "memory");
}

// ---- pair-CTA (cta_group::2) forms: one MMA over two SMs of a cluster pair --
// TMA tile load into this CTA's shared memory whose byte count completes on
// `bar`, a shared::cluster address (the pair leader's barrier); only this
// CTA's shared memory is written.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar,
                                                 int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(tmap), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
// Whole-warp calls, by the same warp of both CTAs of the pair.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(dst_smem), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// Issued by the leader: rows [0, 128) of D land in its TMEM, rows [128, 256)
// in the peer's, from A and B halves at the same shared addresses in each.
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on the barrier at this shared offset in every CTA of `cta_mask` once
// the pair MMAs issued so far are done.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;"
        ::"r"(bar), "h"(cta_mask) : "memory");
}
// Arrive on a barrier of another CTA of the cluster (a shared::cluster address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
                 ::"r"(bar_cluster) : "memory");
}

// ---- thread-block clusters: rank, barrier, distributed shared memory -------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster arrives (release) and waits
// (acquire): shared-memory writes before it are visible to the cluster after.
// A hardware barrier, not a spin: every path of the kernel must reach it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The address of this CTA's shared-memory location `addr` in CTA `rank`.
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
    return v;
}

// ---- grid-wide barrier on one 64-bit word of global memory -------------------
// Orders this thread's generic-proxy accesses (global and shared) with
// async-proxy (TMA) ones: a TMA load of data that generic stores wrote, or
// into shared memory that generic stores wrote before.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async;" ::: "memory");
}
// The word holds (tag << 16) | count, where `tag` (48 bits, never 0) names
// one call and so one grid size `n` (a replay repeats both). Install: a CTA that finds the word holding anything but this
// call's tag with a count below `n` replaces it with (tag, 0) -- either
// another call's word or this tag's word left complete by an earlier launch
// of the same call (a CUDA graph replay), never this launch's, which cannot
// reach n before this CTA arrives. Wait: the CTA adds 1 (release) and waits
// (acquire) until the count reaches `n`; the word is left as (tag, n). A CTA
// whose wait runs past kWaitLimitNs clears the word and returns false: the
// others then time out too, and nothing of the failed launch survives it.
// Each CTA installs once (after the previous kernel on the stream has
// completed) and then waits once, on every path, from one thread; every CTA
// of the grid must become resident (n CTAs on distinct SMs, nothing that
// waits on this grid occupying the rest).
__device__ __forceinline__ void grid_barrier_install(unsigned long long* word, uint64_t tag,
                                                     uint32_t n) {
    const unsigned long long mine = static_cast<unsigned long long>(tag) << 16;
    unsigned long long v = *reinterpret_cast<volatile unsigned long long*>(word);
    while (!((v >> 16) == tag && (v & 0xffffull) < n)) {
        const unsigned long long prev = atomicCAS(word, v, mine);
        if (prev == v) break;
        v = prev;
    }
}
__device__ __forceinline__ bool grid_barrier_wait(unsigned long long* word, uint64_t tag,
                                                  uint32_t n, uint64_t limit_ns = kWaitLimitNs) {
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(word) : "memory");
    const uint64_t t0 = global_timer();
    for (int polls = 0;; ++polls) {
        unsigned long long w;
        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(word) : "memory");
        if ((w >> 16) == tag && (w & 0xffffull) >= n) return true;
        if ((polls & 15) == 15 && global_timer() - t0 > limit_ns) break;
        __nanosleep(32);
    }
    atomicExch(word, 0ull);
    return false;
}

}  // namespace tc
}  // namespace gdn
