// gdn_selftest.cu -- checks of the library's failure detection on the GPU.
//
// Every tcgen05 kernel of the library waits on mbarriers through
// tc::mbar_wait, which gives up after a time limit and lets the kernel
// record an error bit and return instead of hanging. bounded_wait_kernel
// exercises exactly that path: one thread waits on an mbarrier that expects
// one arrival; with `arrive` = 0 nothing ever arrives, so the wait must run
// out after `limit_ns`, and the kernel reports the timeout bit and the time
// it waited. With `arrive` = 1 the thread arrives first and the wait returns
// at once. grid_barrier_kernel does the same for the one-kernel short-conv
// mixer's grid-wide barrier (tc::grid_barrier_install / _wait): `ctas` CTAs
// meet on a caller's word expecting `expect` arrivals; with expect > ctas the
// count never gets there and every wait must run out. Nothing faults, traps
// or spins without a bound.
#include <cstdio>

#include <cuda_runtime.h>

#include "gdn.h"
#include "gdn_internal.h"
#include "gdn_tc.cuh"

namespace gdn {
namespace {

__global__ void bounded_wait_kernel(uint32_t* __restrict__ result, uint64_t limit_ns,
                                    int arrive) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = tc::smem_u32(&bar);
    tc::mbar_init(b, 1);
    tc::fence_mbar_init();
    if (arrive) tc::mbar_arrive(b);
    const uint64_t t0 = tc::global_timer();
    const bool ok = tc::mbar_wait(b, 0, limit_ns);
    const uint64_t waited = tc::global_timer() - t0;
    result[0] = ok ? 0u : tc::kTimeoutProducer;
    result[1] = static_cast<uint32_t>(waited / 1000u);        // microseconds
}

__global__ void grid_barrier_kernel(unsigned long long* word, uint32_t* __restrict__ result,
                                    uint64_t tag, uint32_t expect, uint64_t limit_ns) {
    if (threadIdx.x != 0) return;
    tc::grid_barrier_install(word, tag, expect);
    const uint64_t t0 = tc::global_timer();
    const bool ok = tc::grid_barrier_wait(word, tag, expect, limit_ns);
    const uint64_t waited = tc::global_timer() - t0;
    result[blockIdx.x] = ok ? 0u : tc::kTimeoutGrid;
    result[gridDim.x + blockIdx.x] = static_cast<uint32_t>(waited / 1000u);   // microseconds
}

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_selftest_grid_barrier(unsigned long long* word, uint32_t* result,
                                                uint64_t tag, int ctas, int expect,
                                                uint64_t limit_ns, void* stream) {
    if (!word || !result) return static_cast<gdn_status>(
        gdn::report_error(GDN_ERR_NULL, "gdn_selftest_grid_barrier: word or result is NULL"));
    if (ctas < 1 || ctas > 32 || expect < 1 || expect > 64 || tag == 0 || (tag >> 48) != 0 ||
        limit_ns == 0 || limit_ns > gdn::tc::kWaitLimitNs)
        return static_cast<gdn_status>(gdn::report_error(
            GDN_ERR_UNSUPPORTED, "gdn_selftest_grid_barrier: need 1 <= ctas <= 32, "
                                 "1 <= expect <= 64, 0 < tag < 2^48, limit_ns in (0, 2e9]"));
    if (reinterpret_cast<uintptr_t>(word) % 8 != 0 || reinterpret_cast<uintptr_t>(result) % 4 != 0)
        return static_cast<gdn_status>(gdn::report_error(
            GDN_ERR_ALIGN, "gdn_selftest_grid_barrier: word or result is misaligned"));
    gdn::grid_barrier_kernel<<<ctas, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        word, result, tag, static_cast<uint32_t>(expect), limit_ns);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "gdn_selftest_grid_barrier: %s", cudaGetErrorString(err));
        return static_cast<gdn_status>(gdn::report_error(GDN_ERR_CUDA, msg));
    }
    gdn::report_error(GDN_OK, "");
    return GDN_OK;
}

extern "C" gdn_status gdn_selftest_bounded_wait(uint32_t* result, uint64_t limit_ns, int arrive,
                                                void* stream) {
    if (!result) return static_cast<gdn_status>(
        gdn::report_error(GDN_ERR_NULL, "gdn_selftest_bounded_wait: result is NULL"));
    if (limit_ns == 0 || limit_ns > gdn::tc::kWaitLimitNs)
        return static_cast<gdn_status>(gdn::report_error(
            GDN_ERR_UNSUPPORTED, "gdn_selftest_bounded_wait: limit_ns must be in (0, 2e9]"));
    if (reinterpret_cast<uintptr_t>(result) % 4 != 0)
        return static_cast<gdn_status>(
            gdn::report_error(GDN_ERR_ALIGN, "gdn_selftest_bounded_wait: result is misaligned"));
    gdn::bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(result, limit_ns,
                                                                            arrive ? 1 : 0);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof(msg), "gdn_selftest_bounded_wait: %s", cudaGetErrorString(err));
        return static_cast<gdn_status>(gdn::report_error(GDN_ERR_CUDA, msg));
    }
    gdn::report_error(GDN_OK, "");
    return GDN_OK;
}
