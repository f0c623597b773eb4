// gdn_selftest.cu -- a check of the library's failure detection on the GPU.
//
// Every tcgen05 kernel of the library waits on mbarriers through
// tc::mbar_wait, which gives up after a time limit and lets the kernel
// record an error bit and return instead of hanging. This kernel exercises
// exactly that path: one thread waits on an mbarrier that expects one
// arrival; with `arrive` = 0 nothing ever arrives, so the wait must run out
// after `limit_ns`, and the kernel reports the timeout bit and the time it
// waited. With `arrive` = 1 the thread arrives first and the wait returns at
// once. Nothing faults, traps or spins without a bound.
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

}  // namespace
}  // namespace gdn

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
