// gdn_forward_batch_noalloc.cu -- gdn_forward_batch for callers that cannot
// allocate device memory.
//
// gdn_forward_batch needs a scratch workspace for its intermediates (the
// projections, the conv output, the gates, the recurrence output and the
// bf16 tail). Most callers allocate it with cudaMalloc or their framework's
// allocator. Some cannot: code that runs as a plugin inside a host program
// which owns every device allocation and offers no allocation hook, code
// restricted to a fixed memory budget set up before it runs, or a
// latency-critical path where an allocation (and a possible device-wide
// synchronisation) is not allowed. This entry point gives them the same
// layer with the workspace taken from a fixed array that lives in the
// library itself.
//
// The array below is a file-scope __device__ object: every GPU that loads
// this library holds its 16 MiB until the process exits, whether or not the
// entry point is used. In host code its name is only a host-side handle, so
// the device address is obtained once per device with cudaGetSymbolAddress
// (with that device current) and passed to the kernels like any workspace.
// The first call on a device performs that lookup; make it before any stream
// capture. All calls share the one array, so two calls whose work overlaps
// on the GPU (different streams, or different host threads on one device)
// race on it: order them. Nothing in the array needs to start at zero --
// every intermediate is written before it is read -- so nothing is cleared
// between calls.
#include <atomic>
#include <cstdio>

#include <cuda_runtime.h>

#include "gdn.h"
#include "gdn_common.cuh"
#include "gdn_internal.h"

// The built-in scratch: 16 MiB, enough for about 215 positions of the
// pages' geometry (Hk = 16, Hv = 32, dk = dv = 128).
static constexpr size_t kStaticScratchBytes = static_cast<size_t>(16) << 20;
static __device__ __align__(256) unsigned char g_forward_scratch[kStaticScratchBytes];

namespace gdn {
namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_address[kMaxDevices];

// Device address of g_forward_scratch on the current device (looked up once
// per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < kMaxDevices) {
        void* cached = g_scratch_address[dev].load(std::memory_order_acquire);
        if (cached) {
            *out = cached;
            return cudaSuccess;
        }
    }
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_forward_scratch);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < kMaxDevices) g_scratch_address[dev].store(p, std::memory_order_release);
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_forward_batch_noalloc(
    const void* hidden, const void* w_qkv, const void* w_z, const void* w_ba, const void* w_out,
    float* conv_ring, const float* conv_w, const float* A_log, const float* dt_bias,
    const float* norm_w, float l2_eps, float norm_eps, float* state, float* out, int64_t B,
    int64_t T, int64_t D, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, int64_t K,
    uint32_t* status, void* stream) {
    void* ws = nullptr;
    if (B > 0 && T > 0) {
        const size_t need = gdn_forward_batch_workspace_size(B, T, Hk, Hv, dk, dv);
        if (need > kStaticScratchBytes) {
            char msg[256];
            snprintf(msg, sizeof(msg),
                     "gdn_forward_batch_noalloc: B*T=%lld positions need %zu bytes of scratch; "
                     "the built-in scratch holds %zu bytes (use gdn_forward_batch with a "
                     "workspace for larger batches)",
                     static_cast<long long>(B * T), need, kStaticScratchBytes);
            return static_cast<gdn_status>(gdn::report_error(GDN_ERR_UNSUPPORTED, msg));
        }
        // need == 0 flags an invalid shape; gdn_forward_batch reports it.
        cudaError_t err = gdn::scratch_address(&ws);
        if (err != cudaSuccess) {
            char msg[256];
            snprintf(msg, sizeof(msg),
                     "gdn_forward_batch_noalloc: looking up the built-in scratch failed: %s",
                     cudaGetErrorString(err));
            return static_cast<gdn_status>(gdn::report_error(GDN_ERR_CUDA, msg));
        }
    }
    return gdn_forward_batch(hidden, w_qkv, w_z, w_ba, w_out, conv_ring, conv_w, A_log, dt_bias,
                             norm_w, l2_eps, norm_eps, state, out, ws, kStaticScratchBytes,
                             B, T, D, Hk, Hv, dk, dv, K, status, stream);
}
