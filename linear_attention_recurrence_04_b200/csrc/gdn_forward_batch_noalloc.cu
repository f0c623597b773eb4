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
// the device address is obtained with cudaGetSymbolAddress (with the device
// current) and passed to the kernels like any workspace. The address belongs
// to one CUDA context: it is cached per device together with the driver's ID
// of the context it was looked up in, and looked up again when the current
// context has another ID (after cudaDeviceReset, or in a context the caller
// created). The first call in a context performs that lookup; make it before
// any stream capture. All calls share the one array, so two calls whose work
// overlaps on the GPU (different streams, or different host threads on one
// device) race on it: order them. Nothing in the array needs to start at
// zero -- every intermediate is written before it is read -- so nothing is
// cleared between calls.
#include <cstdio>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gdn.h"
#include "gdn_common.cuh"
#include "gdn_internal.h"

// The built-in scratch: 16 MiB. At the pages' geometry (Hk = 16, Hv = 32,
// dk = dv = 128) a call needs about 72.5 KiB per position plus 96 KiB per
// started 32-position tile of each sequence, so it holds B = 1 with
// T <= 216, B = 67 with T = 2 and B = 97 with T = 1.
static constexpr size_t kStaticScratchBytes = static_cast<size_t>(16) << 20;
static __device__ __align__(256) unsigned char g_forward_scratch[kStaticScratchBytes];

namespace gdn {
namespace {

constexpr int kMaxDevices = 64;

struct ScratchEntry {
    unsigned long long ctx_id = 0;      // driver context ID the address belongs to (0: none)
    void* address = nullptr;
};
std::mutex g_scratch_mutex;
ScratchEntry g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The driver's unique ID of the current context, or 0 when there is none or
// the driver does not provide the query (then nothing is cached).
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                    cudaSuccess && q == cudaDriverEntryPointSuccess)
                   ? reinterpret_cast<CtxGetCurrentFn>(p) : nullptr;
    }();
    static CtxGetIdFn get_id = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        return (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) ==
                    cudaSuccess && q == cudaDriverEntryPointSuccess)
                   ? reinterpret_cast<CtxGetIdFn>(p) : nullptr;
    }();
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_forward_scratch in the current context of the current
// device (looked up once per context).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    const bool cacheable = dev >= 0 && dev < kMaxDevices;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    const unsigned long long ctx = current_context_id();
    if (cacheable && ctx != 0 && g_scratch[dev].ctx_id == ctx) {
        *out = g_scratch[dev].address;
        return cudaSuccess;
    }
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_forward_scratch);   // also makes the context current
    if (err != cudaSuccess) return err;
    if (cacheable) g_scratch[dev] = ScratchEntry{current_context_id(), p};
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
