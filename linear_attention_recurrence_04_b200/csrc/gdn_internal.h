// gdn_internal.h -- launchers behind the C ABI (not exported).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace gdn {

struct StepArgs {
    float* state;
    const float* q;
    const float* k;
    const float* v;
    const float* beta;
    const float* gate;
    float* out;
    int64_t n_heads;   // L * B * Hv
    int Hk;
    int Hv;
};

struct PrefillArgs {
    float* state;
    const float* q;
    const float* k;
    const float* v;
    const float* beta;
    const float* gate;
    float* out;
    int64_t B;
    int64_t T;
    int Hk;
    int Hv;
    // Elements between consecutive positions of q and k, of v, and of
    // beta/gate; 0 selects the contiguous layouts [B][T][Hk][dk],
    // [B][T][Hv][dv] and [B][T][Hv].
    int64_t qk_stride = 0;
    int64_t v_stride = 0;
    int64_t bg_stride = 0;
    uint32_t* status = nullptr;   // optional device word for timeout bits
};

struct LayerArgs {
    const float* mixed_qkv;
    const float* z;
    const float* a;
    const float* b;
    float* conv_ring;
    const float* conv_w;
    const float* A_log;
    const float* dt_bias;
    const float* norm_w;
    float l2_eps;
    float norm_eps;
    float* state;
    float* out;
    int64_t B;
    int Hk;
    int Hv;
    float* scratch_ring;    // pair only: ring after the tentative position
    float* scratch_state;   // pair only: state after the tentative position
};

struct LinearArgs {
    const void* x;     // [M][K] bf16
    const void* w;     // [N][K] bf16
    float* y;          // [M][N]
    int64_t M;
    int64_t N;
    int64_t K;
    uint32_t* status;  // optional device word for timeout bits
};

struct ForwardBatchArgs {
    const void* hidden;    // [B][T][D] bf16
    const void* w_qkv;     // [C][D] bf16
    const void* w_z;       // [Hv*dv][D] bf16
    const void* w_ba;      // [2*Hv][D] bf16: rows 0..Hv-1 give b, Hv..2Hv-1 give a
    const void* w_out;     // [D][Hv*dv] bf16
    float* conv_ring;
    const float* conv_w;
    const float* A_log;
    const float* dt_bias;
    const float* norm_w;
    float l2_eps;
    float norm_eps;
    float* state;
    float* out;            // [B][T][D]
    void* workspace;
    int64_t B;
    int64_t T;
    int64_t D;
    int Hk;
    int Hv;
    uint32_t* status;
};

// Byte offsets of the forward-batch intermediates inside the workspace.
struct ForwardBatchLayout {
    size_t act, z, ba, beta, gate, o, y, halo, total;
};
ForwardBatchLayout forward_batch_layout(int64_t B, int64_t T, int Hk, int Hv);

// The LFM2 short-conv mixer over T positions (gdn_short_conv.cu).
struct ShortConvArgs {
    const void* hidden;    // [B][T][D] bf16
    const void* w_in;      // [3D][D] bf16: input gate | output gate | value rows
    const void* w_out;     // [D][D] bf16
    float* conv_ring;      // [B][K-1][D] gated inputs, oldest first (in/out)
    float* scratch_ring;   // [B][K-1][D] ring after the last position, or null
    const float* conv_w;   // [D][K]
    float* out;            // [B][T][D] fp32
    void* workspace;       // short_conv_layout(B, T, D).total bytes, 256-aligned
    int64_t B, T, D;
    int K;                 // 2, 3 or 4
    int64_t n_commit;      // conv_ring receives the ring after position n_commit - 1
    uint32_t* status;
};
struct ShortConvLayout {
    size_t proj, y, bar, total;   // bar: the one-kernel form's barrier word
};
// Calls of at most 128 rows (B*T): the input projection, split over K in a
// cluster, with the gate and conv as its epilogue -- y (bf16, [B*T][D]) and
// both rings are written, proj is not. cudaErrorNotSupported when the call
// is larger or the product too small to split (use the separate kernels).
cudaError_t launch_short_conv_in_gate(const ShortConvArgs& a, void* y, cudaStream_t stream);
// Calls of one or two positions and at most 128 rows: the whole mixer as one
// kernel (both projections split as above, a grid-wide barrier on the word
// `bar` of the workspace between the conv and the output projection).
// cudaErrorNotSupported when the shape does not fit that form.
cudaError_t launch_short_conv_fused(const ShortConvArgs& a, void* y, unsigned long long* bar,
                                    cudaStream_t stream);
ShortConvLayout short_conv_layout(int64_t B, int64_t T, int64_t D);

// Each launcher enqueues its kernel on `stream` and returns the launch status.
cudaError_t launch_step(const StepArgs& a, cudaStream_t stream);
// KDA core: StepArgs / PrefillArgs with `gate` holding a log-decay per key
// channel, [..][Hv][dk] (contiguous).
cudaError_t launch_kda_step(const StepArgs& a, cudaStream_t stream);
cudaError_t launch_kda_prefill(const PrefillArgs& a, cudaStream_t stream);
// Two-position verify: StepArgs with q, k, v, beta, gate and out holding two
// positions per sequence ([L][B][2][..]); the state after position 0 goes to
// a.state, the state after position 1 to `scratch`.
cudaError_t launch_pair(const StepArgs& a, float* scratch, cudaStream_t stream);
cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream);
cudaError_t launch_layer_decode(const LayerArgs& a, cudaStream_t stream);
cudaError_t launch_layer_pair(const LayerArgs& a, cudaStream_t stream);
cudaError_t launch_linear_bf16(const LinearArgs& a, cudaStream_t stream);
// The same product for M <= 128 split over K across a thread-block cluster
// (fixed per (N, K) and device; rows are identical across such calls, and
// differ from launch_linear_bf16's by accumulation order); M > 128, or a
// product too small to split, goes to launch_linear_bf16.
cudaError_t launch_linear_bf16_split(const LinearArgs& a, cudaStream_t stream);
cudaError_t launch_forward_batch(const ForwardBatchArgs& a, cudaStream_t stream);
cudaError_t launch_short_conv(const ShortConvArgs& a, cudaStream_t stream);

// Value-heads-per-key-head ratios the fused layer kernel is compiled for.
bool layer_decode_supports(int G);

// Records `message` as this host thread's gdn_last_error() text and returns
// `status` (for entry points defined outside gdn_api.cu).
int report_error(int status, const char* message);

// Number of SMs of the current device, cached per device.
int device_sm_count();

// Resident CTAs per SM of `kernel` at `threads` threads and no dynamic shared
// memory on the current device (at least 1), cached per (device, kernel) so a
// launch inside stream capture makes no occupancy query.
cudaError_t resident_ctas_per_sm(const void* kernel, int threads, int* per_sm);

}  // namespace gdn
