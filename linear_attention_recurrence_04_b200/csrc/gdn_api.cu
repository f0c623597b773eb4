// gdn_api.cu -- the extern "C" entry points of libgdn.so (declared in
// include/gdn.h): host-side argument checks, then one kernel launch each.
#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "gdn.h"
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

thread_local char g_last_error[512] = "";
// The text of the last GDN_ERR_CUDA on this thread; kept until the next one.
thread_local char g_last_cuda_error[512] = "";

// An NVTX range over one entry point (named after it), so a timeline tool
// shows each library call; free when no tool is attached.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

gdn_status fail(gdn_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    if (st == GDN_ERR_CUDA) snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s", g_last_error);
    return st;
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

// Checked product of non-negative sizes; false on overflow of int64.
bool mul_ok(int64_t a, int64_t b, int64_t* r) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *r = a * b;
    return true;
}

struct Span {
    const void* p;
    int64_t bytes;
    const char* name;
};

bool overlaps(const Span& x, const Span& y) {
    if (!x.p || !y.p || x.bytes == 0 || y.bytes == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(x.p), a1 = a0 + x.bytes;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(y.p), b1 = b0 + y.bytes;
    return a0 < b1 && b0 < a1;
}

bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

gdn_status check_geometry(int64_t Hk, int64_t Hv, int64_t dk, int64_t dv) {
    if (Hk <= 0 || Hv <= 0) return fail(GDN_ERR_SHAPE, "Hk=%lld and Hv=%lld must be positive",
                                        (long long)Hk, (long long)Hv);
    if (Hv % Hk != 0) return fail(GDN_ERR_SHAPE, "Hv=%lld is not a multiple of Hk=%lld",
                                  (long long)Hv, (long long)Hk);
    if (dk != kDk || dv != kDv)
        return fail(GDN_ERR_UNSUPPORTED, "dk=%lld dv=%lld: only dk = dv = 128 is implemented",
                    (long long)dk, (long long)dv);
    if (Hv > (1 << 20)) return fail(GDN_ERR_OVERFLOW, "Hv=%lld is too large", (long long)Hv);
    return GDN_OK;
}

// `out` must not overlap anything; a buffer updated in place (the first
// `n_inplace` entries of `in`) must not overlap any other entry either.
gdn_status check_spans(const Span* in, int n_in, int n_inplace, const Span& out) {
    for (int i = 0; i < n_in; ++i)
        if (overlaps(in[i], out))
            return fail(GDN_ERR_ALIAS, "out overlaps %s", in[i].name);
    for (int i = 0; i < n_inplace; ++i)
        for (int j = 0; j < n_in; ++j)
            if (j != i && overlaps(in[i], in[j]))
                return fail(GDN_ERR_ALIAS, "%s (updated in place) overlaps %s", in[i].name,
                            in[j].name);
    return GDN_OK;
}

gdn_status launched(cudaError_t err, const char* what) {
    if (err != cudaSuccess)
        return fail(GDN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(err),
                    cudaGetErrorName(err));
    g_last_error[0] = '\0';
    return GDN_OK;
}

}  // namespace

int report_error(int status, const char* message) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", message);
    if (status == GDN_ERR_CUDA) snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s", message);
    return status;
}

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < kMaxDevices) {
        const int cached = g_sm_count[dev].load(std::memory_order_relaxed);
        if (cached > 0) return cached;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < kMaxDevices) g_sm_count[dev].store(n, std::memory_order_relaxed);
    return n;
}

namespace {

struct OccEntry {
    std::atomic<const void*> kernel{nullptr};
    std::atomic<int> threads{0};
    std::atomic<int> per_sm{0};
};
constexpr int kOccSlots = 16;
OccEntry g_occ[kMaxDevices][kOccSlots];

}  // namespace

cudaError_t resident_ctas_per_sm(const void* kernel, int threads, int* per_sm) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < kMaxDevices) {
        for (int i = 0; i < kOccSlots; ++i) {
            OccEntry& e = g_occ[dev][i];
            if (e.kernel.load(std::memory_order_acquire) == kernel &&
                e.threads.load(std::memory_order_relaxed) == threads) {
                const int v = e.per_sm.load(std::memory_order_relaxed);
                if (v > 0) { *per_sm = v; return cudaSuccess; }
            }
        }
    }
    int n = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0);
    if (err != cudaSuccess) return err;
    if (n < 1) n = 1;
    *per_sm = n;
    if (dev >= 0 && dev < kMaxDevices) {
        for (int i = 0; i < kOccSlots; ++i) {
            OccEntry& e = g_occ[dev][i];
            const void* expected = nullptr;
            if (e.kernel.compare_exchange_strong(expected, kernel, std::memory_order_acq_rel) ||
                expected == kernel) {
                e.threads.store(threads, std::memory_order_relaxed);
                e.per_sm.store(n, std::memory_order_relaxed);
                break;
            }
        }
    }
    return cudaSuccess;
}

}  // namespace gdn

using namespace gdn;

extern "C" {

const char* gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "ok";
        case GDN_ERR_NULL: return "a required pointer is NULL";
        case GDN_ERR_SHAPE: return "invalid shape";
        case GDN_ERR_UNSUPPORTED: return "unsupported geometry";
        case GDN_ERR_ALIGN: return "misaligned pointer";
        case GDN_ERR_OVERFLOW: return "size overflow";
        case GDN_ERR_CUDA: return "CUDA launch error";
        case GDN_ERR_ALIAS: return "output overlaps an input";
        default: return "unknown status";
    }
}

const char* gdn_last_error(void) { return g_last_error; }

const char* gdn_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"

namespace {

// Checks shared by the decode entries: gdn_step (one log-decay per head,
// gate_w = 1) and gdn_kda_step (one per head and key channel, gate_w = dk).
gdn_status step_call(const char* fn, float* state, const float* q, const float* k,
                     const float* v, const float* beta, const float* gate, float* out,
                     int64_t L, int64_t B, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                     bool channel_decay, void* stream) {
    NvtxRange nvtx_range(fn);
    if (L < 0 || B < 0) return fail(GDN_ERR_SHAPE, "%s: negative L=%lld or B=%lld", fn,
                                    (long long)L, (long long)B);
    gdn_status st = check_geometry(Hk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    int64_t lb = 0, heads = 0, state_n = 0, qk_n = 0, v_n = 0, gate_n = 0;
    if (!mul_ok(L, B, &lb) || !mul_ok(lb, Hv, &heads) || !mul_ok(heads, dv * dk, &state_n) ||
        !mul_ok(lb, Hk * dk, &qk_n) || !mul_ok(heads, dv, &v_n) ||
        !mul_ok(heads, channel_decay ? dk : 1, &gate_n) || state_n > INT64_MAX / 8)
        return fail(GDN_ERR_OVERFLOW, "%s: L*B*Hv*dv*dk overflows int64", fn);
    if (heads == 0) { g_last_error[0] = '\0'; return GDN_OK; }
    if (!state || !q || !k || !v || !beta || !gate || !out)
        return fail(GDN_ERR_NULL, "%s: a tensor pointer is NULL", fn);
    if (!aligned(state, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(out, 16) || !aligned(beta, 4) || !aligned(gate, channel_decay ? 16 : 4))
        return fail(GDN_ERR_ALIGN, "%s: state/q/k/v/out%s need 16-byte, beta%s 4-byte alignment",
                    fn, channel_decay ? "/g" : "", channel_decay ? "" : "/gate");
    const Span ins[] = {{state, state_n * 4, "state"}, {q, qk_n * 4, "q"}, {k, qk_n * 4, "k"},
                        {v, v_n * 4, "v"}, {beta, heads * 4, "beta"},
                        {gate, gate_n * 4, channel_decay ? "g" : "gate"}};
    st = check_spans(ins, 6, 1, Span{out, v_n * 4, "out"});
    if (st != GDN_OK) return st;
    StepArgs a{state, q, k, v, beta, gate, out, heads, static_cast<int>(Hk), static_cast<int>(Hv)};
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return launched(channel_decay ? launch_kda_step(a, s) : launch_step(a, s), fn);
}

// gdn_pair: the checks of gdn_step with two positions per sequence and a
// second state-sized output.
gdn_status pair_call(const char* fn, float* state, float* scratch, const float* q,
                     const float* k, const float* v, const float* beta, const float* gate,
                     float* out, int64_t L, int64_t B, int64_t Hk, int64_t Hv, int64_t dk,
                     int64_t dv, void* stream) {
    NvtxRange nvtx_range(fn);
    if (L < 0 || B < 0) return fail(GDN_ERR_SHAPE, "%s: negative L=%lld or B=%lld", fn,
                                    (long long)L, (long long)B);
    gdn_status st = check_geometry(Hk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    int64_t lb = 0, heads = 0, state_n = 0, qk_n = 0, v_n = 0;
    if (!mul_ok(L, B, &lb) || !mul_ok(lb, Hv, &heads) || !mul_ok(heads, dv * dk, &state_n) ||
        !mul_ok(lb, 2 * Hk * dk, &qk_n) || !mul_ok(heads, 2 * dv, &v_n) ||
        state_n > INT64_MAX / 8 || qk_n > INT64_MAX / 8 || v_n > INT64_MAX / 8)
        return fail(GDN_ERR_OVERFLOW, "%s: L*B*Hv*dv*dk overflows int64", fn);
    if (heads == 0) { g_last_error[0] = '\0'; return GDN_OK; }
    if (!state || !scratch || !q || !k || !v || !beta || !gate || !out)
        return fail(GDN_ERR_NULL, "%s: a tensor pointer is NULL", fn);
    if (!aligned(state, 16) || !aligned(scratch, 16) || !aligned(q, 16) || !aligned(k, 16) ||
        !aligned(v, 16) || !aligned(out, 16) || !aligned(beta, 4) || !aligned(gate, 4))
        return fail(GDN_ERR_ALIGN,
                    "%s: state/scratch_state/q/k/v/out need 16-byte, beta/gate 4-byte alignment",
                    fn);
    const Span ins[] = {{state, state_n * 4, "state"}, {q, qk_n * 4, "q"}, {k, qk_n * 4, "k"},
                        {v, v_n * 4, "v"}, {beta, heads * 2 * 4, "beta"},
                        {gate, heads * 2 * 4, "gate"}, {out, v_n * 4, "out"}};
    st = check_spans(ins, 6, 1, Span{out, v_n * 4, "out"});
    if (st != GDN_OK) return st;
    st = check_spans(ins, 7, 1, Span{scratch, state_n * 4, "scratch_state"});
    if (st != GDN_OK) return st;
    StepArgs a{state, q, k, v, beta, gate, out, heads, static_cast<int>(Hk), static_cast<int>(Hv)};
    return launched(launch_pair(a, scratch, static_cast<cudaStream_t>(stream)), fn);
}

// Checks shared by the multi-position entries gdn_prefill and gdn_kda_prefill.
gdn_status prefill_call(const char* fn, float* state, const float* q, const float* k,
                        const float* v, const float* beta, const float* gate, float* out,
                        int64_t B, int64_t T, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                        bool channel_decay, uint32_t* status, void* stream) {
    NvtxRange nvtx_range(fn);
    if (B < 0 || T < 0) return fail(GDN_ERR_SHAPE, "%s: negative B=%lld or T=%lld", fn,
                                    (long long)B, (long long)T);
    gdn_status st = check_geometry(Hk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    int64_t bt = 0, heads = 0, state_n = 0, qk_n = 0, v_n = 0, bh = 0, gate_n = 0;
    if (!mul_ok(B, T, &bt) || !mul_ok(B, Hv, &heads) || !mul_ok(heads, dv * dk, &state_n) ||
        !mul_ok(bt, Hk * dk, &qk_n) || !mul_ok(bt, Hv * dv, &v_n) || !mul_ok(bt, Hv, &bh) ||
        !mul_ok(bh, channel_decay ? dk : 1, &gate_n) || v_n > INT64_MAX / 8 ||
        qk_n > INT64_MAX / 8 || gate_n > INT64_MAX / 8)
        return fail(GDN_ERR_OVERFLOW, "%s: B*T*Hv*dv overflows int64", fn);
    // One warp per 8 rows of a head (pair); the grid must fit gridDim.x.
    if (heads * (kDv / 8) > INT32_MAX)
        return fail(GDN_ERR_OVERFLOW, "%s: B*Hv=%lld exceeds the launch grid", fn,
                    (long long)heads);
    if (bt == 0 || heads == 0) { g_last_error[0] = '\0'; return GDN_OK; }
    if (!state || !q || !k || !v || !beta || !gate || !out)
        return fail(GDN_ERR_NULL, "%s: a tensor pointer is NULL", fn);
    if (!aligned(state, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(out, 16) || !aligned(beta, 4) || !aligned(gate, channel_decay ? 16 : 4))
        return fail(GDN_ERR_ALIGN, "%s: state/q/k/v/out%s need 16-byte, beta%s 4-byte alignment",
                    fn, channel_decay ? "/g" : "", channel_decay ? "" : "/gate");
    const Span ins[] = {{state, state_n * 4, "state"}, {q, qk_n * 4, "q"}, {k, qk_n * 4, "k"},
                        {v, v_n * 4, "v"}, {beta, bh * 4, "beta"},
                        {gate, gate_n * 4, channel_decay ? "g" : "gate"}};
    st = check_spans(ins, 6, 1, Span{out, v_n * 4, "out"});
    if (st != GDN_OK) return st;
    if (status && !aligned(status, 4))
        return fail(GDN_ERR_ALIGN, "%s: status needs 4-byte alignment", fn);
    PrefillArgs a{state, q, k, v, beta, gate, out, B, T, static_cast<int>(Hk), static_cast<int>(Hv)};
    a.status = status;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    return launched(channel_decay ? launch_kda_prefill(a, s) : launch_prefill(a, s), fn);
}

}  // namespace

extern "C" {

gdn_status gdn_step(float* state, const float* q, const float* k, const float* v,
                    const float* beta, const float* gate, float* out, int64_t L, int64_t B,
                    int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, void* stream) {
    return step_call("gdn_step", state, q, k, v, beta, gate, out, L, B, Hk, Hv, dk, dv, false,
                     stream);
}

gdn_status gdn_prefill(float* state, const float* q, const float* k, const float* v,
                       const float* beta, const float* gate, float* out, int64_t B, int64_t T,
                       int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, uint32_t* status,
                       void* stream) {
    return prefill_call("gdn_prefill", state, q, k, v, beta, gate, out, B, T, Hk, Hv, dk, dv,
                        false, status, stream);
}

gdn_status gdn_pair(float* state, float* scratch_state, const float* q, const float* k,
                    const float* v, const float* beta, const float* gate, float* out, int64_t L,
                    int64_t B, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, void* stream) {
    return pair_call("gdn_pair", state, scratch_state, q, k, v, beta, gate, out, L, B, Hk, Hv, dk,
                     dv, stream);
}

gdn_status gdn_kda_step(float* state, const float* q, const float* k, const float* v,
                        const float* beta, const float* g, float* out, int64_t L, int64_t B,
                        int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, void* stream) {
    return step_call("gdn_kda_step", state, q, k, v, beta, g, out, L, B, Hk, Hv, dk, dv, true,
                     stream);
}

gdn_status gdn_kda_prefill(float* state, const float* q, const float* k, const float* v,
                           const float* beta, const float* g, float* out, int64_t B, int64_t T,
                           int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, void* stream) {
    return prefill_call("gdn_kda_prefill", state, q, k, v, beta, g, out, B, T, Hk, Hv, dk, dv,
                        true, nullptr, stream);
}

namespace {

// Shared checks of the fused layer entry points; npos = 1 (decode) or 2 (pair).
gdn_status check_layer(const char* fn, int npos, const float* mixed_qkv, const float* z,
                       const float* a, const float* b, const float* conv_ring,
                       const float* conv_w, const float* A_log, const float* dt_bias,
                       const float* norm_w, const float* state, const float* scratch_ring,
                       const float* scratch_state, const float* out, int64_t B, int64_t Hk,
                       int64_t Hv, int64_t dk, int64_t dv, int64_t K, bool* empty) {
    *empty = false;
    if (B < 0) return fail(GDN_ERR_SHAPE, "%s: negative B=%lld", fn, (long long)B);
    gdn_status st = check_geometry(Hk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    if (K != kConvK) return fail(GDN_ERR_UNSUPPORTED, "%s: K=%lld: only a conv kernel of 4 is implemented",
                                 fn, (long long)K);
    if (!layer_decode_supports(static_cast<int>(Hv / Hk)))
        return fail(GDN_ERR_UNSUPPORTED, "%s: Hv/Hk=%lld: the fused layer supports 1, 2 or 4",
                    fn, (long long)(Hv / Hk));
    const int64_t C = 2 * Hk * dk + Hv * dv;
    int64_t x_n = 0, z_n = 0, bh = 0, ring_n = 0, state_n = 0, grid = 0;
    if (!mul_ok(B * npos, C, &x_n) || !mul_ok(B * npos, Hv * dv, &z_n) ||
        !mul_ok(B * npos, Hv, &bh) || !mul_ok(B, (K - 1) * C, &ring_n) ||
        !mul_ok(B * Hv, dv * dk, &state_n) || !mul_ok(B, Hk, &grid) ||
        B > INT64_MAX / 8 / Hv || state_n > INT64_MAX / 8 || ring_n > INT64_MAX / 8)
        return fail(GDN_ERR_OVERFLOW, "%s: B*Hv*dv*dk overflows int64", fn);
    if (grid > INT32_MAX) return fail(GDN_ERR_OVERFLOW, "%s: B*Hk=%lld exceeds the launch grid",
                                      fn, (long long)grid);
    if (B == 0) { *empty = true; return GDN_OK; }
    if (!mixed_qkv || !z || !a || !b || !conv_ring || !conv_w || !A_log || !dt_bias || !norm_w ||
        !state || !out || (npos == 2 && (!scratch_ring || !scratch_state)))
        return fail(GDN_ERR_NULL, "%s: a tensor pointer is NULL", fn);
    if (!aligned(mixed_qkv, 16) || !aligned(z, 16) || !aligned(conv_ring, 16) ||
        !aligned(conv_w, 16) || !aligned(state, 16) || !aligned(out, 16) || !aligned(a, 4) ||
        !aligned(b, 4) || !aligned(A_log, 4) || !aligned(dt_bias, 4) || !aligned(norm_w, 4) ||
        (npos == 2 && (!aligned(scratch_ring, 16) || !aligned(scratch_state, 16))))
        return fail(GDN_ERR_ALIGN, "%s: alignment rule violated", fn);
    const Span ins[] = {{state, state_n * 4, "state"}, {conv_ring, ring_n * 4, "conv_ring"},
                        {scratch_state, npos == 2 ? state_n * 4 : 0, "scratch_state"},
                        {scratch_ring, npos == 2 ? ring_n * 4 : 0, "scratch_ring"},
                        {mixed_qkv, x_n * 4, "mixed_qkv"}, {z, z_n * 4, "z"}, {a, bh * 4, "a"},
                        {b, bh * 4, "b"}, {conv_w, C * K * 4, "conv_w"},
                        {A_log, Hv * 4, "A_log"}, {dt_bias, Hv * 4, "dt_bias"},
                        {norm_w, dv * 4, "norm_w"}};
    return check_spans(ins, 12, 4, Span{out, z_n * 4, "out"});
}


// Checks shared by the two projection entries; `split` selects the split-K
// launcher for products of at most 128 rows.
gdn_status linear_call(const char* fn, const void* x, const void* w, float* y, int64_t M,
                       int64_t N, int64_t K, uint32_t* status, void* stream, bool split) {
    if (M < 0 || N < 0 || K < 0)
        return fail(GDN_ERR_SHAPE, "%s: negative M=%lld N=%lld K=%lld", fn, (long long)M,
                    (long long)N, (long long)K);
    if (K % 8 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "%s: K=%lld must be a multiple of 8", fn, (long long)K);
    if (M > (int64_t)65535 * 128 || N > INT32_MAX / 2 || K > INT32_MAX / 2)
        return fail(GDN_ERR_OVERFLOW, "%s: M, N or K too large", fn);
    int64_t xy = 0, xk = 0, wk = 0;
    if (!mul_ok(M, N, &xy) || !mul_ok(M, K, &xk) || !mul_ok(N, K, &wk))
        return fail(GDN_ERR_OVERFLOW, "%s: size overflow", fn);
    if (M == 0 || N == 0) { g_last_error[0] = '\0'; return GDN_OK; }
    if (!y || (K > 0 && (!x || !w)))
        return fail(GDN_ERR_NULL, "%s: a tensor pointer is NULL", fn);
    if (!aligned(y, 16) || (K > 0 && (!aligned(x, 16) || !aligned(w, 16))) ||
        (status && !aligned(status, 4)))
        return fail(GDN_ERR_ALIGN, "%s: x, w, y need 16-byte alignment", fn);
    const Span ins[] = {{x, xk * 2, "x"}, {w, wk * 2, "w"}, {status, status ? 4 : 0, "status"}};
    gdn_status st = check_spans(ins, 3, 0, Span{y, xy * 4, "y"});
    if (st != GDN_OK) return st;
    if (K == 0)    // an empty sum: y = 0
        return launched(cudaMemsetAsync(y, 0, static_cast<size_t>(xy) * 4,
                                        static_cast<cudaStream_t>(stream)), fn);
    LinearArgs a{x, w, y, M, N, K, status};
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    return launched(split ? launch_linear_bf16_split(a, cs) : launch_linear_bf16(a, cs), fn);
}

}  // namespace

gdn_status gdn_layer_decode(const float* mixed_qkv, const float* z, const float* a,
                            const float* b, float* conv_ring, const float* conv_w,
                            const float* A_log, const float* dt_bias, const float* norm_w,
                            float l2_eps, float norm_eps, float* state, float* out, int64_t B,
                            int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, int64_t K,
                            void* stream) {
    NvtxRange nvtx_range("gdn_layer_decode");
    bool empty = false;
    gdn_status st = check_layer("gdn_layer_decode", 1, mixed_qkv, z, a, b, conv_ring, conv_w,
                                A_log, dt_bias, norm_w, state, nullptr, nullptr, out, B, Hk,
                                Hv, dk, dv, K, &empty);
    if (st != GDN_OK || empty) {
        if (st == GDN_OK) g_last_error[0] = '\0';
        return st;
    }
    LayerArgs args{mixed_qkv, z, a, b, conv_ring, conv_w, A_log, dt_bias, norm_w, l2_eps,
                   norm_eps, state, out, B, static_cast<int>(Hk), static_cast<int>(Hv),
                   nullptr, nullptr};
    return launched(launch_layer_decode(args, static_cast<cudaStream_t>(stream)),
                    "gdn_layer_decode");
}

gdn_status gdn_layer_pair(const float* mixed_qkv, const float* z, const float* a, const float* b,
                          float* conv_ring, const float* conv_w, const float* A_log,
                          const float* dt_bias, const float* norm_w, float l2_eps,
                          float norm_eps, float* state, float* scratch_ring,
                          float* scratch_state, float* out, int64_t B, int64_t Hk, int64_t Hv,
                          int64_t dk, int64_t dv, int64_t K, void* stream) {
    NvtxRange nvtx_range("gdn_layer_pair");
    bool empty = false;
    gdn_status st = check_layer("gdn_layer_pair", 2, mixed_qkv, z, a, b, conv_ring, conv_w,
                                A_log, dt_bias, norm_w, state, scratch_ring, scratch_state, out,
                                B, Hk, Hv, dk, dv, K, &empty);
    if (st != GDN_OK || empty) {
        if (st == GDN_OK) g_last_error[0] = '\0';
        return st;
    }
    LayerArgs args{mixed_qkv, z, a, b, conv_ring, conv_w, A_log, dt_bias, norm_w, l2_eps,
                   norm_eps, state, out, B, static_cast<int>(Hk), static_cast<int>(Hv),
                   scratch_ring, scratch_state};
    return launched(launch_layer_pair(args, static_cast<cudaStream_t>(stream)),
                    "gdn_layer_pair");
}

gdn_status gdn_linear_bf16(const void* x, const void* w, float* y, int64_t M, int64_t N,
                           int64_t K, uint32_t* status, void* stream) {
    NvtxRange nvtx_range("gdn_linear_bf16");
    return linear_call("gdn_linear_bf16", x, w, y, M, N, K, status, stream, false);
}

gdn_status gdn_linear_bf16_split_k(const void* x, const void* w, float* y, int64_t M, int64_t N,
                                   int64_t K, uint32_t* status, void* stream) {
    NvtxRange nvtx_range("gdn_linear_bf16_split_k");
    return linear_call("gdn_linear_bf16_split_k", x, w, y, M, N, K, status, stream, true);
}

size_t gdn_forward_batch_workspace_size(int64_t B, int64_t T, int64_t Hk, int64_t Hv,
                                        int64_t dk, int64_t dv) {
    if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || Hv % Hk != 0 || dk != kDk || dv != kDv ||
        Hv > (1 << 20) || B > 65535 || T > (int64_t)65535 * 32 ||
        B * T > (int64_t)65535 * 128)
        return 0;
    return forward_batch_layout(B, T, static_cast<int>(Hk), static_cast<int>(Hv)).total;
}

gdn_status gdn_forward_batch(const void* hidden, const void* w_qkv, const void* w_z,
                             const void* w_ba, const void* w_out, float* conv_ring,
                             const float* conv_w, const float* A_log, const float* dt_bias,
                             const float* norm_w, float l2_eps, float norm_eps, float* state,
                             float* out, void* workspace, size_t workspace_bytes, int64_t B,
                             int64_t T, int64_t D, int64_t Hk, int64_t Hv, int64_t dk,
                             int64_t dv, int64_t K, uint32_t* status, void* stream) {
    NvtxRange nvtx_range("gdn_forward_batch");
    const char* fn = "gdn_forward_batch";
    if (B < 0 || T < 0 || D < 0) return fail(GDN_ERR_SHAPE, "%s: negative B, T or D", fn);
    gdn_status st = check_geometry(Hk, Hv, dk, dv);
    if (st != GDN_OK) return st;
    if (K != kConvK) return fail(GDN_ERR_UNSUPPORTED, "%s: K=%lld: only a conv kernel of 4 is implemented",
                                 fn, (long long)K);
    if (D == 0 || D % 8 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "%s: D=%lld must be a positive multiple of 8", fn, (long long)D);
    // B*T rows of the projection GEMMs (M tiles of 128); the conv walks tiles
    // of 32 positions in one grid dimension, and the sequences in another.
    if (B > 65535 || T > (int64_t)65535 * 32 || B * T > (int64_t)65535 * 128 || D > (1 << 24))
        return fail(GDN_ERR_OVERFLOW, "%s: B=%lld, T=%lld, B*T or D too large", fn, (long long)B,
                    (long long)T);
    const int64_t BT = B * T;
    const int64_t C = 2 * Hk * dk + Hv * dv;
    const int64_t HD = Hv * dv;
    if (BT == 0) { g_last_error[0] = '\0'; return GDN_OK; }
    const size_t need = forward_batch_layout(B, T, static_cast<int>(Hk), static_cast<int>(Hv)).total;
    if (!hidden || !w_qkv || !w_z || !w_ba || !w_out || !conv_ring || !conv_w || !A_log ||
        !dt_bias || !norm_w || !state || !out || !workspace)
        return fail(GDN_ERR_NULL, "%s: a tensor pointer is NULL", fn);
    if (workspace_bytes < need)
        return fail(GDN_ERR_SHAPE, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes, need);
    if (!aligned(hidden, 16) || !aligned(w_qkv, 16) || !aligned(w_z, 16) || !aligned(w_ba, 16) ||
        !aligned(w_out, 16) || !aligned(conv_ring, 16) || !aligned(conv_w, 16) ||
        !aligned(state, 16) || !aligned(out, 16) || !aligned(workspace, 256) ||
        !aligned(A_log, 4) || !aligned(dt_bias, 4) || !aligned(norm_w, 4) ||
        (status && !aligned(status, 4)))
        return fail(GDN_ERR_ALIGN, "%s: alignment rule violated (workspace needs 256 bytes)", fn);
    const Span ins[] = {{state, B * Hv * dv * dk * 4, "state"},
                        {conv_ring, B * (K - 1) * C * 4, "conv_ring"},
                        {workspace, static_cast<int64_t>(need), "workspace"},
                        {status, status ? 4 : 0, "status"},
                        {hidden, BT * D * 2, "hidden"}, {w_qkv, C * D * 2, "w_qkv"},
                        {w_z, HD * D * 2, "w_z"}, {w_ba, 2 * Hv * D * 2, "w_ba"},
                        {w_out, D * HD * 2, "w_out"}, {conv_w, C * K * 4, "conv_w"},
                        {A_log, Hv * 4, "A_log"}, {dt_bias, Hv * 4, "dt_bias"},
                        {norm_w, dv * 4, "norm_w"}};
    st = check_spans(ins, 13, 4, Span{out, BT * D * 4, "out"});
    if (st != GDN_OK) return st;
    ForwardBatchArgs a{hidden, w_qkv, w_z, w_ba, w_out, conv_ring, conv_w, A_log, dt_bias, norm_w,
                       l2_eps, norm_eps, state, out, workspace, B, T, D, static_cast<int>(Hk),
                       static_cast<int>(Hv), status};
    return launched(launch_forward_batch(a, static_cast<cudaStream_t>(stream)), fn);
}

size_t gdn_short_conv_workspace_size(int64_t B, int64_t T, int64_t D) {
    if (B < 0 || T < 0 || D <= 0 || D % 8 != 0 || D > (1 << 24) || B > 65535 ||
        T > (int64_t)65535 * 32 || B * T > (int64_t)65535 * 128)
        return 0;
    return short_conv_layout(B, T, D).total;
}

}  // extern "C"

namespace {

// Shared checks of the three short-conv entries; n_commit positions go to
// conv_ring, the ring after the last position to scratch_ring (if given).
gdn_status short_conv_call(const char* fn, const void* hidden, const void* w_in,
                           const void* w_out, float* conv_ring, float* scratch_ring,
                           const float* conv_w, float* out, void* workspace,
                           size_t workspace_bytes, int64_t B, int64_t T, int64_t D, int64_t K,
                           int64_t n_commit, uint32_t* status, void* stream) {
    NvtxRange nvtx_range(fn);
    if (B < 0 || T < 0 || D < 0) return fail(GDN_ERR_SHAPE, "%s: negative B, T or D", fn);
    if (K < 2 || K > 4)
        return fail(GDN_ERR_UNSUPPORTED, "%s: K=%lld: conv kernels of 2, 3 or 4 are implemented",
                    fn, (long long)K);
    if (D == 0 || D % 8 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "%s: D=%lld must be a positive multiple of 8", fn,
                    (long long)D);
    // the gate/conv kernel walks tiles of 32 positions in one grid dimension
    if (B > 65535 || T > (int64_t)65535 * 32 || B * T > (int64_t)65535 * 128 || D > (1 << 24))
        return fail(GDN_ERR_OVERFLOW, "%s: B=%lld, T=%lld, B*T or D too large", fn, (long long)B,
                    (long long)T);
    const int64_t BT = B * T;
    if (BT == 0) { g_last_error[0] = '\0'; return GDN_OK; }
    const size_t need = short_conv_layout(B, T, D).total;
    if (!hidden || !w_in || !w_out || !conv_ring || !conv_w || !out || !workspace)
        return fail(GDN_ERR_NULL, "%s: a tensor pointer is NULL", fn);
    if (workspace_bytes < need)
        return fail(GDN_ERR_SHAPE, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes,
                    need);
    if (!aligned(hidden, 16) || !aligned(w_in, 16) || !aligned(w_out, 16) ||
        !aligned(conv_ring, 16) || !aligned(conv_w, 16) || !aligned(out, 16) ||
        (scratch_ring && !aligned(scratch_ring, 16)) || !aligned(workspace, 256) ||
        (status && !aligned(status, 4)))
        return fail(GDN_ERR_ALIGN, "%s: alignment rule violated (workspace needs 256 bytes)", fn);
    const int64_t ring_bytes = B * (K - 1) * D * 4;
    const Span ins[] = {{conv_ring, ring_bytes, "conv_ring"},
                        {scratch_ring, scratch_ring ? ring_bytes : 0, "scratch_ring"},
                        {workspace, static_cast<int64_t>(need), "workspace"},
                        {status, status ? 4 : 0, "status"},
                        {hidden, BT * D * 2, "hidden"}, {w_in, 3 * D * D * 2, "w_in"},
                        {w_out, D * D * 2, "w_out"}, {conv_w, D * K * 4, "conv_w"}};
    gdn_status st = check_spans(ins, 8, 4, Span{out, BT * D * 4, "out"});
    if (st != GDN_OK) return st;
    ShortConvArgs a{hidden, w_in, w_out, conv_ring, scratch_ring, conv_w, out, workspace,
                    B, T, D, static_cast<int>(K), n_commit, status};
    return launched(launch_short_conv(a, static_cast<cudaStream_t>(stream)), fn);
}

}  // namespace

extern "C" {

gdn_status gdn_short_conv_forward_batch(const void* hidden, const void* w_in, const void* w_out,
                                        float* conv_ring, const float* conv_w, float* out,
                                        void* workspace, size_t workspace_bytes, int64_t B,
                                        int64_t T, int64_t D, int64_t K, uint32_t* status,
                                        void* stream) {
    return short_conv_call("gdn_short_conv_forward_batch", hidden, w_in, w_out, conv_ring,
                           nullptr, conv_w, out, workspace, workspace_bytes, B, T, D, K, T,
                           status, stream);
}

gdn_status gdn_short_conv_forward(const void* hidden, const void* w_in, const void* w_out,
                                  float* conv_ring, const float* conv_w, float* out,
                                  void* workspace, size_t workspace_bytes, int64_t B, int64_t D,
                                  int64_t K, uint32_t* status, void* stream) {
    return short_conv_call("gdn_short_conv_forward", hidden, w_in, w_out, conv_ring, nullptr,
                           conv_w, out, workspace, workspace_bytes, B, 1, D, K, 1, status,
                           stream);
}

gdn_status gdn_short_conv_pair(const void* hidden, const void* w_in, const void* w_out,
                               float* conv_ring, float* scratch_ring, const float* conv_w,
                               float* out, void* workspace, size_t workspace_bytes, int64_t B,
                               int64_t D, int64_t K, uint32_t* status, void* stream) {
    if (B > 0 && !scratch_ring)
        return fail(GDN_ERR_NULL, "gdn_short_conv_pair: scratch_ring is NULL");
    return short_conv_call("gdn_short_conv_pair", hidden, w_in, w_out, conv_ring, scratch_ring,
                           conv_w, out, workspace, workspace_bytes, B, 2, D, K, 1, status,
                           stream);
}

}  // extern "C"
