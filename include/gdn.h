/*
 * gdn.h -- C ABI of libgdn.so: the Gated DeltaNet recurrent-state update on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (page "Red Lite dev15c -- Gated DeltaNet recurrent-state
 * parity", section "Pinned llama.cpp semantics"): for every value head h,
 * with q and k taken from key head h % Hk and the fp32 state held transposed
 * as M[j][i] = S[i][j] (row j = value index, i = key index), one token does
 *   1. M *= exp(gate[h])
 *   2. sk[j] = dot(M[j], k)
 *   3. delta[j] = (v[j] - sk[j]) * beta[h]
 *   4. M[j][i] += delta[j] * k[i]
 *   5. out[j] = dot(M[j], q) / sqrt(dk)      (the updated state)
 *
 * Conventions shared by every entry point
 *   - All tensors are dense, C-contiguous, row-major arrays in DEVICE memory
 *     of the current CUDA device (no host pointers): float32, except the
 *     projections' operands (hidden, x and the weight matrices), which are
 *     bf16 bit patterns where an entry point says so.
 *   - The caller allocates and frees every buffer. The library allocates no
 *     memory, never synchronises, and enqueues its kernels on `stream`
 *     (a cudaStream_t; NULL means the legacy default stream). Results are
 *     ready once the stream reaches that point.
 *   - Supported geometry: dk = dv = 128, Hk >= 1, Hv a multiple of Hk, conv
 *     kernel K = 4 for the recurrent layer's calls and K in {2, 3, 4} for the
 *     short-conv mixer. Other values return GDN_ERR_UNSUPPORTED.
 *   - `state` and `conv_ring` are updated in place and must not overlap any
 *     other argument; `out` and the scratch outputs must not overlap any
 *     argument either (GDN_ERR_ALIAS otherwise). Read-only inputs may share
 *     memory.
 *   - Alignment: state, scratch_state, q, k, v, g, out, mixed_qkv, z,
 *     conv_ring, conv_w, hidden, x and the weight matrices must be 16-byte
 *     aligned, workspaces 256-byte aligned; the per-head scalars (beta,
 *     gate, a, b, A_log, dt_bias), norm_w and the optional status words need
 *     4-byte alignment.
 *   - Status words (gdn_prefill, gdn_linear_bf16*, gdn_forward_batch*,
 *     gdn_short_conv_*): an optional zero-initialised device uint32 into
 *     which a kernel ORs a bit if one of its bounded waits (2 s) ever gives
 *     up; the kernel then returns without hanging. NULL: not reported.
 *   - Arguments are checked on the host before anything is enqueued; on any
 *     error nothing is written and nothing is launched. A problem with no
 *     work (a zero size) returns GDN_OK without touching any pointer.
 *   - Sizes are int64_t. Kernel faults are asynchronous and surface at the
 *     caller's next synchronisation, as for any CUDA kernel.
 *   - Thread safety: calls from several host threads are safe; calls that
 *     update the same state buffer, or share a workspace, must be ordered by
 *     the caller (gdn_forward_batch_noalloc's built-in scratch is shared by
 *     all its calls).
 *   - Every entry point opens an NVTX range named after itself.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_NULL = 1,        /* a required pointer is NULL                     */
    GDN_ERR_SHAPE = 2,       /* a negative size, or Hv not a multiple of Hk    */
    GDN_ERR_UNSUPPORTED = 3, /* dk, dv or K outside what the kernels implement */
    GDN_ERR_ALIGN = 4,       /* a pointer violates the alignment rule above    */
    GDN_ERR_OVERFLOW = 5,    /* an element count does not fit the index type   */
    GDN_ERR_CUDA = 6,        /* the CUDA runtime refused the launch            */
    GDN_ERR_ALIAS = 7        /* an output or in-place buffer overlaps another  */
} gdn_status;

/* Static English text for a status code (never NULL). */
const char *gdn_status_string(int status);

/* Text describing the last failed call on this host thread ("" if none):
 * any status, cleared by a call that succeeds. The pointer stays valid until
 * the next call of this library on the same thread. */
const char *gdn_last_error(void);

/* Text of the last call on this host thread that returned GDN_ERR_CUDA ("" if
 * none has): the CUDA runtime's name and description of the refused launch.
 * Unlike gdn_last_error() it only changes when another call returns
 * GDN_ERR_CUDA; argument errors and later successful calls leave it as it is.
 * Thread-local; the pointer stays valid for the life of the thread. */
const char *gdn_last_cuda_error(void);

/*
 * gdn_step -- one decode token for L layers x B sequences x Hv value heads,
 * in a single launch. Each (layer, sequence, value head) is an independent
 * recurrence; value head h reads q/k of key head h % Hk.
 * ("Red Lite dev15c -- Gated DeltaNet recurrent-state parity", section
 * "Pinned llama.cpp semantics", steps 1-5.)
 *
 *   state [L][B][Hv][dv][dk]  in/out, transposed layout M[j][i]
 *   q, k  [L][B][Hk][dk]      query and key (the kernel does not normalise)
 *   v     [L][B][Hv][dv]
 *   beta  [L][B][Hv]          write strength (used as given)
 *   gate  [L][B][Hv]          log-decay: the state is scaled by exp(gate)
 *   out   [L][B][Hv][dv]      out[j] = dot(M_new[j], q) / sqrt(dk)
 */
gdn_status gdn_step(float *state, const float *q, const float *k, const float *v,
                    const float *beta, const float *gate, float *out,
                    int64_t L, int64_t B, int64_t Hk, int64_t Hv, int64_t dk,
                    int64_t dv, void *stream);

/*
 * gdn_prefill -- T positions per sequence, run in order: position t starts
 * from the state left by position t-1, so the result equals T calls of
 * gdn_step with L = 1. ("Module linear_core", entry "gdn_forward_batch":
 * the recurrence runs sequentially over positions and is elementwise
 * identical to the one-position path; steps as for gdn_step.)
 *
 *   state [B][Hv][dv][dk]  in: initial state, out: state after position T-1
 *   q, k  [B][T][Hk][dk]
 *   v     [B][T][Hv][dv]
 *   beta, gate [B][T][Hv]
 *   out   [B][T][Hv][dv]
 *   status optional zero-initialised device word: the kernel's stage
 *          pipeline waits are bounded (2 s); if one ever times out, a
 *          non-zero bit is ORed into it and the kernel returns without
 *          hanging (its outputs are then incomplete). NULL: not reported.
 */
gdn_status gdn_prefill(float *state, const float *q, const float *k, const float *v,
                       const float *beta, const float *gate, float *out,
                       int64_t B, int64_t T, int64_t Hk, int64_t Hv, int64_t dk,
                       int64_t dv, uint32_t *status, void *stream);

/*
 * gdn_pair -- two-position speculative verify of the recurrence, one launch
 * for L layers x B sequences x Hv value heads. Position 0 commits into
 * `state`; position 1 continues from that state into `scratch_state`, which
 * the caller takes as the new state when it accepts the draft token (by
 * swapping the two buffers) and ignores otherwise. Each state row is read
 * once and written twice. The results equal two gdn_step calls, bit for bit.
 * ("Module linear_core", entry "gdn_pair": lane 1 commits, lane 2 is
 * tentative in scratch; steps as for gdn_step.)
 *
 *   state          [L][B][Hv][dv][dk]  in: before position 0,
 *                                      out: after position 0
 *   scratch_state  [L][B][Hv][dv][dk]  out: after position 1 (never read)
 *   q, k           [L][B][2][Hk][dk]   position p of sequence (l, b) at [l][b][p]
 *   v              [L][B][2][Hv][dv]
 *   beta, gate     [L][B][2][Hv]
 *   out            [L][B][2][Hv][dv]
 *
 * scratch_state and out must not overlap each other or any input; state may
 * not overlap an input.
 */
gdn_status gdn_pair(float *state, float *scratch_state, const float *q, const float *k,
                    const float *v, const float *beta, const float *gate, float *out,
                    int64_t L, int64_t B, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                    void *stream);

/*
 * gdn_layer_decode -- the single-token recurrent layer between the input
 * projections and the output projection, fused in one launch
 * ("Red Lite dev15e -- complete recurrent DeltaNet layer composition",
 * opening list; stage order from "Red Lite dev15a -- DeltaNet projection
 * field validation", section "Validation boundary"):
 *   1. causal depthwise conv over the window (conv_ring[0..K-2], mixed_qkv),
 *      oldest first, tap t of conv_w multiplying window[t], no bias; the
 *      ring then holds (conv_ring[1..K-2], mixed_qkv): raw inputs, shifted;
 *   2. SiLU; split into q [Hk][dk] | k [Hk][dk] | v [Hv][dv] (contiguous,
 *      head-major);
 *   3. q and k of each key head scaled by 1 / max(||x||_2, l2_eps);
 *   4. beta = sigmoid(b), gate = -exp(A_log) * softplus(a + dt_bias);
 *   5. the recurrence of gdn_step for every value head;
 *   6. gated RMSNorm per value head:
 *      out[j] = o[j] / sqrt(mean(o^2) + norm_eps) * norm_w[j] * SiLU(z[j]).
 *
 *   mixed_qkv [B][C], C = 2*Hk*dk + Hv*dv   pre-conv input of this token
 *   z         [B][Hv*dv]                    output gate input
 *   a, b      [B][Hv]                       raw decay / write-strength inputs
 *   conv_ring [B][K-1][C]                   in/out; slot 0 is the oldest
 *   conv_w    [C][K]
 *   A_log, dt_bias [Hv]
 *   norm_w    [dv]                          shared by all value heads
 *   state     [B][Hv][dv][dk]               in/out
 *   out       [B][Hv*dv]
 */
gdn_status gdn_layer_decode(const float *mixed_qkv, const float *z, const float *a,
                            const float *b, float *conv_ring, const float *conv_w,
                            const float *A_log, const float *dt_bias,
                            const float *norm_w, float l2_eps, float norm_eps,
                            float *state, float *out, int64_t B, int64_t Hk,
                            int64_t Hv, int64_t dk, int64_t dv, int64_t K,
                            void *stream);

/*
 * gdn_layer_pair -- the fused layer for two consecutive positions of each
 * sequence, for speculative verification ("Module linear_core", entry
 * "gdn_pair": lane 1 commits into the state, lane 2 is tentative in scratch,
 * the conv ring and the recurrent state moving together). Position 0 runs
 * gdn_layer_decode's six stages and commits: conv_ring and state are updated
 * in place. Position 1 continues from that committed result; the ring and
 * state it leaves are written to scratch_ring and scratch_state, and the
 * live buffers keep position 0's result. To accept the draft the caller
 * makes the scratch buffers live (swap pointers or copy); to reject it, it
 * ignores them. The result equals gdn_layer_decode on position 0 followed
 * by gdn_layer_decode on position 1 applied to copies of the updated
 * buffers; each state row is read once and written twice.
 *
 *   mixed_qkv     [B][2][C]
 *   z             [B][2][Hv*dv]
 *   a, b          [B][2][Hv]
 *   conv_ring     [B][K-1][C]        in/out: after position 0
 *   conv_w        [C][K];  A_log, dt_bias [Hv];  norm_w [dv]
 *   state         [B][Hv][dv][dk]    in/out: after position 0
 *   scratch_ring  [B][K-1][C]        out: after position 1
 *   scratch_state [B][Hv][dv][dk]    out: after position 1
 *   out           [B][2][Hv*dv]      both positions' outputs
 * scratch_ring and scratch_state are caller-allocated outputs, 16-byte
 * aligned, and must not overlap any other argument.
 */
gdn_status gdn_layer_pair(const float *mixed_qkv, const float *z, const float *a,
                          const float *b, float *conv_ring, const float *conv_w,
                          const float *A_log, const float *dt_bias,
                          const float *norm_w, float l2_eps, float norm_eps,
                          float *state, float *scratch_ring, float *scratch_state,
                          float *out, int64_t B, int64_t Hk, int64_t Hv, int64_t dk,
                          int64_t dv, int64_t K, void *stream);

/*
 * gdn_linear_bf16 -- dense projection on the tensor cores:
 *   y[M][N] = x[M][K] . w[N][K]^T
 * with bf16 inputs and fp32 accumulation and output. These are the layer's
 * projections ("Red Lite dev15e -- complete recurrent DeltaNet layer
 * composition", opening list: attn_qkv 2048 -> 8192, attn_gate 2048 ->
 * 4096, ssm_ba 2048 -> 64, ssm_out 4096 -> 2048), here with dense bf16
 * weights, run as matrix-matrix products over a batch of positions
 * ("Module linear_core", entry "gdn_forward_batch").
 *
 *   x       [M][K] bf16 (uint16 bit patterns), row-major, 16-byte aligned
 *   w       [N][K] bf16, row-major (the usual [out][in] weight layout)
 *   y       [M][N] fp32 output, 16-byte aligned, must not overlap x or w
 *   K       a multiple of 8 (16-byte rows for the tensor-memory copies);
 *           K = 0 gives y = 0
 *   status  optional device pointer to a zero-initialised 32-bit word; if a
 *           kernel-internal wait ever times out (2 s) a non-zero bit is ORed
 *           into it and the kernel returns without hanging. NULL: not reported.
 */
gdn_status gdn_linear_bf16(const void *x, const void *w, float *y, int64_t M, int64_t N,
                           int64_t K, uint32_t *status, void *stream);

/*
 * gdn_linear_bf16_split_k -- the same product for decode-sized calls. With
 * M <= 128 rows, K is split into S chunks (S <= 8, fixed by N, K and the
 * device, never by M); the S CTAs of a thread-block cluster each accumulate
 * one chunk on the tensor cores and the chunk sums are added in fp32 in chunk
 * order through distributed shared memory. Every row is then the same in any
 * call of at most 128 rows; it differs from gdn_linear_bf16's row by the
 * rounding of that grouped sum (same error bound). M > 128, or a product too
 * small to split, runs gdn_linear_bf16. Arguments, alignment, aliasing,
 * status and errors as gdn_linear_bf16.
 */
gdn_status gdn_linear_bf16_split_k(const void *x, const void *w, float *y, int64_t M, int64_t N,
                                   int64_t K, uint32_t *status, void *stream);

/*
 * gdn_forward_batch -- the recurrent layer over T consecutive positions of
 * each of B sequences, with dense bf16 projections ("Module linear_core",
 * entry "gdn_forward_batch": the qkv/z/a/b and out_proj projections are
 * matrix-matrix products over the batch while the recurrence runs
 * sequentially over positions; stages as in gdn_layer_decode). Per position,
 * in order:
 *   mixed = W_qkv h,  z = W_z h,  (b | a) = W_ba h        (tensor-core GEMMs)
 *   stages 1-6 of gdn_layer_decode (conv with ring, SiLU, split, L2 norms,
 *   beta/gate, recurrence, gated RMSNorm), the recurrence carried across
 *   positions as in gdn_prefill;
 *   y rounded to bf16, out = W_out y                        (tensor-core GEMM)
 *
 *   hidden    [B][T][D] bf16        D a multiple of 8
 *   w_qkv     [C][D] bf16, C = 2*Hk*dk + Hv*dv
 *   w_z       [Hv*dv][D] bf16
 *   w_ba      [2*Hv][D] bf16        rows 0..Hv-1 give b, rows Hv..2Hv-1 give a
 *   w_out     [D][Hv*dv] bf16
 *   conv_ring [B][K-1][C] in/out    after position T-1
 *   conv_w [C][K]; A_log, dt_bias [Hv]; norm_w [dv]   (fp32)
 *   state     [B][Hv][dv][dk] in/out
 *   out       [B][T][D] fp32
 *   workspace device scratch of at least gdn_forward_batch_workspace_size()
 *             bytes, 256-byte aligned, owned by the caller; its contents on
 *             entry do not matter and are undefined afterwards
 *   status    optional zero-initialised device word for timeout bits (see
 *             gdn_linear_bf16)
 * Limits: B <= 65535, T <= 65535 * 32, B*T <= 65535 * 128 (GDN_ERR_OVERFLOW
 * otherwise; the workspace size function returns 0).
 */
size_t gdn_forward_batch_workspace_size(int64_t B, int64_t T, int64_t Hk, int64_t Hv,
                                        int64_t dk, int64_t dv);
gdn_status gdn_forward_batch(const void *hidden, const void *w_qkv, const void *w_z,
                             const void *w_ba, const void *w_out, float *conv_ring,
                             const float *conv_w, const float *A_log, const float *dt_bias,
                             const float *norm_w, float l2_eps, float norm_eps, float *state,
                             float *out, void *workspace, size_t workspace_bytes, int64_t B,
                             int64_t T, int64_t D, int64_t Hk, int64_t Hv, int64_t dk,
                             int64_t dv, int64_t K, uint32_t *status, void *stream);

/*
 * gdn_forward_batch_noalloc -- gdn_forward_batch without a caller-provided
 * workspace, for callers that cannot allocate device memory (a plugin whose
 * host program owns every device allocation and offers no hook, code held to
 * a memory budget fixed before it runs, or a latency-critical path where an
 * allocation is not allowed). There is no counterpart on the source pages:
 * it is a deployment variant of the same layer. Arguments and results are
 * those of gdn_forward_batch without `workspace` and `workspace_bytes`.
 *
 * The workspace is a 16 MiB array built into the library (held on every GPU
 * that loads the library until the process exits). A call is accepted when
 * gdn_forward_batch_workspace_size(B, T, ...) fits in 16 MiB: at Hk = 16,
 * Hv = 32, dk = dv = 128 that is about 72.5 KiB per position plus 96 KiB per
 * started 32-position tile of each sequence, so B = 1 with T <= 216, B = 67
 * with T = 2, B = 97 with T = 1. Larger calls are rejected with
 * GDN_ERR_UNSUPPORTED and a message; nothing is launched.
 *
 * The array's device address is looked up with cudaGetSymbolAddress in the
 * current context and cached per device under the driver's ID of that
 * context; the first call in a context (the first on a device, and the
 * first after cudaDeviceReset or in another context the caller made
 * current) does that lookup, so make it before any stream capture. Every
 * call uses the same array, so calls whose GPU work overlaps (other streams,
 * other host threads on the same device) race and must be ordered by the
 * caller. The library performs no allocation of any kind for this call.
 */
gdn_status gdn_forward_batch_noalloc(const void *hidden, const void *w_qkv, const void *w_z,
                                     const void *w_ba, const void *w_out, float *conv_ring,
                                     const float *conv_w, const float *A_log,
                                     const float *dt_bias, const float *norm_w, float l2_eps,
                                     float norm_eps, float *state, float *out, int64_t B,
                                     int64_t T, int64_t D, int64_t Hk, int64_t Hv, int64_t dk,
                                     int64_t dv, int64_t K, uint32_t *status, void *stream);

/*
 * gdn_kda_step / gdn_kda_prefill -- the KDA core ("Module linear_core",
 * entries "kda_forward": one position, advances the state, and
 * "kda_forward_batch": the recurrence sequential per position, elementwise
 * identical to the one-position path). The pages give no equations; the
 * update implemented is the published Kimi Delta Attention rule, the
 * delta rule with a decay per key channel. In the layout of gdn_step
 * (M[j][i] = S[i][j]), per value head h reading key head h % Hk:
 *   1. M[j][i] *= exp(g[h][i])  2. sk[j] = M[j].k  3. delta[j] = (v[j] - sk[j]) beta
 *   4. M[j] += delta[j] k       5. out[j] = M_new[j].q / sqrt(dk)
 * Arguments, layouts, ownership and errors are those of gdn_step and
 * gdn_prefill, except the log-decay:
 *   gdn_kda_step:    g [L][B][Hv][dk]
 *   gdn_kda_prefill: g [B][T][Hv][dk]   (contiguous)
 * g must be 16-byte aligned. Values at or below 0 are expected (decays in
 * (0, 1]); others are applied as given.
 */
gdn_status gdn_kda_step(float *state, const float *q, const float *k, const float *v,
                        const float *beta, const float *g, float *out, int64_t L, int64_t B,
                        int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, void *stream);
gdn_status gdn_kda_prefill(float *state, const float *q, const float *k, const float *v,
                           const float *beta, const float *g, float *out, int64_t B, int64_t T,
                           int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, void *stream);

/*
 * The LFM2 short-convolution mixer ("Module linear_core", struct
 * "ShortConvWeights": no recurrent state, the only state is the causal conv
 * ring holding the last kernel-1 gated inputs of every channel; entries
 * "short_conv_forward", "short_conv_forward_batch" and "short_conv_pair").
 * The pages give no formula; the mixer implemented is, per position t and
 * channel d:
 *   (bg | cg | xv) = W_in h_t        rows [0,D) | [D,2D) | [2D,3D) of W_in
 *   u = bg[d] * xv[d]                the gated input, rounded to fp32
 *   conv = sum_{tau<K} conv_w[d][tau] * window[tau],
 *          window = (ring[0..K-2], u) oldest first, no bias
 *   y = cg[d] * conv                 rounded to bf16
 *   out_t = W_out y                  (tensor-core GEMMs, fp32 accumulation)
 * and the ring drops its oldest slot and appends u.
 *
 *   hidden    [B][T][D] bf16        D a positive multiple of 8
 *   w_in      [3D][D] bf16
 *   w_out     [D][D] bf16
 *   conv_ring [B][K-1][D] fp32 in/out, slot 0 oldest
 *   conv_w    [D][K] fp32, tap 0 multiplies the oldest slot; K in {2, 3, 4}
 *   out       [B][T][D] fp32
 *   workspace device scratch of gdn_short_conv_workspace_size(B, T, D) bytes,
 *             256-byte aligned, owned by the caller; contents on entry do
 *             not matter and are undefined afterwards (its last 256 bytes
 *             hold the one-kernel form's barrier word, below)
 *   status    optional zero-initialised device word for timeout bits (see
 *             gdn_linear_bf16)
 * All pointers are device pointers, 16-byte aligned. conv_ring is updated in
 * place and may overlap nothing else; out may overlap no argument.
 * Limits: B <= 65535, T <= 65535 * 32, B*T <= 65535 * 128 (GDN_ERR_OVERFLOW
 * otherwise). gdn_short_conv_workspace_size returns 0 for an invalid shape.
 *
 * Calls of at most 128 rows (B*T) run the input projection split over K in a
 * thread-block cluster, with the gate, conv and ring update as its epilogue,
 * and the output projection split the same way (see gdn_linear_bf16_split_k).
 * Outputs and rings are then identical, bit for bit, across all such calls
 * (any chunking into calls, single positions, the verify). Between a call of
 * at most 128 rows and a larger one they differ by the fp32 rounding of the
 * projections' accumulation order.
 *
 * One-kernel form: calls of one or two positions (decode, verify) with D a
 * multiple of 64 whose two projections take the same K split run the whole
 * mixer as one kernel, with the same bits. Between the conv and the output
 * projection its CTAs meet at a grid-wide barrier: a 64-bit word at offset
 * workspace_size - 256 that the call tags with a number of its own (any
 * earlier content is replaced; a CUDA graph replay finds and replaces its
 * own completed count). The barrier needs every CTA of the grid resident at
 * once (one per SM, at most 148): a kernel on another stream that holds SMs
 * for longer than the 2 s wait limit makes the call time out, ORing 16 into
 * `status` (the outputs are then undefined). Two calls that share a
 * workspace must be ordered, as for any workspace. The environment variable
 * GDN_SHORT_CONV_ONE_KERNEL=0, read at every call, selects the two-kernel
 * path instead (the same bits), e.g. where other work holds SMs for long.
 *
 * gdn_short_conv_forward_batch runs T positions in order; conv_ring ends as
 * the ring after position T-1 (T = 0 does nothing).
 * gdn_short_conv_forward is the same call for one position per sequence:
 * hidden [B][D], out [B][D].
 * gdn_short_conv_pair is the two-position verify: hidden [B][2][D],
 * out [B][2][D]; conv_ring receives the ring after position 0 (committed)
 * and scratch_ring [B][K-1][D] the ring after position 1 (tentative, to be
 * swapped in on acceptance). scratch_ring may overlap nothing else.
 */
size_t gdn_short_conv_workspace_size(int64_t B, int64_t T, int64_t D);
gdn_status gdn_short_conv_forward_batch(const void *hidden, const void *w_in, const void *w_out,
                                        float *conv_ring, const float *conv_w, float *out,
                                        void *workspace, size_t workspace_bytes, int64_t B,
                                        int64_t T, int64_t D, int64_t K, uint32_t *status,
                                        void *stream);
gdn_status gdn_short_conv_forward(const void *hidden, const void *w_in, const void *w_out,
                                  float *conv_ring, const float *conv_w, float *out,
                                  void *workspace, size_t workspace_bytes, int64_t B, int64_t D,
                                  int64_t K, uint32_t *status, void *stream);
gdn_status gdn_short_conv_pair(const void *hidden, const void *w_in, const void *w_out,
                               float *conv_ring, float *scratch_ring, const float *conv_w,
                               float *out, void *workspace, size_t workspace_bytes, int64_t B,
                               int64_t D, int64_t K, uint32_t *status, void *stream);

/*
 * gdn_selftest_bounded_wait -- a check of the library's failure detection,
 * with no counterpart on the source pages. Every tensor-core kernel of the
 * library (gdn_linear_bf16 and the calls built on it) waits on mbarriers with
 * a time limit; a wait that runs out sets a bit in the caller's status word
 * and the kernel returns, leaving the context usable. This call runs that
 * same bounded wait in a one-thread kernel on an mbarrier that expects one
 * arrival: with arrive = 0 nothing arrives and the wait must give up after
 * limit_ns nanoseconds (0 < limit_ns <= 2e9, the library's own limit); with
 * arrive = 1 the thread arrives first and the wait returns at once.
 *   result  device words [2]: result[0] = 0 (completed) or 1 (timed out,
 *           the producer-timeout bit of gdn_linear_bf16's status word);
 *           result[1] = microseconds waited. 4-byte aligned.
 * Errors: GDN_ERR_NULL, GDN_ERR_UNSUPPORTED (limit out of range),
 * GDN_ERR_ALIGN, GDN_ERR_CUDA (launch refused).
 */
gdn_status gdn_selftest_bounded_wait(uint32_t *result, uint64_t limit_ns, int arrive,
                                     void *stream);

/*
 * gdn_selftest_grid_barrier -- the same check for the grid-wide barrier of
 * the one-kernel short-conv mixer (see gdn_short_conv_forward), with no
 * counterpart on the source pages. `ctas` CTAs (1..32, one thread each)
 * install `tag` into `word` and wait, each with the limit limit_ns
 * (0 < limit_ns <= 2e9), until `expect` (1..64) have arrived.
 *   word    device uint64, 8-byte aligned: (tag << 16) | count; on entry
 *           anything (another tag, a completed count of this tag); on
 *           return (tag << 16) | ctas when every wait completed, and 0 after
 *           a wait ran out (expect > ctas makes every wait run out)
 *   result  device words [2 * ctas]: result[i] = 0 (CTA i passed) or 16
 *           (timed out: the bit the mixer ORs into its status word);
 *           result[ctas + i] = microseconds CTA i waited. 4-byte aligned.
 *   tag     0 < tag < 2^48; as in the mixer, a tag names one grid: a word
 *           left as (tag, c) with c < expect counts as that grid in progress
 * Errors: GDN_ERR_NULL, GDN_ERR_UNSUPPORTED (a size, the tag or the limit
 * out of range), GDN_ERR_ALIGN, GDN_ERR_CUDA (launch refused).
 */
gdn_status gdn_selftest_grid_barrier(unsigned long long *word, uint32_t *result, uint64_t tag,
                                     int ctas, int expect, uint64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
