/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle of the Gated DeltaNet
 * recurrent-state update and of the single-token recurrent layer around it.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this file's library. The CUDA library never links,
 * includes or calls it, and this file includes nothing from the CUDA side.
 *
 * Every value is held in double. Inputs arrive as double arrays (the callers
 * widen fp32 data exactly), outputs leave as double arrays. The loops follow
 * the pages' step order with no blocking, fusion or reordering; sums run in
 * ascending index order.
 *
 * Sources (page title, section):
 *   [S] "Red Lite dev15c -- Gated DeltaNet recurrent-state parity",
 *       section "Pinned llama.cpp semantics": value head h reads Q/K of key
 *       head h % 16; state layout M[j][i] = S[i][j]; one token runs the five
 *       numbered steps; the output uses the updated state.
 *   [L] "Red Lite dev15e -- complete recurrent DeltaNet layer composition",
 *       opening list and section "M4 field result": conv/prestate path with
 *       beta/decay transforms and Q/K L2 normalisation, the recurrence, then
 *       gated RMSNorm with ssm_norm.weight and SiLU(z); geometry
 *       channels=8192, qk=2048, value=4096, heads(k/v)=16/32, conv cache.
 *   [P] "Red Lite dev15a -- DeltaNet projection field validation", section
 *       "Validation boundary": stage order conv-state shift, ssm_conv1d,
 *       SiLU, Q/K/V split, per-head Q/K L2 normalisation.
 *   [B] "Module linear_core" (cortiq_engine), entry "gdn_forward_batch":
 *       the recurrence runs sequentially over positions and is elementwise
 *       identical to the one-position path; entry "gdn_pair": a fused
 *       two-position forward for speculative verification, where lane 1
 *       commits into the state and lane 2 is tentative in scratch, the conv
 *       ring and the recurrent state moving together; entry
 *       "gdn_forward_batch" also names the layer's projections (qkv, z, a/b,
 *       out_proj) as matrix products over a batch of positions.
 *   [K] "Module linear_core", struct "KdaWeights" and entries "kda_forward"
 *       and "kda_forward_batch": the KDA recurrence with the same
 *       one-position and sequential-batch contract (no equations given).
 *   [SC] "Module linear_core", struct "ShortConvWeights" and entries
 *       "short_conv_forward", "short_conv_forward_batch",
 *       "short_conv_pair": the LFM2 short-convolution mixer, whose only
 *       state is the causal conv ring of the last kernel-1 gated inputs per
 *       channel.
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes): gate is a log-decay applied as exp(gate); the output scale
 * 1/sqrt(128) is 1/sqrt(dk); the conv window is (ring[0..K-2], x) oldest
 * first with tap t multiplying window[t], no bias, and the ring keeps raw
 * (pre-conv) inputs; q | k | v are contiguous head-major slices of the conv
 * output; L2 normalisation is x / max(||x||, l2_eps); beta = sigmoid(b);
 * gate = -exp(A_log) * softplus(a + dt_bias); the tail is
 * o * (mean(o^2) + eps)^(-1/2) * w[j] * SiLU(z) with one weight vector of
 * length dv shared by all heads.
 *
 * Return codes: 0 on success, -1 on a bad argument (nothing is written),
 * -2 when a scratch allocation fails.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* The recurrence for one value head and one token. [S], steps 1-5.         */
/* M is [dv][dk] (row j = value index, i = key index, M[j][i] = S[i][j]).   */
/* ------------------------------------------------------------------------ */
static int gdn_head_token(double *M, const double *q, const double *k,
                          const double *v, double beta, double gate,
                          double *out, int64_t dk, int64_t dv)
{
    double *sk = (double *)malloc((size_t)dv * sizeof(double));
    double *delta = (double *)malloc((size_t)dv * sizeof(double));
    if (!sk || !delta) {
        free(sk);
        free(delta);
        return -2;
    }

    /* step 1: M *= exp(gate[h]) */
    const double decay = exp(gate);
    for (int64_t j = 0; j < dv; ++j)
        for (int64_t i = 0; i < dk; ++i)
            M[j * dk + i] *= decay;

    /* step 2: sk[j] = dot(M[j], k), on the decayed state */
    for (int64_t j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            acc += M[j * dk + i] * k[i];
        sk[j] = acc;
    }

    /* step 3: delta[j] = (v[j] - sk[j]) * beta[h] */
    for (int64_t j = 0; j < dv; ++j)
        delta[j] = (v[j] - sk[j]) * beta;

    /* step 4: M[j][i] += delta[j] * k[i] */
    for (int64_t j = 0; j < dv; ++j)
        for (int64_t i = 0; i < dk; ++i)
            M[j * dk + i] += delta[j] * k[i];

    /* step 5: out[j] = dot(M[j], q) / sqrt(dk), on the updated state */
    const double scale_div = sqrt((double)dk);
    for (int64_t j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            acc += M[j * dk + i] * q[i];
        out[j] = acc / scale_div;
    }

    free(sk);
    free(delta);
    return 0;
}

static int dims_ok(int64_t Hk, int64_t Hv, int64_t dk, int64_t dv)
{
    return Hk > 0 && Hv > 0 && dk > 0 && dv > 0 && Hv % Hk == 0;
}

/*
 * Batched single-token decode over L layers x B sequences x Hv value heads.
 *   state [L][B][Hv][dv][dk]  in/out
 *   q, k  [L][B][Hk][dk]
 *   v     [L][B][Hv][dv]
 *   beta, gate [L][B][Hv]
 *   out   [L][B][Hv][dv]      (only the listed units are written)
 * units: flat unit indices u = (l*B + b)*Hv + h to compute, or NULL for all.
 * [S]: each (layer, sequence, value head) is an independent recurrence; the
 * value head h takes q/k of key head h % Hk.
 */
int oracle_gdn_step(double *state, const double *q, const double *k,
                    const double *v, const double *beta, const double *gate,
                    double *out, int64_t L, int64_t B, int64_t Hk, int64_t Hv,
                    int64_t dk, int64_t dv, const int64_t *units,
                    int64_t n_units)
{
    if (L < 0 || B < 0 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t total = L * B * Hv;
    const int64_t count = units ? n_units : total;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        if (u < 0 || u >= total)
            return -1;
    }
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        const int64_t lb = u / Hv;           /* l*B + b */
        const int64_t h = u % Hv;
        const int64_t g = h % Hk;            /* key head read by value head h */
        const double *qg = q + (lb * Hk + g) * dk;
        const double *kg = k + (lb * Hk + g) * dk;
        int rc = gdn_head_token(state + u * dv * dk, qg, kg, v + u * dv,
                                beta[u], gate[u], out + u * dv, dk, dv);
        if (rc)
            return rc;
    }
    return 0;
}

/*
 * Sequential prefill over T positions, [B]: position t runs the one-token
 * recurrence on the state left by position t-1.
 *   state [B][Hv][dv][dk]  in: initial, out: final
 *   q, k  [B][T][Hk][dk]
 *   v     [B][T][Hv][dv]
 *   beta, gate [B][T][Hv]
 *   out   [B][T][Hv][dv]
 * units: flat indices u = b*Hv + h, or NULL for all.
 */
int oracle_gdn_prefill(double *state, const double *q, const double *k,
                       const double *v, const double *beta, const double *gate,
                       double *out, int64_t B, int64_t T, int64_t Hk,
                       int64_t Hv, int64_t dk, int64_t dv,
                       const int64_t *units, int64_t n_units)
{
    if (B < 0 || T < 0 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t total = B * Hv;
    const int64_t count = units ? n_units : total;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        if (u < 0 || u >= total)
            return -1;
    }
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        const int64_t b = u / Hv;
        const int64_t h = u % Hv;
        const int64_t g = h % Hk;
        double *M = state + u * dv * dk;
        for (int64_t t = 0; t < T; ++t) {
            const int64_t bt = b * T + t;
            int rc = gdn_head_token(M, q + (bt * Hk + g) * dk,
                                    k + (bt * Hk + g) * dk,
                                    v + (bt * Hv + h) * dv,
                                    beta[bt * Hv + h], gate[bt * Hv + h],
                                    out + (bt * Hv + h) * dv, dk, dv);
            if (rc)
                return rc;
        }
    }
    return 0;
}

/*
 * Two-position speculative verify of the bare recurrence, [B] entry
 * "gdn_pair": position 0 commits into the state, position 1 continues from
 * it into a scratch state that the caller swaps in when it accepts the draft.
 * Both are the one-token recurrence [S] run in order, as in the prefill.
 *   state   [L][B][Hv][dv][dk]  in: before position 0, out: after position 0
 *   scratch [L][B][Hv][dv][dk]  out: after position 1 (listed units only)
 *   q, k    [L][B][2][Hk][dk]
 *   v       [L][B][2][Hv][dv]
 *   beta, gate [L][B][2][Hv]
 *   out     [L][B][2][Hv][dv]
 * units: flat indices u = (l*B + b)*Hv + h, or NULL for all.
 */
int oracle_gdn_pair(double *state, double *scratch, const double *q,
                    const double *k, const double *v, const double *beta,
                    const double *gate, double *out, int64_t L, int64_t B,
                    int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                    const int64_t *units, int64_t n_units)
{
    if (L < 0 || B < 0 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t total = L * B * Hv;
    const int64_t count = units ? n_units : total;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        if (u < 0 || u >= total)
            return -1;
    }
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        const int64_t lb = u / Hv;           /* l*B + b */
        const int64_t h = u % Hv;
        const int64_t g = h % Hk;
        double *live = state + u * dv * dk;
        double *tent = scratch + u * dv * dk;
        for (int64_t pos = 0; pos < 2; ++pos) {
            const int64_t lbp = lb * 2 + pos;    /* (l, b, position) */
            double *M = pos == 0 ? live : tent;
            if (pos == 1)                        /* position 1 starts from the committed state */
                memcpy(tent, live, (size_t)(dv * dk) * sizeof(double));
            int rc = gdn_head_token(M, q + (lbp * Hk + g) * dk, k + (lbp * Hk + g) * dk,
                                    v + (lbp * Hv + h) * dv, beta[lbp * Hv + h],
                                    gate[lbp * Hv + h], out + (lbp * Hv + h) * dv, dk, dv);
            if (rc)
                return rc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Prestate pieces, [L] and [P].                                             */
/* ------------------------------------------------------------------------ */

/* SiLU(x) = x * sigmoid(x) */
static double silu(double x) { return x / (1.0 + exp(-x)); }

/* sigmoid(x) = 1 / (1 + e^-x) */
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* softplus(x) = ln(1 + e^x), written as max(x,0) + ln(1 + e^-|x|) */
static double softplus(double x)
{
    return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));
}

/*
 * Causal depthwise conv1d over one token with the conv-state ring, [P]
 * section "Validation boundary" (the conv-state shift, then the fp32
 * depthwise conv).
 *   x    [C]        this token's pre-conv input (mixed q|k|v)
 *   ring [K-1][C]   in/out; slot 0 is the oldest past input
 *   w    [C][K]     tap t multiplies window[t], window = (ring[0..K-2], x)
 *   y    [C]        conv output (before SiLU)
 * The ring afterwards holds (ring[1..K-2], x): the raw inputs, shifted.
 */
static void conv_ring_token(const double *x, double *ring, const double *w,
                            double *y, int64_t C, int64_t K)
{
    for (int64_t c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int64_t t = 0; t < K; ++t) {
            const double win = (t < K - 1) ? ring[t * C + c] : x[c];
            acc += w[c * K + t] * win;
        }
        y[c] = acc;
    }
    for (int64_t c = 0; c < C; ++c) {
        for (int64_t t = 0; t + 1 < K - 1; ++t)
            ring[t * C + c] = ring[(t + 1) * C + c];
        if (K > 1)
            ring[(K - 2) * C + c] = x[c];
    }
}

/* x /= max(||x||_2, eps), [L] "Q/K L2 normalization" */
static void l2_normalize(double *x, int64_t n, double eps)
{
    double ss = 0.0;
    for (int64_t i = 0; i < n; ++i)
        ss += x[i] * x[i];
    double norm = sqrt(ss);
    if (norm < eps)
        norm = eps;
    for (int64_t i = 0; i < n; ++i)
        x[i] = x[i] / norm;
}

/*
 * Prestate of one token of one sequence, [L] and [P]:
 *   conv (with ring shift) -> SiLU -> split q|k|v -> L2(q), L2(k) per key
 *   head -> beta = sigmoid(b_in), gate = -exp(A_log) * softplus(a + dt_bias).
 *   x [C = 2*Hk*dk + Hv*dv], ring [K-1][C] in/out, conv_w [C][K],
 *   a_in, b_in, A_log, dt_bias [Hv].
 * Outputs: q, k [Hk][dk], v [Hv][dv], beta, gate [Hv].
 */
static int prestate_token(const double *x, double *ring, const double *conv_w,
                          const double *a_in, const double *b_in,
                          const double *A_log, const double *dt_bias,
                          double l2_eps, double *q, double *k, double *v,
                          double *beta, double *gate, int64_t Hk, int64_t Hv,
                          int64_t dk, int64_t dv, int64_t K)
{
    const int64_t C = 2 * Hk * dk + Hv * dv;
    double *y = (double *)malloc((size_t)C * sizeof(double));
    if (!y)
        return -2;
    conv_ring_token(x, ring, conv_w, y, C, K);
    for (int64_t c = 0; c < C; ++c)
        y[c] = silu(y[c]);
    memcpy(q, y, (size_t)(Hk * dk) * sizeof(double));
    memcpy(k, y + Hk * dk, (size_t)(Hk * dk) * sizeof(double));
    memcpy(v, y + 2 * Hk * dk, (size_t)(Hv * dv) * sizeof(double));
    free(y);
    for (int64_t g = 0; g < Hk; ++g) {
        l2_normalize(q + g * dk, dk, l2_eps);
        l2_normalize(k + g * dk, dk, l2_eps);
    }
    for (int64_t h = 0; h < Hv; ++h) {
        beta[h] = sigmoid(b_in[h]);
        gate[h] = -exp(A_log[h]) * softplus(a_in[h] + dt_bias[h]);
    }
    return 0;
}

/*
 * Gated RMSNorm tail of one head, [L] ("gated RMSNorm with ssm_norm.weight
 * and SiLU(z)"): y[j] = o[j] * (mean(o^2) + eps)^(-1/2) * w[j] * SiLU(z[j]).
 */
static void gated_rmsnorm_head(const double *o, const double *z,
                               const double *w, double eps, double *y,
                               int64_t dv)
{
    double ss = 0.0;
    for (int64_t j = 0; j < dv; ++j)
        ss += o[j] * o[j];
    const double inv_rms = 1.0 / sqrt(ss / (double)dv + eps);
    for (int64_t j = 0; j < dv; ++j)
        y[j] = o[j] * inv_rms * w[j] * silu(z[j]);
}

/*
 * Stage entry: prestate for the listed sequences (NULL = all B).
 *   x [B][C], ring [B][K-1][C] in/out, conv_w [C][K], a_in, b_in [B][Hv],
 *   A_log, dt_bias [Hv]; outputs q, k [B][Hk][dk], v [B][Hv][dv],
 *   beta, gate [B][Hv].
 */
int oracle_gdn_prestate(const double *x, double *ring, const double *conv_w,
                        const double *a_in, const double *b_in,
                        const double *A_log, const double *dt_bias,
                        double l2_eps, double *q, double *k, double *v,
                        double *beta, double *gate, int64_t B, int64_t Hk,
                        int64_t Hv, int64_t dk, int64_t dv, int64_t K,
                        const int64_t *seqs, int64_t n_seqs)
{
    if (B < 0 || K < 1 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t C = 2 * Hk * dk + Hv * dv;
    const int64_t count = seqs ? n_seqs : B;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        if (b < 0 || b >= B)
            return -1;
    }
    for (int64_t n = 0; n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        int rc = prestate_token(x + b * C, ring + b * (K - 1) * C, conv_w,
                                a_in + b * Hv, b_in + b * Hv, A_log, dt_bias,
                                l2_eps, q + b * Hk * dk, k + b * Hk * dk,
                                v + b * Hv * dv, beta + b * Hv, gate + b * Hv,
                                Hk, Hv, dk, dv, K);
        if (rc)
            return rc;
    }
    return 0;
}

/*
 * Stage entry: gated RMSNorm tail over rows of dv values.
 *   o, z, y [n_rows][dv]; w [dv] shared by every row.
 */
int oracle_gated_rmsnorm(const double *o, const double *z, const double *w,
                         double eps, double *y, int64_t n_rows, int64_t dv)
{
    if (n_rows < 0 || dv <= 0)
        return -1;
    for (int64_t r = 0; r < n_rows; ++r)
        gated_rmsnorm_head(o + r * dv, z + r * dv, w, eps, y + r * dv, dv);
    return 0;
}

/*
 * The single-token recurrent layer, [L]: prestate -> recurrence [S] for
 * every value head -> gated RMSNorm tail, for the listed sequences.
 *   mixed_qkv [B][C]; z [B][Hv*dv]; a_in, b_in [B][Hv]
 *   ring [B][K-1][C] in/out; conv_w [C][K]; A_log, dt_bias [Hv]; norm_w [dv]
 *   state [B][Hv][dv][dk] in/out; out [B][Hv*dv]
 */
int oracle_gdn_layer_decode(const double *mixed_qkv, const double *z,
                            const double *a_in, const double *b_in,
                            double *ring, const double *conv_w,
                            const double *A_log, const double *dt_bias,
                            const double *norm_w, double l2_eps,
                            double norm_eps, double *state, double *out,
                            int64_t B, int64_t Hk, int64_t Hv, int64_t dk,
                            int64_t dv, int64_t K, const int64_t *seqs,
                            int64_t n_seqs)
{
    if (B < 0 || K < 1 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t C = 2 * Hk * dk + Hv * dv;
    const int64_t count = seqs ? n_seqs : B;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        if (b < 0 || b >= B)
            return -1;
    }
    double *q = (double *)malloc((size_t)(Hk * dk) * sizeof(double));
    double *k = (double *)malloc((size_t)(Hk * dk) * sizeof(double));
    double *v = (double *)malloc((size_t)(Hv * dv) * sizeof(double));
    double *beta = (double *)malloc((size_t)Hv * sizeof(double));
    double *gate = (double *)malloc((size_t)Hv * sizeof(double));
    double *o = (double *)malloc((size_t)dv * sizeof(double));
    int rc = (q && k && v && beta && gate && o) ? 0 : -2;
    for (int64_t n = 0; rc == 0 && n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        rc = prestate_token(mixed_qkv + b * C, ring + b * (K - 1) * C, conv_w,
                            a_in + b * Hv, b_in + b * Hv, A_log, dt_bias,
                            l2_eps, q, k, v, beta, gate, Hk, Hv, dk, dv, K);
        for (int64_t h = 0; rc == 0 && h < Hv; ++h) {
            const int64_t g = h % Hk;
            rc = gdn_head_token(state + (b * Hv + h) * dv * dk, q + g * dk,
                                k + g * dk, v + h * dv, beta[h], gate[h], o,
                                dk, dv);
            if (rc == 0)
                gated_rmsnorm_head(o, z + b * Hv * dv + h * dv, norm_w,
                                   norm_eps, out + b * Hv * dv + h * dv, dv);
        }
    }
    free(q);
    free(k);
    free(v);
    free(beta);
    free(gate);
    free(o);
    return rc;
}

/*
 * Two-position speculative verify of the single-token layer, [B] entry
 * "gdn_pair" and [L]: position 1 runs the layer and commits (ring and state
 * are updated in place); position 2 continues from that committed result
 * and its ring and state go to scratch (the caller keeps them on accept and
 * drops them on reject). Plainly: two calls of the one-token layer, the
 * first on the live buffers, the second on copies of them.
 *   mixed_qkv [B][2][C]; z [B][2][Hv*dv]; a_in, b_in [B][2][Hv]
 *   ring [B][K-1][C] in/out; state [B][Hv][dv][dk] in/out
 *   scratch_ring [B][K-1][C] out; scratch_state [B][Hv][dv][dk] out
 *   out [B][2][Hv*dv]
 */
int oracle_gdn_layer_pair(const double *mixed_qkv, const double *z,
                          const double *a_in, const double *b_in,
                          double *ring, const double *conv_w,
                          const double *A_log, const double *dt_bias,
                          const double *norm_w, double l2_eps,
                          double norm_eps, double *state,
                          double *scratch_ring, double *scratch_state,
                          double *out, int64_t B, int64_t Hk, int64_t Hv,
                          int64_t dk, int64_t dv, int64_t K,
                          const int64_t *seqs, int64_t n_seqs)
{
    if (B < 0 || K < 1 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t C = 2 * Hk * dk + Hv * dv;
    const int64_t count = seqs ? n_seqs : B;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        if (b < 0 || b >= B)
            return -1;
    }
    for (int64_t n = 0; n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        double *rg = ring + b * (K - 1) * C;
        double *st = state + b * Hv * dv * dk;
        double *srg = scratch_ring + b * (K - 1) * C;
        double *sst = scratch_state + b * Hv * dv * dk;
        /* lane 1: commits into the live ring and state */
        int rc = oracle_gdn_layer_decode(mixed_qkv + (b * 2 + 0) * C,
                                         z + (b * 2 + 0) * Hv * dv,
                                         a_in + (b * 2 + 0) * Hv,
                                         b_in + (b * 2 + 0) * Hv, rg, conv_w,
                                         A_log, dt_bias, norm_w, l2_eps,
                                         norm_eps, st, out + (b * 2 + 0) * Hv * dv,
                                         1, Hk, Hv, dk, dv, K, NULL, 0);
        if (rc)
            return rc;
        /* lane 2: continues on copies of the committed ring and state */
        memcpy(srg, rg, (size_t)((K - 1) * C) * sizeof(double));
        memcpy(sst, st, (size_t)(Hv * dv * dk) * sizeof(double));
        rc = oracle_gdn_layer_decode(mixed_qkv + (b * 2 + 1) * C,
                                     z + (b * 2 + 1) * Hv * dv,
                                     a_in + (b * 2 + 1) * Hv,
                                     b_in + (b * 2 + 1) * Hv, srg, conv_w, A_log,
                                     dt_bias, norm_w, l2_eps, norm_eps, sst,
                                     out + (b * 2 + 1) * Hv * dv, 1, Hk, Hv, dk,
                                     dv, K, NULL, 0);
        if (rc)
            return rc;
    }
    return 0;
}

/* Nearest bf16 value (round half to even) of x, for normal-range x: keep 8
 * significant bits of the binary significand. */
static double round_to_bf16(double x)
{
    if (x == 0.0 || !isfinite(x))
        return x;
    int e;
    const double m = frexp(x, &e);          /* x = m 2^e, 0.5 <= |m| < 1 */
    return ldexp(nearbyint(ldexp(m, 8)), e - 8);
}

/*
 * The layer for T positions of B sequences with dense projections, [L] and
 * [B] entry "gdn_forward_batch". Position by position, in order:
 *   mixed = W_qkv h_t,  z = W_z h_t,  (b_in | a_in) = W_ba h_t   (matvecs)
 *   prestate -> recurrence of every value head -> gated RMSNorm tail (as in
 *   oracle_gdn_layer_decode), then out_t = W_out y_t.
 * The tail output y is rounded to bf16 before the output projection when
 * round_y is non-zero (the precision the projection consumes).
 *   hidden [B][T][D]; W_qkv [C][D], C = 2*Hk*dk + Hv*dv; W_z [Hv*dv][D];
 *   W_ba [2*Hv][D] (rows 0..Hv-1 give b, rows Hv..2Hv-1 give a);
 *   W_out [D][Hv*dv]; ring [B][K-1][C] in/out; state [B][Hv][dv][dk] in/out;
 *   out [B][T][D].
 */
int oracle_gdn_forward_batch(const double *hidden, const double *W_qkv,
                             const double *W_z, const double *W_ba,
                             const double *W_out, double *ring,
                             const double *conv_w, const double *A_log,
                             const double *dt_bias, const double *norm_w,
                             double l2_eps, double norm_eps, double *state,
                             double *out, int64_t B, int64_t T, int64_t D,
                             int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                             int64_t K, int round_y, const int64_t *seqs,
                             int64_t n_seqs)
{
    if (B < 0 || T < 0 || D <= 0 || K < 1 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t C = 2 * Hk * dk + Hv * dv;
    const int64_t HD = Hv * dv;
    const int64_t count = seqs ? n_seqs : B;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        if (b < 0 || b >= B)
            return -1;
    }
    double *mixed = (double *)malloc((size_t)C * sizeof(double));
    double *z = (double *)malloc((size_t)HD * sizeof(double));
    double *ab = (double *)malloc((size_t)(2 * Hv) * sizeof(double));
    double *y = (double *)malloc((size_t)HD * sizeof(double));
    int rc = (mixed && z && ab && y) ? 0 : -2;
    for (int64_t n = 0; rc == 0 && n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        for (int64_t t = 0; rc == 0 && t < T; ++t) {
            const double *h = hidden + (b * T + t) * D;
            for (int64_t r = 0; r < C; ++r) {
                double acc = 0.0;
                for (int64_t i = 0; i < D; ++i)
                    acc += W_qkv[r * D + i] * h[i];
                mixed[r] = acc;
            }
            for (int64_t r = 0; r < HD; ++r) {
                double acc = 0.0;
                for (int64_t i = 0; i < D; ++i)
                    acc += W_z[r * D + i] * h[i];
                z[r] = acc;
            }
            for (int64_t r = 0; r < 2 * Hv; ++r) {
                double acc = 0.0;
                for (int64_t i = 0; i < D; ++i)
                    acc += W_ba[r * D + i] * h[i];
                ab[r] = acc;
            }
            /* b_in = ab[0..Hv), a_in = ab[Hv..2Hv) */
            rc = oracle_gdn_layer_decode(mixed, z, ab + Hv, ab, ring + b * (K - 1) * C,
                                         conv_w, A_log, dt_bias, norm_w, l2_eps,
                                         norm_eps, state + b * Hv * dv * dk, y, 1, Hk,
                                         Hv, dk, dv, K, NULL, 0);
            if (rc)
                break;
            if (round_y)
                for (int64_t r = 0; r < HD; ++r)
                    y[r] = round_to_bf16(y[r]);
            double *o = out + (b * T + t) * D;
            for (int64_t r = 0; r < D; ++r) {
                double acc = 0.0;
                for (int64_t i = 0; i < HD; ++i)
                    acc += W_out[r * HD + i] * y[i];
                o[r] = acc;
            }
        }
    }
    free(mixed);
    free(z);
    free(ab);
    free(y);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* LFM2 short-convolution mixer. [SC] "Module linear_core", struct          */
/* "ShortConvWeights" and entries "short_conv_forward",                     */
/* "short_conv_forward_batch", "short_conv_pair": no recurrent state, only  */
/* the causal conv ring holding the last K-1 gated inputs of each channel;   */
/* in_proj and out_proj are matrix products, the conv walks the positions    */
/* in order. Readings (the pages give no formula): in_proj maps D to 3D     */
/* rows split into the input gate bg = rows [0, D), the output gate         */
/* cg = rows [D, 2D) and the value xv = rows [2D, 3D); the gated input is   */
/* u = bg * xv; conv = sum_t conv_w[d][t] * window[t] over the window       */
/* (ring[0..K-2], u) oldest first, no bias; y = cg * conv; out = W_out y.   */
/* ------------------------------------------------------------------------ */

/* One position of one sequence: h [D] -> o [D]; ring [K-1][D] advances. */
static int short_conv_token(const double *h, const double *W_in,
                            const double *W_out, double *ring,
                            const double *conv_w, double *o, int64_t D,
                            int64_t K, int round_y, double *proj, double *y,
                            double *window)
{
    for (int64_t r = 0; r < 3 * D; ++r) {
        double acc = 0.0;
        for (int64_t i = 0; i < D; ++i)
            acc += W_in[r * D + i] * h[i];
        proj[r] = acc;
    }
    const double *bg = proj;
    const double *cg = proj + D;
    const double *xv = proj + 2 * D;
    for (int64_t d = 0; d < D; ++d) {
        for (int64_t t = 0; t < K - 1; ++t)
            window[t] = ring[t * D + d];
        window[K - 1] = bg[d] * xv[d];
        double conv = 0.0;
        for (int64_t t = 0; t < K; ++t)
            conv += conv_w[d * K + t] * window[t];
        for (int64_t t = 0; t < K - 1; ++t)
            ring[t * D + d] = window[t + 1];
        y[d] = cg[d] * conv;
        if (round_y)
            y[d] = round_to_bf16(y[d]);
    }
    for (int64_t r = 0; r < D; ++r) {
        double acc = 0.0;
        for (int64_t i = 0; i < D; ++i)
            acc += W_out[r * D + i] * y[i];
        o[r] = acc;
    }
    return 0;
}

/*
 * T positions of B sequences, [SC] "short_conv_forward_batch" (T = 1 is
 * "short_conv_forward"). hidden [B][T][D]; W_in [3D][D]; W_out [D][D];
 * ring [B][K-1][D] in/out; conv_w [D][K]; out [B][T][D]. round_y rounds y
 * to the nearest bf16 value (ties to even) before the output projection.
 * seqs (optional) restricts the work to the listed sequences.
 */
int oracle_short_conv_forward_batch(const double *hidden, const double *W_in,
                                    const double *W_out, double *ring,
                                    const double *conv_w, double *out,
                                    int64_t B, int64_t T, int64_t D, int64_t K,
                                    int round_y, const int64_t *seqs,
                                    int64_t n_seqs)
{
    if (B < 0 || T < 0 || D <= 0 || K < 1)
        return -1;
    const int64_t count = seqs ? n_seqs : B;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        if (b < 0 || b >= B)
            return -1;
    }
    double *proj = (double *)malloc((size_t)(3 * D) * sizeof(double));
    double *y = (double *)malloc((size_t)D * sizeof(double));
    double *window = (double *)malloc((size_t)K * sizeof(double));
    int rc = (proj && y && window) ? 0 : -2;
    for (int64_t n = 0; rc == 0 && n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        for (int64_t t = 0; rc == 0 && t < T; ++t)
            rc = short_conv_token(hidden + (b * T + t) * D, W_in, W_out,
                                  ring + b * (K - 1) * D, conv_w,
                                  out + (b * T + t) * D, D, K, round_y, proj, y,
                                  window);
    }
    free(proj);
    free(y);
    free(window);
    return rc;
}

/*
 * Two positions per sequence, [SC] "short_conv_pair": position 0 commits
 * into ring; position 1 continues from a copy of the committed ring and
 * leaves its ring in scratch_ring [B][K-1][D]. hidden [B][2][D],
 * out [B][2][D].
 */
int oracle_short_conv_pair(const double *hidden, const double *W_in,
                           const double *W_out, double *ring,
                           double *scratch_ring, const double *conv_w,
                           double *out, int64_t B, int64_t D, int64_t K,
                           int round_y, const int64_t *seqs, int64_t n_seqs)
{
    if (B < 0 || D <= 0 || K < 1)
        return -1;
    const int64_t count = seqs ? n_seqs : B;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        if (b < 0 || b >= B)
            return -1;
    }
    double *proj = (double *)malloc((size_t)(3 * D) * sizeof(double));
    double *y = (double *)malloc((size_t)D * sizeof(double));
    double *window = (double *)malloc((size_t)K * sizeof(double));
    int rc = (proj && y && window) ? 0 : -2;
    for (int64_t n = 0; rc == 0 && n < count; ++n) {
        const int64_t b = seqs ? seqs[n] : n;
        double *rg = ring + b * (K - 1) * D;
        double *srg = scratch_ring + b * (K - 1) * D;
        rc = short_conv_token(hidden + (b * 2) * D, W_in, W_out, rg, conv_w,
                              out + (b * 2) * D, D, K, round_y, proj, y, window);
        if (rc)
            break;
        memcpy(srg, rg, (size_t)((K - 1) * D) * sizeof(double));
        rc = short_conv_token(hidden + (b * 2 + 1) * D, W_in, W_out, srg, conv_w,
                              out + (b * 2 + 1) * D, D, K, round_y, proj, y,
                              window);
    }
    free(proj);
    free(y);
    free(window);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* KDA core: the delta-rule recurrence with a decay per key channel.        */
/* [K] "Module linear_core", entries "kda_forward" (one position, advances  */
/* the state) and "kda_forward_batch" (the recurrence sequential per        */
/* position). The pages give no equations; the reading is the published    */
/* Kimi Delta Attention update S_t = (I - b k k^T) Diag(a_t) S_{t-1}        */
/* + b k v^T, o_t = S_t^T q_t, with a_t = exp(g_t) per key channel and the  */
/* scale 1/sqrt(dk) of the one-position path. In the transposed layout      */
/* M[j][i] = S[i][j] the five steps of [S] hold with step 1 decaying column */
/* i by exp(g[i]).                                                          */
/* ------------------------------------------------------------------------ */
static int kda_head_token(double *M, const double *q, const double *k,
                          const double *v, double beta, const double *g,
                          double *out, int64_t dk, int64_t dv)
{
    double *sk = (double *)malloc((size_t)dv * sizeof(double));
    double *delta = (double *)malloc((size_t)dv * sizeof(double));
    double *alpha = (double *)malloc((size_t)dk * sizeof(double));
    if (!sk || !delta || !alpha) {
        free(sk);
        free(delta);
        free(alpha);
        return -2;
    }

    /* step 1: column i of M decays by exp(g[i]) */
    for (int64_t i = 0; i < dk; ++i)
        alpha[i] = exp(g[i]);
    for (int64_t j = 0; j < dv; ++j)
        for (int64_t i = 0; i < dk; ++i)
            M[j * dk + i] *= alpha[i];

    /* step 2: sk[j] = dot(M[j], k) on the decayed state */
    for (int64_t j = 0; j < dv; ++j) {
        double dot = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            dot += M[j * dk + i] * k[i];
        sk[j] = dot;
    }

    /* step 3: delta[j] = (v[j] - sk[j]) * beta */
    for (int64_t j = 0; j < dv; ++j)
        delta[j] = beta * (v[j] - sk[j]);

    /* step 4: M[j][i] += delta[j] * k[i] */
    for (int64_t j = 0; j < dv; ++j)
        for (int64_t i = 0; i < dk; ++i)
            M[j * dk + i] += k[i] * delta[j];

    /* step 5: out[j] = dot(M[j], q) / sqrt(dk) on the updated state */
    const double root_dk = sqrt((double)dk);
    for (int64_t j = 0; j < dv; ++j) {
        double dot = 0.0;
        for (int64_t i = 0; i < dk; ++i)
            dot += M[j * dk + i] * q[i];
        out[j] = dot / root_dk;
    }

    free(sk);
    free(delta);
    free(alpha);
    return 0;
}

/*
 * KDA decode over L layers x B sequences x Hv value heads, [K]
 * "kda_forward". Shapes as oracle_gdn_step except
 *   g [L][B][Hv][dk]   log-decay per value head and key channel.
 * Value head h reads q/k of key head h % Hk.
 */
int oracle_kda_step(double *state, const double *q, const double *k,
                    const double *v, const double *beta, const double *g,
                    double *out, int64_t L, int64_t B, int64_t Hk, int64_t Hv,
                    int64_t dk, int64_t dv, const int64_t *units,
                    int64_t n_units)
{
    if (L < 0 || B < 0 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t total = L * B * Hv;
    const int64_t count = units ? n_units : total;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        if (u < 0 || u >= total)
            return -1;
    }
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        const int64_t lb = u / Hv;
        const int64_t key = lb * Hk + (u % Hv) % Hk;
        int rc = kda_head_token(state + u * dv * dk, q + key * dk, k + key * dk,
                                v + u * dv, beta[u], g + u * dk, out + u * dv,
                                dk, dv);
        if (rc)
            return rc;
    }
    return 0;
}

/*
 * KDA over T positions in order, [K] "kda_forward_batch": position t runs the
 * one-position update on the state left by position t-1.
 *   state [B][Hv][dv][dk]; q, k [B][T][Hk][dk]; v [B][T][Hv][dv];
 *   beta [B][T][Hv]; g [B][T][Hv][dk]; out [B][T][Hv][dv].
 */
int oracle_kda_prefill(double *state, const double *q, const double *k,
                       const double *v, const double *beta, const double *g,
                       double *out, int64_t B, int64_t T, int64_t Hk,
                       int64_t Hv, int64_t dk, int64_t dv,
                       const int64_t *units, int64_t n_units)
{
    if (B < 0 || T < 0 || !dims_ok(Hk, Hv, dk, dv))
        return -1;
    const int64_t total = B * Hv;
    const int64_t count = units ? n_units : total;
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        if (u < 0 || u >= total)
            return -1;
    }
    for (int64_t n = 0; n < count; ++n) {
        const int64_t u = units ? units[n] : n;
        const int64_t b = u / Hv;
        const int64_t h = u % Hv;
        double *M = state + u * dv * dk;
        for (int64_t t = 0; t < T; ++t) {
            const int64_t row = (b * T + t) * Hv + h;     /* (b, t, h) */
            const int64_t key = (b * T + t) * Hk + h % Hk;
            int rc = kda_head_token(M, q + key * dk, k + key * dk, v + row * dv,
                                    beta[row], g + row * dk, out + row * dv, dk,
                                    dv);
            if (rc)
                return rc;
        }
    }
    return 0;
}
