/*
 * gdn_oracle_f32.c -- the literal fp32 instantiation of the oracle's
 * recurrence: the same five steps as gdn_oracle.c, in the same order, with
 * every value held in float.
 *
 * TEST INFRASTRUCTURE, and not a parity reference. Parity is judged against
 * the double oracle in gdn_oracle.c; this file exists because the pages time
 * their CPU path as a plain F32 step ("Red Lite dev15c -- Gated DeltaNet
 * recurrent-state parity", section "M4 Pro ARM64 field validation": an F32
 * state, one token, on the CPU). The benchmark's CPU-baseline leg times these
 * two functions on the host cores; the CPU tests check them against the
 * double oracle within the library tolerance. Nothing here is shared with the
 * CUDA path or with gdn_oracle.c.
 *
 * Source of the arithmetic: "Red Lite dev15c", section "Pinned llama.cpp
 * semantics". For each value head h, with q/k of key head h % Hk and the
 * state held as M[j][i] = S[i][j]:
 *   1. M *= exp(gate)   2. sk[j] = M[j].k   3. delta[j] = (v[j] - sk[j]) beta
 *   4. M[j] += delta[j] k   5. out[j] = M_new[j].q / sqrt(dk)
 * Sums run in ascending index order, one rounding per operation (the build
 * disables contraction into fused multiply-adds).
 *
 * Return codes: 0 on success, -1 on a bad argument (nothing is written),
 * -2 when a scratch allocation fails.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/* One value head, one token: M is [dv][dk]. */
static int head_token_f32(float *M, const float *q, const float *k, const float *v,
                          float beta, float gate, float *out, int64_t dk, int64_t dv)
{
    float *delta = (float *)malloc((size_t)dv * sizeof(float));
    if (!delta)
        return -2;
    const float decay = expf(gate);                      /* step 1 */
    for (int64_t j = 0; j < dv; ++j)
        for (int64_t i = 0; i < dk; ++i)
            M[j * dk + i] *= decay;
    for (int64_t j = 0; j < dv; ++j) {                   /* steps 2 and 3 */
        float sk = 0.0f;
        for (int64_t i = 0; i < dk; ++i)
            sk += M[j * dk + i] * k[i];
        delta[j] = (v[j] - sk) * beta;
    }
    for (int64_t j = 0; j < dv; ++j)                     /* step 4 */
        for (int64_t i = 0; i < dk; ++i)
            M[j * dk + i] += delta[j] * k[i];
    const float root_dk = sqrtf((float)dk);
    for (int64_t j = 0; j < dv; ++j) {                   /* step 5, updated state */
        float acc = 0.0f;
        for (int64_t i = 0; i < dk; ++i)
            acc += M[j * dk + i] * q[i];
        out[j] = acc / root_dk;
    }
    free(delta);
    return 0;
}

static int dims_ok_f32(int64_t Hk, int64_t Hv, int64_t dk, int64_t dv)
{
    return Hk > 0 && Hv > 0 && dk > 0 && dv > 0 && Hv % Hk == 0;
}

/*
 * Decode, one token per (layer, sequence, value head) unit; the layouts of
 * oracle_gdn_step in float:
 *   state [L][B][Hv][dv][dk] in/out; q, k [L][B][Hk][dk]; v, out [L][B][Hv][dv];
 *   beta, gate [L][B][Hv].
 * units: flat indices u = (l*B + b)*Hv + h, or NULL for all.
 */
int oracle_gdn_step_f32(float *state, const float *q, const float *k, const float *v,
                        const float *beta, const float *gate, float *out, int64_t L,
                        int64_t B, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                        const int64_t *units, int64_t n_units)
{
    if (L < 0 || B < 0 || !dims_ok_f32(Hk, Hv, dk, dv))
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
        const int64_t lb = u / Hv, h = u % Hv, g = h % Hk;
        int rc = head_token_f32(state + u * dv * dk, q + (lb * Hk + g) * dk,
                                k + (lb * Hk + g) * dk, v + u * dv, beta[u], gate[u],
                                out + u * dv, dk, dv);
        if (rc)
            return rc;
    }
    return 0;
}

/*
 * Sequential prefill: position t runs the one-token recurrence on the state
 * left by position t-1 ("Module linear_core", entry "gdn_forward_batch").
 * Layouts of oracle_gdn_prefill in float:
 *   state [B][Hv][dv][dk] in/out; q, k [B][T][Hk][dk]; v, out [B][T][Hv][dv];
 *   beta, gate [B][T][Hv].
 * units: flat indices u = b*Hv + h, or NULL for all.
 */
int oracle_gdn_prefill_f32(float *state, const float *q, const float *k, const float *v,
                           const float *beta, const float *gate, float *out, int64_t B,
                           int64_t T, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv,
                           const int64_t *units, int64_t n_units)
{
    if (B < 0 || T < 0 || !dims_ok_f32(Hk, Hv, dk, dv))
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
        const int64_t b = u / Hv, h = u % Hv, g = h % Hk;
        for (int64_t t = 0; t < T; ++t) {
            const int64_t bt = b * T + t;
            int rc = head_token_f32(state + u * dv * dk, q + (bt * Hk + g) * dk,
                                    k + (bt * Hk + g) * dk, v + (bt * Hv + h) * dv,
                                    beta[bt * Hv + h], gate[bt * Hv + h],
                                    out + (bt * Hv + h) * dv, dk, dv);
            if (rc)
                return rc;
        }
    }
    return 0;
}
