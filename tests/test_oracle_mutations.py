"""Plant plausible mistakes in copies of the oracle's C source and check that
the pins catch every one of them.

Each mutation edits exactly one spot of ``oracle/gdn_oracle.c`` (the target
text must occur once), is compiled into a temporary library with the same
flags as the real build, and is run through all pins in
``oracle_pins.ALL_PINS``. A mutation that no pin detects means the pins have
a blind spot. Every edit keeps all memory accesses in bounds.
"""
import os
import tempfile

import pytest

from oracle import build as oracle_build
from oracle.gdn_oracle import Oracle, OracleError
from oracle_pins import ALL_PINS

MUTATIONS = [
    # recurrence, "Pinned llama.cpp semantics" steps 1-5
    ("decay dropped", "M[j * dk + i] *= decay;", "M[j * dk + i] *= 1.0;"),
    ("decay uses -gate", "const double decay = exp(gate);", "const double decay = exp(-gate);"),
    ("sk reads q", "acc += M[j * dk + i] * k[i];\n        sk[j] = acc;",
     "acc += M[j * dk + i] * q[i];\n        sk[j] = acc;"),
    ("delta sign", "delta[j] = (v[j] - sk[j]) * beta;", "delta[j] = (sk[j] - v[j]) * beta;"),
    ("beta dropped", "delta[j] = (v[j] - sk[j]) * beta;", "delta[j] = (v[j] - sk[j]);"),
    ("update sign", "M[j * dk + i] += delta[j] * k[i];", "M[j * dk + i] -= delta[j] * k[i];"),
    ("update writes q", "M[j * dk + i] += delta[j] * k[i];", "M[j * dk + i] += delta[j] * q[i];"),
    ("output reads k", "acc += M[j * dk + i] * q[i];\n        out[j]",
     "acc += M[j * dk + i] * k[i];\n        out[j]"),
    ("output scale dropped", "out[j] = acc / scale_div;", "out[j] = acc;"),
    ("output scale 1/dk", "const double scale_div = sqrt((double)dk);",
     "const double scale_div = (double)dk;"),
    ("step broadcast h/2", "const int64_t g = h % Hk;            /* key head read by value head h */",
     "const int64_t g = h / (Hv / Hk);"),
    ("prefill broadcast h/2", "const int64_t g = h % Hk;\n        double *M",
     "const int64_t g = h / (Hv / Hk);\n        double *M"),
    ("prefill order reversed", "const int64_t bt = b * T + t;",
     "const int64_t bt = b * T + (T - 1 - t);"),
    # two-position verify ("Module linear_core", entry "gdn_pair")
    ("pair position 1 from the input state",
     "memcpy(tent, live, (size_t)(dv * dk) * sizeof(double));",
     "memset(tent, 0, (size_t)(dv * dk) * sizeof(double));"),
    ("pair positions swapped", "const int64_t lbp = lb * 2 + pos;",
     "const int64_t lbp = lb * 2 + (1 - pos);"),
    ("pair commits position 1", "double *M = pos == 0 ? live : tent;",
     "double *M = live;"),
    # prestate
    ("conv taps reversed", "acc += w[c * K + t] * win;", "acc += w[c * K + (K - 1 - t)] * win;"),
    ("ring not refreshed", "ring[(K - 2) * C + c] = x[c];",
     "ring[(K - 2) * C + c] = ring[(K - 2) * C + c];"),
    ("ring stores conv output", "ring[(K - 2) * C + c] = x[c];", "ring[(K - 2) * C + c] = y[c];"),
    ("silu is sigmoid", "static double silu(double x) { return x / (1.0 + exp(-x)); }",
     "static double silu(double x) { return 1.0 / (1.0 + exp(-x)); }"),
    ("softplus lost max", "return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));",
     "return log1p(exp(-fabs(x)));"),
    ("gate sign", "gate[h] = -exp(A_log[h]) *", "gate[h] = exp(A_log[h]) *"),
    ("gate drops dt_bias", "softplus(a_in[h] + dt_bias[h]);", "softplus(a_in[h]);"),
    ("beta not squashed", "beta[h] = sigmoid(b_in[h]);", "beta[h] = b_in[h];"),
    ("no L2 norm", "x[i] = x[i] / norm;", "x[i] = x[i];"),
    ("q takes k slice", "memcpy(q, y, ", "memcpy(q, y + Hk * dk, "),
    # tail
    ("rms eps outside sqrt", "1.0 / sqrt(ss / (double)dv + eps);",
     "1.0 / (sqrt(ss / (double)dv) + eps);"),
    ("rms sum not mean", "1.0 / sqrt(ss / (double)dv + eps);", "1.0 / sqrt(ss + eps);"),
    ("tail weight dropped", "y[j] = o[j] * inv_rms * w[j] * silu(z[j]);",
     "y[j] = o[j] * inv_rms * silu(z[j]);"),
    ("tail gate not silu", "y[j] = o[j] * inv_rms * w[j] * silu(z[j]);",
     "y[j] = o[j] * inv_rms * w[j] * z[j];"),
    ("layer broadcast h/2", "const int64_t g = h % Hk;\n            rc = gdn_head_token",
     "const int64_t g = h / (Hv / Hk);\n            rc = gdn_head_token"),
    ("layer tail reads head 0 z", "z + b * Hv * dv + h * dv, norm_w", "z + b * Hv * dv, norm_w"),
    # two-position verify
    ("pair lane 2 reuses lane 1 input", "rc = oracle_gdn_layer_decode(mixed_qkv + (b * 2 + 1) * C,",
     "rc = oracle_gdn_layer_decode(mixed_qkv + (b * 2 + 0) * C,"),
    ("pair scratch starts from lane-2 ring slot", "memcpy(srg, rg, (size_t)((K - 1) * C) * sizeof(double));",
     "memcpy(srg, rg, (size_t)((K - 1) * C) * sizeof(double)); srg[0] = srg[1];"),
    # batched forward with projections
    ("forward a/b swapped", "rc = oracle_gdn_layer_decode(mixed, z, ab + Hv, ab,",
     "rc = oracle_gdn_layer_decode(mixed, z, ab, ab + Hv,"),
    ("forward y not rounded", "y[r] = round_to_bf16(y[r]);", "y[r] = y[r];"),
    ("bf16 keeps 9 bits", "return ldexp(nearbyint(ldexp(m, 8)), e - 8);",
     "return ldexp(nearbyint(ldexp(m, 9)), e - 9);"),
    # KDA core
    ("kda decay per row", "M[j * dk + i] *= alpha[i];", "M[j * dk + i] *= alpha[j % dk];"),
    ("kda decay dropped", "alpha[i] = exp(g[i]);", "alpha[i] = 1.0;"),
    ("kda decay sign", "alpha[i] = exp(g[i]);", "alpha[i] = exp(-g[i]);"),
    ("kda sk reads q", "dot += M[j * dk + i] * k[i];", "dot += M[j * dk + i] * q[i];"),
    ("kda delta sign", "delta[j] = beta * (v[j] - sk[j]);", "delta[j] = beta * (sk[j] - v[j]);"),
    ("kda update writes q", "M[j * dk + i] += k[i] * delta[j];", "M[j * dk + i] += q[i] * delta[j];"),
    ("kda output unscaled", "out[j] = dot / root_dk;", "out[j] = dot;"),
    ("kda step decay of the key head", "beta[u], g + u * dk,", "beta[u], g + key * dk,"),
    ("kda prefill decay of position 0", "beta[row], g + row * dk,",
     "beta[row], g + (b * T * Hv + h) * dk,"),
    ("kda prefill broadcast h/2", "const int64_t key = (b * T + t) * Hk + h % Hk;",
     "const int64_t key = (b * T + t) * Hk + h / (Hv / Hk);"),
    # LFM2 short-conv mixer
    ("short conv gates swapped", "const double *bg = proj;", "const double *bg = proj + D;"),
    ("short conv input gate dropped", "window[K - 1] = bg[d] * xv[d];", "window[K - 1] = xv[d];"),
    ("short conv output gate dropped", "y[d] = cg[d] * conv;", "y[d] = conv;"),
    ("short conv taps reversed", "conv += conv_w[d * K + t] * window[t];",
     "conv += conv_w[d * K + (K - 1 - t)] * window[t];"),
    ("short conv ring not shifted", "ring[t * D + d] = window[t + 1];",
     "ring[t * D + d] = window[t];"),
    ("short conv y not rounded", "y[d] = round_to_bf16(y[d]);", "y[d] = y[d];"),
    ("short conv pair lane 2 commits", "rc = short_conv_token(hidden + (b * 2 + 1) * D, W_in, W_out, srg,",
     "rc = short_conv_token(hidden + (b * 2 + 1) * D, W_in, W_out, rg,"),
]


@pytest.fixture(scope="module")
def source():
    with open(oracle_build.SOURCE) as fh:
        return fh.read()


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(source, name, old, new):
    assert source.count(old) == 1, f"mutation target for '{name}' must occur exactly once"
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "mutant.c")
        lib = os.path.join(tmp, "libmutant.so")
        with open(src, "w") as fh:
            fh.write(source.replace(old, new))
        oracle_build.build(src, lib, force=True)
        mutant = Oracle(lib)
        caught = []
        for pin in ALL_PINS:
            try:
                pin(mutant)
            except (AssertionError, OracleError) as exc:
                caught.append(f"{pin.__name__}: {str(exc).splitlines()[0][:80]}")
        assert caught, f"no pin detects mutation '{name}'"
