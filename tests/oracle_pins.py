"""Pins that tie the fp64 oracle to facts outside itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` handle and raises
AssertionError when the oracle disagrees with:
  * hand-expanded dyadic cases stored in ``tests/golden`` (bit-exact),
  * closed forms of the delta rule,
  * the textbook matrix (product) form of the gated delta rule, written with
    matrix products in the S^T convention, on non-square heads so a
    transposed operand cannot pass,
  * torch's own conv1d / silu / normalize / softplus / rms_norm routines.

Equations: "Red Lite dev15c -- Gated DeltaNet recurrent-state parity",
section "Pinned llama.cpp semantics" (steps 1-5, transposed layout, key-head
broadcast h % 16); "Red Lite dev15e -- complete recurrent DeltaNet layer
composition" (prestate, tail); "Module linear_core", entry
"gdn_forward_batch" (sequential prefill).

The same functions run against deliberately broken builds of the oracle in
``test_oracle_mutations.py``; every planted mistake must trip at least one.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------
def _parse_num(tok: str) -> float:
    if "/" in tok:
        return float(Fraction(tok))
    return float(tok)


def load_golden(name: str) -> dict:
    """Parse a ``key: v v v`` fixture; repeated keys stack into a matrix."""
    rows: dict = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, vals = line.split(":", 1)
            rows.setdefault(key.strip(), []).append([_parse_num(t) for t in vals.split()])
    out = {}
    for key, lst in rows.items():
        arr = np.array(lst, dtype=np.float64)
        out[key] = arr if arr.shape[0] > 1 else arr[0]
    return out


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def textbook_head(M, q, k, v, beta, gate):
    """Gated delta rule in product form with S = M^T (value-major rows):
    M_new = exp(gate) * M (I - beta k k^T) + beta v k^T ;  out = M_new q / sqrt(dk).
    """
    dk = k.shape[0]
    eye = np.eye(dk)
    M_new = math.exp(gate) * M @ (eye - beta * np.outer(k, k)) + beta * np.outer(v, k)
    return M_new, (M_new @ q) / math.sqrt(dk)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# --------------------------------------------------------------------------
# recurrence pins
# --------------------------------------------------------------------------
def pin_golden_step_cases(o):
    for name in ("gdn_step_dk4_unit_decay.txt", "gdn_step_dk4_half_decay.txt"):
        g = load_golden(name)
        M = g["M"].reshape(1, 1, 1, 4, 4)
        st, out = o.step(M, g["q"].reshape(1, 1, 1, 4), g["k"].reshape(1, 1, 1, 4),
                         g["v"].reshape(1, 1, 1, 4), np.array([[[g["beta"]]]]).reshape(1, 1, 1),
                         np.array([g["gate"]]).reshape(1, 1, 1))
        if g["exact"] == 1:
            assert np.array_equal(st[0, 0, 0], g["expect_M"]), f"{name}: state not bit-exact"
            assert np.array_equal(out[0, 0, 0], g["expect_out"]), f"{name}: out not bit-exact"
        else:
            _close(st[0, 0, 0], g["expect_M"], 4e-16, f"{name} state")
            _close(out[0, 0, 0], g["expect_out"], 4e-16, f"{name} out")


def pin_delta_rule_closed_form(o):
    """gate = 0, beta = 1, |k| = 1: the updated state maps k to v exactly,
    and reading with q = k returns v / sqrt(dk)."""
    r = _rng(11)
    for dk, dv in ((128, 128), (16, 8), (8, 24)):
        Hk, Hv = 2, 4
        M = r.normal(0, 0.5, (1, 2, Hv, dv, dk))
        k = _unit_rows(r.normal(size=(1, 2, Hk, dk)))
        v = r.normal(size=(1, 2, Hv, dv))
        beta = np.ones((1, 2, Hv))
        gate = np.zeros((1, 2, Hv))
        st, out = o.step(M, k, k, v, beta, gate)
        for b in range(2):
            for h in range(Hv):
                kg = k[0, b, h % Hk]
                _close(st[0, b, h] @ kg, v[0, b, h], 1e-12, "M_new k = v")
                _close(out[0, b, h], v[0, b, h] / math.sqrt(dk), 1e-12, "out = v/sqrt(dk)")


def pin_zero_key(o):
    """k = 0: sk = 0, the state is only decayed, out = exp(gate) M q / sqrt(dk)."""
    r = _rng(12)
    dk, dv, Hk, Hv = 16, 8, 1, 2
    M = r.normal(size=(1, 1, Hv, dv, dk))
    q = r.normal(size=(1, 1, Hk, dk))
    k = np.zeros((1, 1, Hk, dk))
    v = r.normal(size=(1, 1, Hv, dv))
    beta = r.uniform(0.1, 0.9, (1, 1, Hv))
    gate = r.uniform(-1, 0, (1, 1, Hv))
    st, out = o.step(M, q, k, v, beta, gate)
    for h in range(Hv):
        e = math.exp(gate[0, 0, h])
        _close(st[0, 0, h], e * M[0, 0, h], 1e-15, "k=0 state")
        _close(out[0, 0, h], e * (M[0, 0, h] @ q[0, 0, 0]) / math.sqrt(dk), 1e-13, "k=0 out")


def pin_zero_beta(o):
    """beta = 0: no write, the state is only decayed."""
    r = _rng(13)
    dk, dv = 8, 16
    M = r.normal(size=(1, 1, 1, dv, dk))
    q = r.normal(size=(1, 1, 1, dk))
    k = _unit_rows(r.normal(size=(1, 1, 1, dk)))
    v = r.normal(size=(1, 1, 1, dv))
    gate = np.array([[[-0.3]]])
    st, out = o.step(M, q, k, v, np.zeros((1, 1, 1)), gate)
    e = math.exp(-0.3)
    _close(st[0, 0, 0], e * M[0, 0, 0], 1e-15, "beta=0 state")
    _close(out[0, 0, 0], e * M[0, 0, 0] @ q[0, 0, 0] / math.sqrt(dk), 1e-13, "beta=0 out")


def pin_textbook_step(o):
    """Random non-square heads with Hv = 2 Hk: the five steps equal the
    product form, with value head h reading key head h % Hk."""
    r = _rng(14)
    L, B, Hk, Hv, dk, dv = 2, 3, 4, 8, 16, 8
    M = r.normal(0, 0.3, (L, B, Hv, dv, dk))
    q = _unit_rows(r.normal(size=(L, B, Hk, dk)))
    k = _unit_rows(r.normal(size=(L, B, Hk, dk)))
    v = r.normal(size=(L, B, Hv, dv))
    beta = r.uniform(0, 1, (L, B, Hv))
    gate = r.uniform(-1, 0, (L, B, Hv))
    st, out = o.step(M, q, k, v, beta, gate)
    for l in range(L):
        for b in range(B):
            for h in range(Hv):
                g = h % Hk
                Mn, on = textbook_head(M[l, b, h], q[l, b, g], k[l, b, g], v[l, b, h],
                                       beta[l, b, h], gate[l, b, h])
                _close(st[l, b, h], Mn, 1e-12, f"textbook state l{l} b{b} h{h}")
                _close(out[l, b, h], on, 1e-12, f"textbook out l{l} b{b} h{h}")


def pin_broadcast_marker(o):
    """Only key head 3 carries a key: with a zero state, only value heads
    3 and 3 + Hk (h % Hk == 3) may produce output or state."""
    Hk, Hv, dk, dv = 16, 32, 8, 8
    r = _rng(15)
    M = np.zeros((1, 1, Hv, dv, dk))
    k = np.zeros((1, 1, Hk, dk))
    k[0, 0, 3] = _unit_rows(r.normal(size=dk))
    q = k.copy()
    v = r.normal(size=(1, 1, Hv, dv))
    beta = np.full((1, 1, Hv), 0.5)
    gate = np.zeros((1, 1, Hv))
    st, out = o.step(M, q, k, v, beta, gate)
    live = [h for h in range(Hv) if np.any(out[0, 0, h] != 0) or np.any(st[0, 0, h] != 0)]
    assert live == [3, 19], f"heads reading key head 3: {live}"


def pin_prefill_associative_memory(o):
    """Orthonormal keys: each write lands in a fresh direction, so
    M_T = sum_s (prod_{r>s} e_r) beta_s v_s k_s^T and a query equal to an
    earlier key reads back that value, decayed."""
    r = _rng(16)
    B, T, Hk, Hv, dk, dv = 1, 6, 1, 1, 8, 5
    basis, _ = np.linalg.qr(r.normal(size=(dk, dk)))
    keys = basis.T[:T]                                  # T orthonormal rows
    k = keys.reshape(B, T, Hk, dk)
    q = np.roll(keys, 2, axis=0).reshape(B, T, Hk, dk)  # q_t = k_{t-2 mod T}
    v = r.normal(size=(B, T, Hv, dv))
    beta = r.uniform(0.2, 1.0, (B, T, Hv))
    gate = r.uniform(-0.7, 0.0, (B, T, Hv))
    st, out = o.prefill(np.zeros((B, Hv, dv, dk)), q, k, v, beta, gate)
    e = np.exp(gate[0, :, 0])
    M = np.zeros((dv, dk))
    for t in range(T):
        M = e[t] * M + beta[0, t, 0] * np.outer(v[0, t, 0], keys[t])
        _close(out[0, t, 0], M @ q[0, t, 0] / math.sqrt(dk), 1e-12, f"assoc out t{t}")
        s = (t - 2) % T
        if s <= t:   # the queried key was already written: read it back
            want = beta[0, s, 0] * np.prod(e[s + 1:t + 1]) * v[0, s, 0] / math.sqrt(dk)
            _close(out[0, t, 0], want, 1e-12, f"assoc recall t{t}")
    _close(st[0, 0], M, 1e-12, "assoc final state")


def pin_prefill_textbook(o):
    """Random prefill on non-square heads equals the product form applied
    position by position."""
    r = _rng(17)
    B, T, Hk, Hv, dk, dv = 2, 7, 2, 4, 8, 6
    S0 = r.normal(0, 0.3, (B, Hv, dv, dk))
    q = _unit_rows(r.normal(size=(B, T, Hk, dk)))
    k = _unit_rows(r.normal(size=(B, T, Hk, dk)))
    v = r.normal(size=(B, T, Hv, dv))
    beta = r.uniform(0, 1, (B, T, Hv))
    gate = r.uniform(-0.5, 0, (B, T, Hv))
    st, out = o.prefill(S0, q, k, v, beta, gate)
    for b in range(B):
        for h in range(Hv):
            M = S0[b, h]
            for t in range(T):
                g = h % Hk
                M, on = textbook_head(M, q[b, t, g], k[b, t, g], v[b, t, h], beta[b, t, h],
                                      gate[b, t, h])
                _close(out[b, t, h], on, 1e-12, f"prefill out b{b} t{t} h{h}")
            _close(st[b, h], M, 1e-12, f"prefill state b{b} h{h}")


def pin_pair_textbook(o):
    """The two-position verify on non-square heads: the committed state, the
    scratch state and both outputs equal the product form applied at
    position 0 and then, from the committed state, at position 1."""
    r = _rng(23)
    L, B, Hk, Hv, dk, dv = 2, 2, 2, 6, 8, 6
    S0 = r.normal(0, 0.3, (L, B, Hv, dv, dk))
    q = _unit_rows(r.normal(size=(L, B, 2, Hk, dk)))
    k = _unit_rows(r.normal(size=(L, B, 2, Hk, dk)))
    v = r.normal(size=(L, B, 2, Hv, dv))
    beta = r.uniform(0, 1, (L, B, 2, Hv))
    gate = r.uniform(-0.5, 0, (L, B, 2, Hv))
    live, tent, out = o.pair(S0, q, k, v, beta, gate)
    for l in range(L):
        for b in range(B):
            for h in range(Hv):
                g = h % Hk
                M = S0[l, b, h]
                for pos in range(2):
                    M, on = textbook_head(M, q[l, b, pos, g], k[l, b, pos, g], v[l, b, pos, h],
                                          beta[l, b, pos, h], gate[l, b, pos, h])
                    _close(out[l, b, pos, h], on, 1e-12, f"pair out l{l} b{b} p{pos} h{h}")
                    _close((live if pos == 0 else tent)[l, b, h], M, 1e-12,
                           f"pair state l{l} b{b} p{pos} h{h}")
    # a unit left out keeps its state and gets zero scratch and output
    part_live, part_tent, part_out = o.pair(S0, q, k, v, beta, gate, units=[3])
    assert np.array_equal(part_live[0, 0, 0], S0[0, 0, 0]), "unlisted unit state"
    assert not part_tent[0, 0, 0].any() and not part_out[0, 0, :, 0].any(), "unlisted unit"
    _close(part_tent[0, 0, 3], tent[0, 0, 3], 0.0, "listed unit scratch")


# --------------------------------------------------------------------------
# layer pins (torch fp64 library routines)
# --------------------------------------------------------------------------
def _torch_prestate(x, ring, w, a, b, A_log, dt_bias, Hk, Hv, dk, dv, l2_eps):
    """Prestate from torch routines: depthwise causal conv1d over the window
    (ring slots oldest first, then x), SiLU, split, F.normalize, sigmoid,
    -exp(A_log) * softplus(a + dt_bias)."""
    Bn, C = x.shape
    K = w.shape[1]
    seq = torch.cat([torch.from_numpy(ring), torch.from_numpy(x)[:, None, :]], dim=1)  # [B,K,C]
    y = F.conv1d(seq.transpose(1, 2), torch.from_numpy(w)[:, None, :], groups=C)    # [B,C,1]
    y = F.silu(y[:, :, -1])
    q = F.normalize(y[:, : Hk * dk].reshape(Bn, Hk, dk), dim=-1, eps=l2_eps)
    k = F.normalize(y[:, Hk * dk: 2 * Hk * dk].reshape(Bn, Hk, dk), dim=-1, eps=l2_eps)
    v = y[:, 2 * Hk * dk:].reshape(Bn, Hv, dv)
    beta = torch.sigmoid(torch.from_numpy(b))
    gate = -torch.exp(torch.from_numpy(A_log)) * F.softplus(
        torch.from_numpy(a) + torch.from_numpy(dt_bias), threshold=60.0)
    new_ring = seq[:, 1:, :]
    return (q.numpy(), k.numpy(), v.numpy(), beta.numpy(), gate.numpy(), new_ring.numpy())


def _layer_case(seed, B=3, Hk=2, Hv=4, dk=8, dv=6, K=4):
    r = _rng(seed)
    C = 2 * Hk * dk + Hv * dv
    return dict(
        x=r.normal(size=(B, C)), z=r.normal(size=(B, Hv * dv)), a=r.normal(size=(B, Hv)),
        b=r.normal(size=(B, Hv)), ring=r.normal(size=(B, K - 1, C)),
        w=r.normal(0, 0.5, (C, K)), A_log=r.uniform(-1, 1, Hv), dt_bias=r.normal(0, 0.3, Hv),
        norm_w=1 + r.normal(0, 0.1, dv), state=r.normal(0, 0.3, (B, Hv, dv, dk)),
        Hk=Hk, Hv=Hv, dk=dk, dv=dv)


def pin_prestate_library(o):
    c = _layer_case(21)
    got = o.prestate(c["x"], c["ring"], c["w"], c["a"], c["b"], c["A_log"], c["dt_bias"],
                     Hk=c["Hk"], Hv=c["Hv"], dk=c["dk"], dv=c["dv"], l2_eps=1e-6)
    q, k, v, beta, gate, ring = _torch_prestate(c["x"], c["ring"], c["w"], c["a"], c["b"],
                                                c["A_log"], c["dt_bias"], c["Hk"], c["Hv"],
                                                c["dk"], c["dv"], 1e-6)
    _close(got["q"], q, 1e-13, "prestate q")
    _close(got["k"], k, 1e-13, "prestate k")
    _close(got["v"], v, 1e-13, "prestate v")
    _close(got["beta"], beta, 1e-15, "prestate beta")
    _close(got["gate"], gate, 1e-13, "prestate gate")
    assert np.array_equal(got["ring"], ring), "ring shift not exact"


def pin_prestate_special_values(o):
    """Tap (0,0,0,1) passes x through; tap (1,0,0,0) reads the oldest slot;
    A_log = 0, a + dt_bias = 0 gives gate = -ln 2; b = 0 gives beta = 1/2;
    a zero head stays zero under the L2 floor."""
    Hk, Hv, dk, dv, K = 1, 2, 4, 4, 4
    C = 2 * Hk * dk + Hv * dv
    r = _rng(22)
    x = r.normal(size=(1, C))
    ring = r.normal(size=(1, K - 1, C))
    x[0, :dk] = 0.0                                    # q head all zeros
    for taps, src in (((0, 0, 0, 1), x[0]), ((1, 0, 0, 0), ring[0, 0])):
        w = np.tile(np.array(taps, dtype=np.float64), (C, 1))
        got = o.prestate(x, ring, w, np.zeros((1, Hv)), np.zeros((1, Hv)), np.zeros(Hv),
                         np.zeros(Hv), Hk=Hk, Hv=Hv, dk=dk, dv=dv)
        silu = F.silu(torch.from_numpy(src)).numpy()
        _close(got["v"][0].ravel(), silu[2 * Hk * dk:], 1e-15, f"taps {taps} v")
        assert np.all(got["beta"] == 0.5), "beta(0) != 1/2"
        _close(got["gate"], np.full((1, Hv), -math.log(2.0)), 2e-16, "gate(0) != -ln2")
        if taps == (0, 0, 0, 1):
            assert np.all(got["q"] == 0.0), "zero q head must stay zero"
        assert np.array_equal(got["ring"][0, :2], ring[0, 1:]), "ring slots not shifted"
        assert np.array_equal(got["ring"][0, 2], x[0]), "newest slot is not the raw input"


def pin_tail_library(o):
    r = _rng(23)
    o_ = r.normal(0, 0.01, (5, 7))
    z = r.normal(size=(5, 7))
    w = 1 + r.normal(0, 0.1, 7)
    got = o.gated_rmsnorm(o_, z, w, eps=1e-6)
    want = F.rms_norm(torch.from_numpy(o_), (7,), weight=torch.from_numpy(w), eps=1e-6) \
        * F.silu(torch.from_numpy(z))
    _close(got, want.numpy(), 1e-13, "gated rmsnorm")


def pin_layer_library(o):
    """The whole single-token layer equals torch's routines composed with the
    product-form recurrence, on non-square heads with Hv = 2 Hk."""
    c = _layer_case(24)
    Hk, Hv, dk, dv = c["Hk"], c["Hv"], c["dk"], c["dv"]
    out, ring, st = o.layer_decode(c["x"], c["z"], c["a"], c["b"], c["ring"], c["w"],
                                   c["A_log"], c["dt_bias"], c["norm_w"], c["state"], Hk=Hk,
                                   l2_eps=1e-6, norm_eps=1e-6)
    q, k, v, beta, gate, ring_t = _torch_prestate(c["x"], c["ring"], c["w"], c["a"], c["b"],
                                                  c["A_log"], c["dt_bias"], Hk, Hv, dk, dv,
                                                  1e-6)
    assert np.array_equal(ring, ring_t), "layer ring"
    B = c["x"].shape[0]
    want = np.zeros((B, Hv * dv))
    for b in range(B):
        for h in range(Hv):
            g = h % Hk
            Mn, on = textbook_head(c["state"][b, h], q[b, g], k[b, g], v[b, h], beta[b, h],
                                   gate[b, h])
            _close(st[b, h], Mn, 1e-12, f"layer state b{b} h{h}")
            zt = torch.from_numpy(c["z"][b, h * dv:(h + 1) * dv])
            y = F.rms_norm(torch.from_numpy(on), (dv,), weight=torch.from_numpy(c["norm_w"]),
                           eps=1e-6) * F.silu(zt)
            want[b, h * dv:(h + 1) * dv] = y.numpy()
    _close(out, want, 1e-11, "layer out")


def _torch_layer(c, x, z, a, b, ring, state):
    """One token of the layer from torch routines and the product-form
    recurrence; returns (out [B, Hv*dv], new ring, new state)."""
    Hk, Hv, dk, dv = c["Hk"], c["Hv"], c["dk"], c["dv"]
    q, k, v, beta, gate, ring_t = _torch_prestate(x, ring, c["w"], a, b, c["A_log"],
                                                  c["dt_bias"], Hk, Hv, dk, dv, 1e-6)
    B = x.shape[0]
    out = np.zeros((B, Hv * dv))
    st = np.zeros_like(state)
    for bb in range(B):
        for h in range(Hv):
            g = h % Hk
            st[bb, h], on = textbook_head(state[bb, h], q[bb, g], k[bb, g], v[bb, h],
                                          beta[bb, h], gate[bb, h])
            zt = torch.from_numpy(z[bb, h * dv:(h + 1) * dv])
            y = F.rms_norm(torch.from_numpy(on), (dv,), weight=torch.from_numpy(c["norm_w"]),
                           eps=1e-6) * F.silu(zt)
            out[bb, h * dv:(h + 1) * dv] = y.numpy()
    return out, ring_t, st


def pin_layer_pair_library(o):
    """Speculative two-position verify ("Module linear_core", gdn_pair):
    position 1 commits (ring and state), position 2 continues from the
    committed result into scratch; checked against the torch composition
    applied twice."""
    c = _layer_case(25)
    r = _rng(26)
    B, C = c["x"].shape
    Hv, dv = c["Hv"], c["dv"]
    x2 = np.stack([c["x"], r.normal(size=(B, C))], axis=1)
    z2 = np.stack([c["z"], r.normal(size=(B, Hv * dv))], axis=1)
    a2 = np.stack([c["a"], r.normal(size=(B, Hv))], axis=1)
    b2 = np.stack([c["b"], r.normal(size=(B, Hv))], axis=1)
    out, ring, st, sring, sst = o.layer_pair(x2, z2, a2, b2, c["ring"], c["w"], c["A_log"],
                                             c["dt_bias"], c["norm_w"], c["state"], Hk=c["Hk"])
    o1, r1, s1 = _torch_layer(c, x2[:, 0], z2[:, 0], a2[:, 0], b2[:, 0], c["ring"], c["state"])
    o2, r2, s2 = _torch_layer(c, x2[:, 1], z2[:, 1], a2[:, 1], b2[:, 1], r1, s1)
    _close(out[:, 0], o1, 1e-11, "pair out 1")
    _close(out[:, 1], o2, 1e-11, "pair out 2")
    assert np.array_equal(ring, r1) and np.array_equal(sring, r2), "pair rings"
    _close(st, s1, 1e-12, "pair committed state")
    _close(sst, s2, 1e-12, "pair scratch state")





def _bf16_exact(x):
    """Round an fp64 array to bf16 values (kept in fp64) with torch."""
    return torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()


def pin_forward_batch_library(o):
    """T positions of the layer with dense projections ("Module linear_core",
    gdn_forward_batch): projections as matmuls, each position through the
    torch-built layer, the tail output rounded to bf16 by torch, then the
    output projection; on non-square heads with Hv = 2 Hk."""
    c = _layer_case(27, B=2)
    r = _rng(28)
    Hk, Hv, dk, dv = c["Hk"], c["Hv"], c["dk"], c["dv"]
    C = c["x"].shape[1]
    B, T, D = 2, 5, 24
    hidden = _bf16_exact(r.normal(size=(B, T, D)))
    Wq = _bf16_exact(r.normal(0, D ** -0.5, (C, D)))
    Wz = _bf16_exact(r.normal(0, D ** -0.5, (Hv * dv, D)))
    Wba = _bf16_exact(r.normal(0, D ** -0.5, (2 * Hv, D)))
    Wo = _bf16_exact(r.normal(0, (Hv * dv) ** -0.5, (D, Hv * dv)))
    out, ring, st = o.forward_batch(hidden, Wq, Wz, Wba, Wo, c["ring"], c["w"], c["A_log"],
                                    c["dt_bias"], c["norm_w"], c["state"], Hk=Hk)
    ring_t, st_t = c["ring"].copy(), c["state"].copy()
    for t in range(T):
        h = hidden[:, t]
        mixed = h @ Wq.T
        z = h @ Wz.T
        ba = h @ Wba.T
        y, ring_t, st_t = _torch_layer(c, mixed, z, ba[:, Hv:], ba[:, :Hv], ring_t, st_t)
        want = _bf16_exact(y) @ Wo.T
        _close(out[:, t], want, 1e-12, f"forward_batch out t{t}")
    assert np.array_equal(ring, ring_t), "forward_batch ring"
    _close(st, st_t, 1e-12, "forward_batch state")


def _lfm2_mixer(W_in, W_out, conv_w):
    """The transformers library's LFM2 short-conv mixer in float64, holding
    the given weights (no biases, the library's default)."""
    from transformers.models.lfm2.configuration_lfm2 import Lfm2Config
    from transformers.models.lfm2.modeling_lfm2 import Lfm2ShortConv
    D, K = conv_w.shape
    m = Lfm2ShortConv(Lfm2Config(hidden_size=D, conv_L_cache=K, conv_bias=False), 0).double()
    with torch.no_grad():
        m.in_proj.weight.copy_(torch.from_numpy(W_in))
        m.out_proj.weight.copy_(torch.from_numpy(W_out))
        m.conv.weight.copy_(torch.from_numpy(conv_w).reshape(D, 1, K))
    return m


def _lfm2_run(W_in, W_out, conv_w, hidden):
    """(out, y) of the library mixer over whole sequences from an empty
    history; y (the gated conv output) is read by running the mixer again
    with an identity output projection."""
    D = conv_w.shape[0]
    with torch.no_grad():
        h = torch.from_numpy(hidden)
        out = _lfm2_mixer(W_in, W_out, conv_w).slow_forward(h).numpy()
        y = _lfm2_mixer(W_in, np.eye(D), conv_w).slow_forward(h).numpy()
    return out, y


def _short_conv_case(seed, B, T, D, K):
    r = _rng(seed)
    return dict(hidden=r.normal(size=(B, T, D)), W_in=r.normal(0, D ** -0.5, (3 * D, D)),
                W_out=r.normal(0, D ** -0.5, (D, D)), conv_w=r.normal(0, 0.5, (D, K)))


def pin_short_conv_library(o):
    """LFM2 short-conv mixer ("Module linear_core", short_conv_forward_batch):
    from an empty ring, the oracle over T1 positions and then, resuming from
    its ring, over T2 more equals the transformers library's LFM2 mixer run
    over all T1 + T2 positions; the ring then holds the last K-1 gated inputs
    (input gate times value, computed here with a matmul); with y rounded to
    bf16 (by torch) the output is W_out y."""
    for K in (3, 4, 2):
        B, T1, T2, D = 2, 4, 3, 12
        c = _short_conv_case(30 + K, B, T1 + T2, D, K)
        want, y = _lfm2_run(c["W_in"], c["W_out"], c["conv_w"], c["hidden"])
        ring0 = np.zeros((B, K - 1, D))
        args = (c["W_in"], c["W_out"])
        out1, ring1 = o.short_conv_forward_batch(c["hidden"][:, :T1], *args, ring0, c["conv_w"],
                                                 round_y=False)
        out2, ring2 = o.short_conv_forward_batch(c["hidden"][:, T1:], *args, ring1, c["conv_w"],
                                                 round_y=False)
        _close(np.concatenate([out1, out2], axis=1), want, 1e-12, f"short_conv out K={K}")
        proj = c["hidden"] @ c["W_in"].T
        gated = proj[..., :D] * proj[..., 2 * D:]
        _close(ring2, gated[:, T1 + T2 - (K - 1):], 1e-12, f"short_conv ring K={K}")
        out_r, _ = o.short_conv_forward_batch(c["hidden"], *args, ring0, c["conv_w"])
        _close(out_r, _bf16_exact(y) @ c["W_out"].T, 1e-12, f"short_conv bf16 y K={K}")


def pin_short_conv_pair_library(o):
    """Speculative two-position verify of the short-conv mixer ("Module
    linear_core", short_conv_pair): after P positions, position P commits its
    ring and position P + 1 continues into scratch; outputs and both rings
    against the library mixer over P + 2 positions and the gated inputs."""
    B, P, D, K = 3, 5, 10, 3
    c = _short_conv_case(34, B, P + 2, D, K)
    want, _ = _lfm2_run(c["W_in"], c["W_out"], c["conv_w"], c["hidden"])
    args = (c["W_in"], c["W_out"])
    _, ring = o.short_conv_forward_batch(c["hidden"][:, :P], *args, np.zeros((B, K - 1, D)),
                                         c["conv_w"], round_y=False)
    out, ring_c, ring_s = o.short_conv_pair(c["hidden"][:, P:], *args, ring, c["conv_w"],
                                            round_y=False)
    _close(out, want[:, P:], 1e-12, "short_conv_pair out")
    proj = c["hidden"] @ c["W_in"].T
    gated = proj[..., :D] * proj[..., 2 * D:]
    _close(ring_c, gated[:, P + 1 - (K - 1):P + 1], 1e-12, "short_conv_pair committed ring")
    _close(ring_s, gated[:, P + 2 - (K - 1):P + 2], 1e-12, "short_conv_pair scratch ring")


def _kda_textbook(M, q, k, v, beta, g, dk):
    """One KDA position on one head in the product form
    M_new = M Diag(exp g) (I - beta k k^T) + beta v k^T, out = M_new q / sqrt(dk)."""
    A = np.diag(np.exp(g)) @ (np.eye(dk) - beta * np.outer(k, k))
    M_new = M @ A + beta * np.outer(v, k)
    return M_new, M_new @ q / math.sqrt(dk)


def pin_kda_textbook(o):
    """KDA ("Module linear_core", kda_forward / kda_forward_batch; the
    published delta rule with a decay per key channel): random non-square
    heads with Hv = 2 Hk, one position and a 5-position sequence, against the
    product form with value head h reading key head h % Hk and its own
    per-channel decay."""
    r = _rng(40)
    L, B, Hk, Hv, dk, dv = 1, 2, 2, 4, 8, 6
    M = r.normal(0, 0.3, (L, B, Hv, dv, dk))
    q = _unit_rows(r.normal(size=(L, B, Hk, dk)))
    k = _unit_rows(r.normal(size=(L, B, Hk, dk)))
    v = r.normal(size=(L, B, Hv, dv))
    beta = r.uniform(0.1, 0.9, (L, B, Hv))
    g = r.uniform(-1.5, 0, (L, B, Hv, dk))
    st, out = o.kda_step(M, q, k, v, beta, g)
    for b in range(B):
        for h in range(Hv):
            Mn, on = _kda_textbook(M[0, b, h], q[0, b, h % Hk], k[0, b, h % Hk], v[0, b, h],
                                   beta[0, b, h], g[0, b, h], dk)
            _close(st[0, b, h], Mn, 1e-13, f"kda step state b{b} h{h}")
            _close(out[0, b, h], on, 1e-13, f"kda step out b{b} h{h}")
    T = 5
    M0 = r.normal(0, 0.3, (B, Hv, dv, dk))
    q = _unit_rows(r.normal(size=(B, T, Hk, dk)))
    k = _unit_rows(r.normal(size=(B, T, Hk, dk)))
    v = r.normal(size=(B, T, Hv, dv))
    beta = r.uniform(0.1, 0.9, (B, T, Hv))
    g = r.uniform(-1.5, 0, (B, T, Hv, dk))
    st, out = o.kda_prefill(M0, q, k, v, beta, g)
    for b in range(B):
        for h in range(Hv):
            Mt = M0[b, h]
            for t in range(T):
                Mt, ot = _kda_textbook(Mt, q[b, t, h % Hk], k[b, t, h % Hk], v[b, t, h],
                                       beta[b, t, h], g[b, t, h], dk)
                _close(out[b, t, h], ot, 1e-12, f"kda prefill out b{b} t{t} h{h}")
            _close(st[b, h], Mt, 1e-12, f"kda prefill state b{b} h{h}")


def pin_kda_channel_marker(o):
    """k = 0 (no write) and a decay on key channel 3 only: column 3 of every
    row shrinks by exp(-30) and every other entry is left exactly as it was;
    the output reads the decayed state."""
    r = _rng(41)
    dk, dv = 8, 5
    M = r.normal(size=(1, 1, 1, dv, dk))
    g = np.zeros((1, 1, 1, dk))
    g[..., 3] = -30.0
    q = _unit_rows(r.normal(size=(1, 1, 1, dk)))
    st, out = o.kda_step(M, q, np.zeros((1, 1, 1, dk)), r.normal(size=(1, 1, 1, dv)),
                         np.full((1, 1, 1), 0.5), g)
    keep = np.ones(dk, bool)
    keep[3] = False
    assert np.array_equal(st[..., keep], M[..., keep]), "kda marker: other channels changed"
    _close(st[..., 3] / M[..., 3], np.full((1, 1, 1, dv), math.exp(-30.0)), 1e-15,
           "kda marker: decayed channel")
    _close(out, st @ q[0, 0, 0] / math.sqrt(dk), 1e-15, "kda marker: out")


def pin_kda_closed_form(o):
    """No decay (g = 0), beta = 1, |k| = 1: the delta rule stores v at k, so
    M_new k = v, and with q = k the output is v / sqrt(dk); with a uniform
    decay the update equals the scalar-gated one (gdn_step)."""
    r = _rng(42)
    dk, dv = 16, 12
    M = r.normal(size=(1, 1, 1, dv, dk))
    k = _unit_rows(r.normal(size=(1, 1, 1, dk)))
    v = r.normal(size=(1, 1, 1, dv))
    st, out = o.kda_step(M, k, k, v, np.ones((1, 1, 1)), np.zeros((1, 1, 1, dk)))
    _close(st[0, 0, 0] @ k[0, 0, 0], v[0, 0, 0], 1e-12, "kda closed form M k")
    _close(out[0, 0, 0], v[0, 0, 0] / math.sqrt(dk), 1e-12, "kda closed form out")
    gate = np.full((1, 1, 1), -0.7)
    q = _unit_rows(r.normal(size=(1, 1, 1, dk)))
    st_k, out_k = o.kda_step(M, q, k, v, np.full((1, 1, 1), 0.3), np.full((1, 1, 1, dk), -0.7))
    st_g, out_g = o.step(M, q, k, v, np.full((1, 1, 1), 0.3), gate)
    _close(st_k, st_g, 1e-14, "kda uniform decay state")
    _close(out_k, out_g, 1e-14, "kda uniform decay out")


ALL_PINS = [
    pin_golden_step_cases,
    pin_delta_rule_closed_form,
    pin_zero_key,
    pin_zero_beta,
    pin_textbook_step,
    pin_broadcast_marker,
    pin_prefill_associative_memory,
    pin_prefill_textbook,
    pin_pair_textbook,
    pin_prestate_library,
    pin_prestate_special_values,
    pin_tail_library,
    pin_layer_library,
    pin_layer_pair_library,
    pin_forward_batch_library,
    pin_kda_textbook,
    pin_kda_channel_marker,
    pin_kda_closed_form,
    pin_short_conv_library,
    pin_short_conv_pair_library,
]
