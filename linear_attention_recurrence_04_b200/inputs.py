"""Seeded synthetic inputs for the Gated DeltaNet workloads.

This module only draws numbers. It holds none of the recurrence's or the
layer's arithmetic, imports nothing from the CUDA binding or the oracle, and
is the one piece both sides share: the same arrays go to the GPU path and to
the CPU oracle.

Recipe (numpy PCG64, every draw in float64, cast to float32 at the end):
  decode (one token per (layer, sequence)):
    state ~ N(0, 0.05^2) in the transposed layout [.., Hv, dv, dk]
    q, k  ~ N(0, 1) per key head, scaled to unit L2 norm (input recipe)
    v     ~ N(0, 1)
    beta  = 1 / (1 + exp(-N(0, 1)))  (a sigmoid-distributed value in (0, 1))
    gate  ~ U(gate_low, 0)           (log-decay; -1 for decode, -0.5 prefill)
    layers use independent child streams spawned from the seed.
  prefill: the same per-position draws, zero initial state, gate ~ U(-0.5, 0).
  layer decode (raw activations before the prestate):
    mixed_qkv, z, a, b, conv ring ~ N(0, 1); conv weight ~ N(0, 0.25^2);
    A_log ~ U(-1, 1); dt_bias ~ N(0, 0.1^2); norm weight ~ 1 + N(0, 0.1^2);
    state ~ N(0, 0.05^2).
The geometry defaults follow the pages' layer: Hk = 16 key heads, Hv = 32
value heads, dk = dv = 128, conv kernel 4 over 2*16*128 + 32*128 = 8192
channels ("Red Lite dev15c", "Audited Qwen3-Next recurrent geometry";
"Red Lite dev15e", "M4 field result").
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict

import numpy as np

HK, HV, DK, DV, KCONV = 16, 32, 128, 128, 4


def _unit_rows(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _squash(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def _f32(x: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


def decode_inputs(L: int, B: int, *, Hk: int = HK, Hv: int = HV, dk: int = DK, dv: int = DV,
                  seed: int = 1000, state_std: float = 0.05,
                  gate_low: float = -1.0) -> Dict[str, np.ndarray]:
    """Inputs of one batched decode token: state [L,B,Hv,dv,dk], q/k [L,B,Hk,dk],
    v [L,B,Hv,dv], beta/gate [L,B,Hv] (float32)."""
    streams = np.random.default_rng(seed).spawn(max(L, 1))
    parts = {n: [] for n in ("state", "q", "k", "v", "beta", "gate")}
    for l in range(L):
        r = streams[l]
        parts["state"].append(_f32(r.normal(0.0, state_std, (B, Hv, dv, dk))))
        parts["q"].append(_f32(_unit_rows(r.normal(size=(B, Hk, dk)))))
        parts["k"].append(_f32(_unit_rows(r.normal(size=(B, Hk, dk)))))
        parts["v"].append(_f32(r.normal(size=(B, Hv, dv))))
        parts["beta"].append(_f32(_squash(r.normal(size=(B, Hv)))))
        parts["gate"].append(_f32(r.uniform(gate_low, 0.0, (B, Hv))))
    shapes = dict(state=(0, B, Hv, dv, dk), q=(0, B, Hk, dk), k=(0, B, Hk, dk),
                  v=(0, B, Hv, dv), beta=(0, B, Hv), gate=(0, B, Hv))
    return {n: (np.stack(p) if p else np.zeros(shapes[n], np.float32)) for n, p in parts.items()}


def pair_inputs(L: int, B: int, *, Hk: int = HK, Hv: int = HV, dk: int = DK, dv: int = DV,
                seed: int = 1015, state_std: float = 0.05,
                gate_low: float = -1.0) -> Dict[str, np.ndarray]:
    """Inputs of the two-position verify: the decode draws of decode_inputs
    with a position axis of 2 after the sequence axis: state [L,B,Hv,dv,dk],
    q/k [L,B,2,Hk,dk], v [L,B,2,Hv,dv], beta/gate [L,B,2,Hv] (float32)."""
    streams = np.random.default_rng(seed).spawn(max(L, 1))
    parts = {n: [] for n in ("state", "q", "k", "v", "beta", "gate")}
    for l in range(L):
        r = streams[l]
        parts["state"].append(_f32(r.normal(0.0, state_std, (B, Hv, dv, dk))))
        parts["q"].append(_f32(_unit_rows(r.normal(size=(B, 2, Hk, dk)))))
        parts["k"].append(_f32(_unit_rows(r.normal(size=(B, 2, Hk, dk)))))
        parts["v"].append(_f32(r.normal(size=(B, 2, Hv, dv))))
        parts["beta"].append(_f32(_squash(r.normal(size=(B, 2, Hv)))))
        parts["gate"].append(_f32(r.uniform(gate_low, 0.0, (B, 2, Hv))))
    shapes = dict(state=(0, B, Hv, dv, dk), q=(0, B, 2, Hk, dk), k=(0, B, 2, Hk, dk),
                  v=(0, B, 2, Hv, dv), beta=(0, B, 2, Hv), gate=(0, B, 2, Hv))
    return {n: (np.stack(p) if p else np.zeros(shapes[n], np.float32)) for n, p in parts.items()}


def prefill_inputs(B: int, T: int, *, Hk: int = HK, Hv: int = HV, dk: int = DK, dv: int = DV,
                   seed: int = 1003, gate_low: float = -0.5,
                   state_std: float = 0.0) -> Dict[str, np.ndarray]:
    """Inputs of a T-position prefill: state [B,Hv,dv,dk] (zero unless
    state_std > 0), q/k [B,T,Hk,dk], v [B,T,Hv,dv], beta/gate [B,T,Hv]."""
    r = np.random.default_rng(seed)
    if state_std > 0:
        state = _f32(r.normal(0.0, state_std, (B, Hv, dv, dk)))
    else:
        state = np.zeros((B, Hv, dv, dk), np.float32)
    return dict(
        state=state,
        q=_f32(_unit_rows(r.normal(size=(B, T, Hk, dk)))),
        k=_f32(_unit_rows(r.normal(size=(B, T, Hk, dk)))),
        v=_f32(r.normal(size=(B, T, Hv, dv))),
        beta=_f32(_squash(r.normal(size=(B, T, Hv)))),
        gate=_f32(r.uniform(gate_low, 0.0, (B, T, Hv))),
    )


def layer_inputs(B: int, *, Hk: int = HK, Hv: int = HV, dk: int = DK, dv: int = DV,
                 K: int = KCONV, seed: int = 1004,
                 state_std: float = 0.05) -> Dict[str, np.ndarray]:
    """Raw activations and parameters of one fused layer-decode token."""
    r = np.random.default_rng(seed)
    C = 2 * Hk * dk + Hv * dv
    return dict(
        mixed_qkv=_f32(r.normal(size=(B, C))),
        z=_f32(r.normal(size=(B, Hv * dv))),
        a=_f32(r.normal(size=(B, Hv))),
        b=_f32(r.normal(size=(B, Hv))),
        conv_ring=_f32(r.normal(size=(B, K - 1, C))),
        conv_w=_f32(r.normal(0.0, 0.25, (C, K))),
        A_log=_f32(r.uniform(-1.0, 1.0, Hv)),
        dt_bias=_f32(r.normal(0.0, 0.1, Hv)),
        norm_w=_f32(1.0 + r.normal(0.0, 0.1, dv)),
        state=_f32(r.normal(0.0, state_std, (B, Hv, dv, dk))),
    )


def kda_decode_inputs(L: int, B: int, *, seed: int = 1013, g_low: float = -1.0,
                      **kw) -> Dict[str, np.ndarray]:
    """decode_inputs plus a log-decay per key channel g ~ U(g_low, 0)
    [L, B, Hv, dk] (the KDA core's gate; the scalar gate is dropped)."""
    d = decode_inputs(L, B, seed=seed, **kw)
    r = np.random.default_rng([seed, 1])
    L_, B_, Hv = d["beta"].shape
    dk = d["q"].shape[-1]
    d["g"] = _f32(r.uniform(g_low, 0.0, (L_, B_, Hv, dk)))
    del d["gate"]
    return d


def kda_prefill_inputs(B: int, T: int, *, seed: int = 1014, g_low: float = -0.5,
                       **kw) -> Dict[str, np.ndarray]:
    """prefill_inputs plus g ~ U(g_low, 0) [B, T, Hv, dk] per key channel."""
    d = prefill_inputs(B, T, seed=seed, **kw)
    r = np.random.default_rng([seed, 1])
    B_, T_, Hv = d["beta"].shape
    dk = d["q"].shape[-1]
    d["g"] = _f32(r.uniform(g_low, 0.0, (B_, T_, Hv, dk)))
    del d["gate"]
    return d


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """float32 array of the nearest bfloat16 values (round half to even), a
    dtype conversion so the GPU (as bf16) and the oracle (as fp64) read the
    same numbers."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def forward_inputs(B: int, T: int, *, D: int = 2048, Hk: int = HK, Hv: int = HV, dk: int = DK,
                   dv: int = DV, K: int = KCONV, seed: int = 1007,
                   state_std: float = 0.0) -> Dict[str, np.ndarray]:
    """A layer over T positions with dense projections: hidden ~ N(0, 1),
    weights ~ N(0, 1/fan_in) (all bf16-representable float32), conv ring
    ~ N(0, 1), conv weight ~ N(0, 0.25^2), A_log ~ U(-1, 1),
    dt_bias ~ N(0, 0.1^2), norm weight ~ 1 + N(0, 0.1^2), state zero (or
    N(0, state_std^2))."""
    r = np.random.default_rng(seed)
    C = 2 * Hk * dk + Hv * dv
    HD = Hv * dv
    bf = lambda a: to_bf16_values(a.astype(np.float32))
    return dict(
        hidden=bf(r.normal(size=(B, T, D))),
        w_qkv=bf(r.normal(0.0, D ** -0.5, (C, D))),
        w_z=bf(r.normal(0.0, D ** -0.5, (HD, D))),
        w_ba=bf(r.normal(0.0, D ** -0.5, (2 * Hv, D))),
        w_out=bf(r.normal(0.0, HD ** -0.5, (D, HD))),
        conv_ring=_f32(r.normal(size=(B, K - 1, C))),
        conv_w=_f32(r.normal(0.0, 0.25, (C, K))),
        A_log=_f32(r.uniform(-1.0, 1.0, Hv)),
        dt_bias=_f32(r.normal(0.0, 0.1, Hv)),
        norm_w=_f32(1.0 + r.normal(0.0, 0.1, dv)),
        state=(_f32(r.normal(0.0, state_std, (B, Hv, dv, dk))) if state_std > 0
               else np.zeros((B, Hv, dv, dk), np.float32)),
    )


def short_conv_inputs(B: int, T: int, *, D: int = 2048, K: int = 3, seed: int = 1008,
                      ring_std: float = 1.0) -> Dict[str, np.ndarray]:
    """The LFM2 short-conv mixer over T positions: hidden ~ N(0, 1),
    w_in ~ N(0, 1/D) [3D, D], w_out ~ N(0, 1/D) [D, D] (all bf16-representable
    float32), conv ring of gated inputs ~ N(0, ring_std^2) [B, K-1, D], conv
    weight ~ N(0, 0.25^2) [D, K]."""
    r = np.random.default_rng(seed)
    bf = lambda a: to_bf16_values(a.astype(np.float32))
    return dict(
        hidden=bf(r.normal(size=(B, T, D))),
        w_in=bf(r.normal(0.0, D ** -0.5, (3 * D, D))),
        w_out=bf(r.normal(0.0, D ** -0.5, (D, D))),
        conv_ring=_f32(r.normal(0.0, ring_std, (B, K - 1, D))),
        conv_w=_f32(r.normal(0.0, 0.25, (D, K))),
    )


@dataclass(frozen=True)
class Workload:
    """One named synthetic workload and how to draw it."""
    name: str
    kind: str                     # "step" | "pair" | "prefill" | "layer" | "forward" | "short_conv" | "kda_*"
    sizes: Dict[str, int] = field(default_factory=dict)
    seed: int = 1000

    def draw(self) -> Dict[str, np.ndarray]:
        if self.kind == "step":
            return decode_inputs(self.sizes["L"], self.sizes["B"], seed=self.seed)
        if self.kind == "pair":
            return pair_inputs(self.sizes["L"], self.sizes["B"], seed=self.seed)
        if self.kind == "prefill":
            return prefill_inputs(self.sizes["B"], self.sizes["T"], seed=self.seed)
        if self.kind == "layer":
            return layer_inputs(self.sizes["B"], seed=self.seed)
        if self.kind == "forward":
            return forward_inputs(self.sizes["B"], self.sizes["T"], seed=self.seed)
        if self.kind == "kda_step":
            return kda_decode_inputs(self.sizes["L"], self.sizes["B"], seed=self.seed)
        if self.kind == "kda_prefill":
            return kda_prefill_inputs(self.sizes["B"], self.sizes["T"], seed=self.seed)
        if self.kind == "short_conv":
            return short_conv_inputs(self.sizes["B"], self.sizes["T"], D=self.sizes["D"],
                                     K=self.sizes["K"], seed=self.seed)
        raise ValueError(self.kind)


# The five workloads: single-sequence decode, batched decode, 36-layer decode,
# sequential prefill, fused layer decode.
WORKLOADS = {
    "decode_l1_b1": Workload("decode_l1_b1", "step", dict(L=1, B=1), seed=1000),
    "decode_l1_b64": Workload("decode_l1_b64", "step", dict(L=1, B=64), seed=1001),
    "decode_l36_b16": Workload("decode_l36_b16", "step", dict(L=36, B=16), seed=1002),
    "prefill_b4_t4096": Workload("prefill_b4_t4096", "prefill", dict(B=4, T=4096), seed=1003),
    "layer_decode_b256": Workload("layer_decode_b256", "layer", dict(B=256), seed=1004),
}

# The two-position speculative verify of the bare recurrence for 64 sequences.
PAIR_WORKLOAD = Workload("pair_l1_b64", "pair", dict(L=1, B=64), seed=1015)

# The batched layer forward with dense projections (D = 2048 hidden).
FORWARD_WORKLOAD = Workload("forward_batch_b4_t4096", "forward", dict(B=4, T=4096), seed=1007)

# The KDA core at the recurrent layer's geometry: one decode token for 64
# sequences, and 4 x 4096 positions from a zero state.
KDA_WORKLOADS = {
    "kda_decode_b64": Workload("kda_decode_b64", "kda_step", dict(L=1, B=64), seed=1013),
    "kda_prefill_b4_t4096": Workload("kda_prefill_b4_t4096", "kda_prefill", dict(B=4, T=4096),
                                     seed=1014),
}

# The LFM2 short-conv mixer at the same hidden size: one decode position for 64
# sequences, the two-position verify for 64 sequences, and 4 x 4096 positions.
SHORT_CONV_WORKLOADS = {
    "short_conv_decode_b64": Workload("short_conv_decode_b64", "short_conv",
                                      dict(B=64, T=1, D=2048, K=3), seed=1008),
    "short_conv_pair_b64": Workload("short_conv_pair_b64", "short_conv",
                                    dict(B=64, T=2, D=2048, K=3), seed=1012),
    "short_conv_batch_b4_t4096": Workload("short_conv_batch_b4_t4096", "short_conv",
                                          dict(B=4, T=4096, D=2048, K=3), seed=1009),
}
