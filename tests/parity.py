"""Parity checks between the CUDA path and the fp64 oracle.

Tolerance: the GPU computes in fp32 and the oracle in fp64. A GPU value
passes when |gpu - ref| <= 1e-5 everywhere AND |gpu - ref| / |ref| <= 1e-4
wherever |ref| > 1e-3. The absolute bound covers values near zero, where a
relative error is meaningless (the pages note that their large relative
errors all sit near zero).
"""
from __future__ import annotations

import numpy as np

ABS_TOL = 1e-5
REL_TOL = 1e-4
REL_FLOOR = 1e-3


def parity_report(gpu, ref) -> dict:
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"shape {g.shape} vs {r.shape}"
    if g.size == 0:
        return dict(max_abs=0.0, max_rel=0.0, n=0, finite=True)
    err = np.abs(g - r)
    mask = np.abs(r) > REL_FLOOR
    rel = float(np.max(err[mask] / np.abs(r[mask]))) if mask.any() else 0.0
    return dict(max_abs=float(np.max(err)), max_rel=rel, n=int(g.size),
                finite=bool(np.all(np.isfinite(g))))


def assert_parity(gpu, ref, what: str) -> dict:
    rep = parity_report(gpu, ref)
    assert rep["finite"], f"{what}: non-finite GPU values"
    assert rep["max_abs"] <= ABS_TOL, f"{what}: max abs {rep['max_abs']:.3e} > {ABS_TOL}"
    assert rep["max_rel"] <= REL_TOL, f"{what}: max rel {rep['max_rel']:.3e} > {REL_TOL}"
    return rep


def gather_step_units(d: dict, units, Hk: int, Hv: int) -> dict:
    """Per-unit slices of decode inputs as an L=1, B=n, Hk=Hv=1 problem, so the
    oracle can compute sampled (layer, sequence, head) units one by one."""
    L, B = d["state"].shape[:2]
    sel = []
    for u in units:
        lb, h = divmod(int(u), Hv)
        l, b = divmod(lb, B)
        sel.append((l, b, h, h % Hk))
    take = lambda name, key: np.stack([d[name][l, b, key(h, g)] for l, b, h, g in sel])[None, :, None]
    return dict(
        state=take("state", lambda h, g: h), q=take("q", lambda h, g: g),
        k=take("k", lambda h, g: g), v=take("v", lambda h, g: h),
        beta=np.stack([d["beta"][l, b, h] for l, b, h, _ in sel])[None, :, None],
        gate=np.stack([d["gate"][l, b, h] for l, b, h, _ in sel])[None, :, None],
    )
