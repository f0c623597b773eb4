"""ctypes wrapper around ``libgdn_oracle.so`` (built from ``gdn_oracle.c``).

TEST INFRASTRUCTURE. The wrapper only marshals arrays: every input is widened
to a C-contiguous float64 copy (fp32 data widens exactly), every output comes
back as a new float64 array, and the caller's arrays are never modified. All
arithmetic is in the C file; see its header for the passages each function
follows.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_I64 = ctypes.c_int64
_DBL = ctypes.c_double
_PD = ctypes.POINTER(ctypes.c_double)
_PI = ctypes.POINTER(ctypes.c_int64)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64)).copy()


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_PD)


def _units(units: Optional[Sequence[int]]):
    if units is None:
        return None, 0, None
    arr = np.ascontiguousarray(np.asarray(units, dtype=np.int64))
    return arr.ctypes.data_as(_PI), int(arr.size), arr


class OracleError(RuntimeError):
    pass


def _chunks(units: Optional[Sequence[int]], total: int, threads: int):
    """The listed units (all when None) split into `threads` contiguous
    lists for parallel calls; each chunk is written by one call only."""
    arr = np.arange(total, dtype=np.int64) if units is None else \
        np.ascontiguousarray(np.asarray(units, dtype=np.int64))
    return [np.ascontiguousarray(c) for c in np.array_split(arr, max(1, threads)) if c.size]


def _run_split(fn, units, total: int, threads: int, what: str) -> None:
    """Call `fn(units_ptr, n_units)` over disjoint unit lists, from `threads`
    host threads at once (ctypes releases the GIL during each call). The C
    entry points write only the state, outputs and rings of the units they
    are given, so the calls touch disjoint memory."""
    if threads <= 1:
        up, nu, _keep = _units(units)
        _check(fn(up, nu), what)
        return
    from concurrent.futures import ThreadPoolExecutor
    parts = _chunks(units, total, threads)
    with ThreadPoolExecutor(len(parts)) as ex:
        rcs = list(ex.map(lambda c: fn(c.ctypes.data_as(_PI), int(c.size)), parts))
    for rc in rcs:
        _check(rc, what)


def _check(rc: int, what: str) -> None:
    if rc == -1:
        raise OracleError(f"{what}: bad argument")
    if rc == -2:
        raise OracleError(f"{what}: out of memory")
    if rc != 0:
        raise OracleError(f"{what}: status {rc}")


class Oracle:
    """Handle on one build of the oracle library (the default, or a given .so)."""

    def __init__(self, so_path: Optional[str] = None):
        if so_path is None:
            so_path = _build.build()
        self.path = so_path
        lib = ctypes.CDLL(os.path.abspath(so_path))
        lib.oracle_gdn_step.restype = ctypes.c_int
        lib.oracle_gdn_step.argtypes = [_PD, _PD, _PD, _PD, _PD, _PD, _PD,
                                        _I64, _I64, _I64, _I64, _I64, _I64, _PI, _I64]
        lib.oracle_gdn_prefill.restype = ctypes.c_int
        lib.oracle_gdn_prefill.argtypes = [_PD, _PD, _PD, _PD, _PD, _PD, _PD,
                                           _I64, _I64, _I64, _I64, _I64, _I64, _PI, _I64]
        lib.oracle_gdn_pair.restype = ctypes.c_int
        lib.oracle_gdn_pair.argtypes = [_PD] * 8 + [_I64] * 6 + [_PI, _I64]
        lib.oracle_gdn_prestate.restype = ctypes.c_int
        lib.oracle_gdn_prestate.argtypes = [_PD, _PD, _PD, _PD, _PD, _PD, _PD, _DBL,
                                            _PD, _PD, _PD, _PD, _PD,
                                            _I64, _I64, _I64, _I64, _I64, _I64, _PI, _I64]
        lib.oracle_gated_rmsnorm.restype = ctypes.c_int
        lib.oracle_gated_rmsnorm.argtypes = [_PD, _PD, _PD, _DBL, _PD, _I64, _I64]
        lib.oracle_gdn_layer_decode.restype = ctypes.c_int
        lib.oracle_gdn_layer_decode.argtypes = [_PD, _PD, _PD, _PD, _PD, _PD, _PD, _PD, _PD,
                                                _DBL, _DBL, _PD, _PD,
                                                _I64, _I64, _I64, _I64, _I64, _I64, _PI, _I64]
        lib.oracle_gdn_layer_pair.restype = ctypes.c_int
        lib.oracle_gdn_layer_pair.argtypes = [_PD, _PD, _PD, _PD, _PD, _PD, _PD, _PD, _PD,
                                              _DBL, _DBL, _PD, _PD, _PD, _PD,
                                              _I64, _I64, _I64, _I64, _I64, _I64, _PI, _I64]
        lib.oracle_gdn_forward_batch.restype = ctypes.c_int
        lib.oracle_gdn_forward_batch.argtypes = [_PD] * 10 + [_DBL, _DBL, _PD, _PD] + [_I64] * 8 + \
            [ctypes.c_int, _PI, _I64]
        for name in ("oracle_kda_step", "oracle_kda_prefill"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [_PD] * 7 + [_I64] * 6 + [_PI, _I64]
        lib.oracle_short_conv_forward_batch.restype = ctypes.c_int
        lib.oracle_short_conv_forward_batch.argtypes = [_PD] * 6 + [_I64] * 4 + \
            [ctypes.c_int, _PI, _I64]
        lib.oracle_short_conv_pair.restype = ctypes.c_int
        lib.oracle_short_conv_pair.argtypes = [_PD] * 7 + [_I64] * 3 + [ctypes.c_int, _PI, _I64]
        self.lib = lib

    # -- recurrence ---------------------------------------------------------
    def step(self, state, q, k, v, beta, gate, units=None, threads=1):
        """One token for every (layer, sequence, value head) unit.

        Shapes: state [L,B,Hv,dv,dk]; q, k [L,B,Hk,dk]; v [L,B,Hv,dv];
        beta, gate [L,B,Hv]. Returns (new_state, out [L,B,Hv,dv]); units that
        are not listed keep their state and get zero output. `threads` > 1
        splits the units over that many host threads (same results).
        """
        st = _f64(state)
        L, B, Hv, dv, dk = st.shape
        Hk = np.shape(q)[2]
        qq, kk, vv, bb, gg = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(gate)
        assert qq.shape == (L, B, Hk, dk) and kk.shape == qq.shape
        assert vv.shape == (L, B, Hv, dv) and bb.shape == (L, B, Hv) and gg.shape == bb.shape
        out = np.zeros((L, B, Hv, dv), dtype=np.float64)
        fn = lambda up, nu: self.lib.oracle_gdn_step(_ptr(st), _ptr(qq), _ptr(kk), _ptr(vv),
                                                     _ptr(bb), _ptr(gg), _ptr(out),
                                                     L, B, Hk, Hv, dk, dv, up, nu)
        _run_split(fn, units, L * B * Hv, threads, "oracle_gdn_step")
        return st, out

    def prefill(self, state, q, k, v, beta, gate, units=None, threads=1):
        """T positions in order, for every (sequence, value head) unit
        (`threads` > 1: the units split over that many host threads).

        Shapes: state [B,Hv,dv,dk]; q, k [B,T,Hk,dk]; v [B,T,Hv,dv];
        beta, gate [B,T,Hv]. Returns (final_state, out [B,T,Hv,dv]).
        """
        st = _f64(state)
        B, Hv, dv, dk = st.shape
        qq, kk, vv, bb, gg = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(gate)
        T, Hk = qq.shape[1], qq.shape[2]
        assert qq.shape == (B, T, Hk, dk) and kk.shape == qq.shape
        assert vv.shape == (B, T, Hv, dv) and bb.shape == (B, T, Hv) and gg.shape == bb.shape
        out = np.zeros((B, T, Hv, dv), dtype=np.float64)
        fn = lambda up, nu: self.lib.oracle_gdn_prefill(_ptr(st), _ptr(qq), _ptr(kk), _ptr(vv),
                                                        _ptr(bb), _ptr(gg), _ptr(out),
                                                        B, T, Hk, Hv, dk, dv, up, nu)
        _run_split(fn, units, B * Hv, threads, "oracle_gdn_prefill")
        return st, out

    def pair(self, state, q, k, v, beta, gate, units=None):
        """Two positions per unit: position 0 into the state, position 1 from
        there into a scratch state.

        Shapes: state [L,B,Hv,dv,dk]; q, k [L,B,2,Hk,dk]; v [L,B,2,Hv,dv];
        beta, gate [L,B,2,Hv]. Returns (committed_state, scratch_state,
        out [L,B,2,Hv,dv]); units that are not listed keep their state, get a
        zero scratch state and zero output.
        """
        st = _f64(state)
        L, B, Hv, dv, dk = st.shape
        Hk = np.shape(q)[3]
        qq, kk, vv, bb, gg = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(gate)
        assert qq.shape == (L, B, 2, Hk, dk) and kk.shape == qq.shape
        assert vv.shape == (L, B, 2, Hv, dv) and bb.shape == (L, B, 2, Hv)
        assert gg.shape == bb.shape
        scratch = np.zeros_like(st)
        out = np.zeros((L, B, 2, Hv, dv), dtype=np.float64)
        up, nu, _keep = _units(units)
        rc = self.lib.oracle_gdn_pair(_ptr(st), _ptr(scratch), _ptr(qq), _ptr(kk), _ptr(vv),
                                      _ptr(bb), _ptr(gg), _ptr(out), L, B, Hk, Hv, dk, dv, up, nu)
        _check(rc, "oracle_gdn_pair")
        return st, scratch, out

    # -- layer pieces -------------------------------------------------------
    def prestate(self, mixed_qkv, ring, conv_w, a, b, A_log, dt_bias, *, Hk, Hv, dk, dv,
                 l2_eps=1e-6, seqs=None):
        """Conv + ring shift, SiLU, split, L2 norm, beta and gate.

        Shapes: mixed_qkv [B,C]; ring [B,K-1,C]; conv_w [C,K]; a, b [B,Hv];
        A_log, dt_bias [Hv]. Returns dict(q [B,Hk,dk], k, v [B,Hv,dv],
        beta [B,Hv], gate [B,Hv], ring [B,K-1,C]).
        """
        x, rg, w = _f64(mixed_qkv), _f64(ring), _f64(conv_w)
        B, C = x.shape
        K = w.shape[1]
        assert C == 2 * Hk * dk + Hv * dv and rg.shape == (B, K - 1, C) and w.shape == (C, K)
        aa, bb, al, dt = _f64(a), _f64(b), _f64(A_log), _f64(dt_bias)
        q = np.zeros((B, Hk, dk)); k = np.zeros((B, Hk, dk)); v = np.zeros((B, Hv, dv))
        beta = np.zeros((B, Hv)); gate = np.zeros((B, Hv))
        sp, ns, _keep = _units(seqs)
        rc = self.lib.oracle_gdn_prestate(_ptr(x), _ptr(rg), _ptr(w), _ptr(aa), _ptr(bb),
                                          _ptr(al), _ptr(dt), float(l2_eps), _ptr(q), _ptr(k),
                                          _ptr(v), _ptr(beta), _ptr(gate),
                                          B, Hk, Hv, dk, dv, K, sp, ns)
        _check(rc, "oracle_gdn_prestate")
        return dict(q=q, k=k, v=v, beta=beta, gate=gate, ring=rg)

    def gated_rmsnorm(self, o, z, w, eps=1e-6):
        """Tail over the last axis: o, z [..., dv]; w [dv]."""
        oo, zz, ww = _f64(o), _f64(z), _f64(w)
        dv = oo.shape[-1]
        assert zz.shape == oo.shape and ww.shape == (dv,)
        y = np.zeros_like(oo)
        rc = self.lib.oracle_gated_rmsnorm(_ptr(oo), _ptr(zz), _ptr(ww), float(eps), _ptr(y),
                                           oo.size // dv, dv)
        _check(rc, "oracle_gated_rmsnorm")
        return y

    def layer_decode(self, mixed_qkv, z, a, b, ring, conv_w, A_log, dt_bias, norm_w, state,
                     *, Hk, l2_eps=1e-6, norm_eps=1e-6, seqs=None, threads=1):
        """Prestate -> recurrence -> gated RMSNorm tail, one token per sequence.

        Shapes: mixed_qkv [B,C]; z [B,Hv*dv]; a, b [B,Hv]; ring [B,K-1,C];
        conv_w [C,K]; A_log, dt_bias [Hv]; norm_w [dv]; state [B,Hv,dv,dk].
        Returns (out [B,Hv*dv], new_ring, new_state).
        """
        st = _f64(state)
        B, Hv, dv, dk = st.shape
        x, zz, aa, bb = _f64(mixed_qkv), _f64(z), _f64(a), _f64(b)
        rg, w, al, dt, nw = _f64(ring), _f64(conv_w), _f64(A_log), _f64(dt_bias), _f64(norm_w)
        C, K = w.shape
        assert x.shape == (B, C) and C == 2 * Hk * dk + Hv * dv
        assert zz.shape == (B, Hv * dv) and rg.shape == (B, K - 1, C) and nw.shape == (dv,)
        out = np.zeros((B, Hv * dv))
        fn = lambda sp, ns: self.lib.oracle_gdn_layer_decode(
            _ptr(x), _ptr(zz), _ptr(aa), _ptr(bb), _ptr(rg), _ptr(w), _ptr(al), _ptr(dt),
            _ptr(nw), float(l2_eps), float(norm_eps), _ptr(st), _ptr(out),
            B, Hk, Hv, dk, dv, K, sp, ns)
        _run_split(fn, seqs, B, threads, "oracle_gdn_layer_decode")
        return out, rg, st


    def layer_pair(self, mixed_qkv, z, a, b, ring, conv_w, A_log, dt_bias, norm_w, state, *,
                   Hk, l2_eps=1e-6, norm_eps=1e-6, seqs=None, threads=1):
        """Two positions per sequence: position 1 commits, position 2 is tentative.

        Shapes: mixed_qkv [B,2,C]; z [B,2,Hv*dv]; a, b [B,2,Hv]; ring [B,K-1,C];
        conv_w [C,K]; A_log, dt_bias [Hv]; norm_w [dv]; state [B,Hv,dv,dk].
        Returns (out [B,2,Hv*dv], ring, state, scratch_ring, scratch_state):
        ring/state after position 1, scratch_* after position 2.
        """
        st = _f64(state)
        B, Hv, dv, dk = st.shape
        x, zz, aa, bb = _f64(mixed_qkv), _f64(z), _f64(a), _f64(b)
        rg, w, al, dt, nw = _f64(ring), _f64(conv_w), _f64(A_log), _f64(dt_bias), _f64(norm_w)
        C, K = w.shape
        assert x.shape == (B, 2, C) and C == 2 * Hk * dk + Hv * dv
        assert zz.shape == (B, 2, Hv * dv) and aa.shape == (B, 2, Hv) and bb.shape == aa.shape
        assert rg.shape == (B, K - 1, C) and nw.shape == (dv,)
        out = np.zeros((B, 2, Hv * dv))
        srg = np.zeros_like(rg)
        sst = np.zeros_like(st)
        fn = lambda sp, ns: self.lib.oracle_gdn_layer_pair(
            _ptr(x), _ptr(zz), _ptr(aa), _ptr(bb), _ptr(rg), _ptr(w), _ptr(al), _ptr(dt),
            _ptr(nw), float(l2_eps), float(norm_eps), _ptr(st), _ptr(srg), _ptr(sst),
            _ptr(out), B, Hk, Hv, dk, dv, K, sp, ns)
        _run_split(fn, seqs, B, threads, "oracle_gdn_layer_pair")
        return out, rg, st, srg, sst


    def forward_batch(self, hidden, W_qkv, W_z, W_ba, W_out, ring, conv_w, A_log, dt_bias,
                      norm_w, state, *, Hk, l2_eps=1e-6, norm_eps=1e-6, round_y=True,
                      seqs=None):
        """T positions of the layer with dense projections.

        Shapes: hidden [B,T,D]; W_qkv [C,D]; W_z [Hv*dv,D]; W_ba [2*Hv,D];
        W_out [D,Hv*dv]; ring [B,K-1,C]; conv_w [C,K]; A_log, dt_bias [Hv];
        norm_w [dv]; state [B,Hv,dv,dk]. Returns (out [B,T,D], ring, state).
        """
        st = _f64(state)
        B, Hv, dv, dk = st.shape
        hh = _f64(hidden)
        T, D = hh.shape[1], hh.shape[2]
        wq, wz, wb, wo = _f64(W_qkv), _f64(W_z), _f64(W_ba), _f64(W_out)
        rg, w, al, dt, nw = _f64(ring), _f64(conv_w), _f64(A_log), _f64(dt_bias), _f64(norm_w)
        C, K = w.shape
        assert hh.shape == (B, T, D) and wq.shape == (C, D) and wz.shape == (Hv * dv, D)
        assert wb.shape == (2 * Hv, D) and wo.shape == (D, Hv * dv) and rg.shape == (B, K - 1, C)
        out = np.zeros((B, T, D))
        sp, ns, _keep = _units(seqs)
        rc = self.lib.oracle_gdn_forward_batch(_ptr(hh), _ptr(wq), _ptr(wz), _ptr(wb), _ptr(wo),
                                               _ptr(rg), _ptr(w), _ptr(al), _ptr(dt), _ptr(nw),
                                               float(l2_eps), float(norm_eps),
                                               _ptr(st), _ptr(out), B, T, D, Hk, Hv, dk, dv, K,
                                               int(bool(round_y)), sp, ns)
        _check(rc, "oracle_gdn_forward_batch")
        return out, rg, st


    # -- KDA core ---------------------------------------------------------------
    def kda_step(self, state, q, k, v, beta, g, units=None):
        """One KDA token per (layer, sequence, value head) unit.

        Shapes: state [L,B,Hv,dv,dk]; q, k [L,B,Hk,dk]; v [L,B,Hv,dv];
        beta [L,B,Hv]; g [L,B,Hv,dk] (log-decay per key channel).
        Returns (new_state, out [L,B,Hv,dv]).
        """
        st = _f64(state)
        L, B, Hv, dv, dk = st.shape
        Hk = np.shape(q)[2]
        qq, kk, vv, bb, gg = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(g)
        assert qq.shape == (L, B, Hk, dk) and kk.shape == qq.shape
        assert vv.shape == (L, B, Hv, dv) and bb.shape == (L, B, Hv)
        assert gg.shape == (L, B, Hv, dk)
        out = np.zeros((L, B, Hv, dv), dtype=np.float64)
        up, nu, _keep = _units(units)
        rc = self.lib.oracle_kda_step(_ptr(st), _ptr(qq), _ptr(kk), _ptr(vv), _ptr(bb),
                                      _ptr(gg), _ptr(out), L, B, Hk, Hv, dk, dv, up, nu)
        _check(rc, "oracle_kda_step")
        return st, out

    def kda_prefill(self, state, q, k, v, beta, g, units=None, threads=1):
        """T KDA positions in order. Shapes: state [B,Hv,dv,dk]; q, k
        [B,T,Hk,dk]; v [B,T,Hv,dv]; beta [B,T,Hv]; g [B,T,Hv,dk].
        Returns (final_state, out [B,T,Hv,dv])."""
        st = _f64(state)
        B, Hv, dv, dk = st.shape
        T, Hk = np.shape(q)[1], np.shape(q)[2]
        qq, kk, vv, bb, gg = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(g)
        assert qq.shape == (B, T, Hk, dk) and kk.shape == qq.shape
        assert vv.shape == (B, T, Hv, dv) and bb.shape == (B, T, Hv)
        assert gg.shape == (B, T, Hv, dk)
        out = np.zeros((B, T, Hv, dv), dtype=np.float64)
        fn = lambda up, nu: self.lib.oracle_kda_prefill(_ptr(st), _ptr(qq), _ptr(kk), _ptr(vv),
                                                        _ptr(bb), _ptr(gg), _ptr(out),
                                                        B, T, Hk, Hv, dk, dv, up, nu)
        _run_split(fn, units, B * Hv, threads, "oracle_kda_prefill")
        return st, out

    # -- LFM2 short-convolution mixer ----------------------------------------
    def short_conv_forward_batch(self, hidden, W_in, W_out, ring, conv_w, *, round_y=True,
                                 seqs=None):
        """T positions of the short-conv mixer.

        Shapes: hidden [B,T,D]; W_in [3D,D] (rows: input gate | output gate |
        value); W_out [D,D]; ring [B,K-1,D] (gated inputs, oldest first);
        conv_w [D,K]. Returns (out [B,T,D], ring).
        """
        hh = _f64(hidden)
        B, T, D = hh.shape
        wi, wo, rg, w = _f64(W_in), _f64(W_out), _f64(ring), _f64(conv_w)
        K = w.shape[1]
        assert wi.shape == (3 * D, D) and wo.shape == (D, D) and w.shape == (D, K)
        assert rg.shape == (B, K - 1, D)
        out = np.zeros((B, T, D))
        sp, ns, _keep = _units(seqs)
        rc = self.lib.oracle_short_conv_forward_batch(_ptr(hh), _ptr(wi), _ptr(wo), _ptr(rg),
                                                      _ptr(w), _ptr(out), B, T, D, K,
                                                      int(bool(round_y)), sp, ns)
        _check(rc, "oracle_short_conv_forward_batch")
        return out, rg

    def short_conv_pair(self, hidden, W_in, W_out, ring, conv_w, *, round_y=True, seqs=None):
        """Two positions per sequence: position 0 commits, position 1 is tentative.

        Shapes: hidden [B,2,D]; the rest as short_conv_forward_batch.
        Returns (out [B,2,D], ring after position 0, scratch_ring after
        position 1).
        """
        hh = _f64(hidden)
        B, two, D = hh.shape
        assert two == 2
        wi, wo, rg, w = _f64(W_in), _f64(W_out), _f64(ring), _f64(conv_w)
        K = w.shape[1]
        assert wi.shape == (3 * D, D) and wo.shape == (D, D) and rg.shape == (B, K - 1, D)
        out = np.zeros((B, 2, D))
        srg = np.zeros_like(rg)
        sp, ns, _keep = _units(seqs)
        rc = self.lib.oracle_short_conv_pair(_ptr(hh), _ptr(wi), _ptr(wo), _ptr(rg), _ptr(srg),
                                             _ptr(w), _ptr(out), B, D, K, int(bool(round_y)),
                                             sp, ns)
        _check(rc, "oracle_short_conv_pair")
        return out, rg, srg


_DEFAULT: Optional[Oracle] = None


def load() -> Oracle:
    """The oracle built from this directory's source (built on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT


class OracleF32:
    """The literal fp32 instantiation of the recurrence (``gdn_oracle_f32.c``):
    decode and prefill with every value in float. Only the benchmark's CPU
    baseline times it; parity is judged against the double oracle above."""

    def __init__(self, so_path: Optional[str] = None):
        if so_path is None:
            so_path = _build.build_f32()
        self.path = so_path
        lib = ctypes.CDLL(os.path.abspath(so_path))
        pf = ctypes.POINTER(ctypes.c_float)
        for name in ("oracle_gdn_step_f32", "oracle_gdn_prefill_f32"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [pf] * 7 + [_I64] * 6 + [_PI, _I64]
        self.lib = lib
        self._pf = pf

    def ptr(self, a: np.ndarray):
        assert a.dtype == np.float32 and a.flags.c_contiguous
        return a.ctypes.data_as(self._pf)

    def step(self, state, q, k, v, beta, gate, units=None):
        """As Oracle.step, in float32 (returns float32 arrays)."""
        f = lambda a: np.ascontiguousarray(np.asarray(a, dtype=np.float32)).copy()
        st, qq, kk, vv, bb, gg = f(state), f(q), f(k), f(v), f(beta), f(gate)
        L, B, Hv, dv, dk = st.shape
        Hk = qq.shape[2]
        out = np.zeros((L, B, Hv, dv), dtype=np.float32)
        up, nu, _keep = _units(units)
        rc = self.lib.oracle_gdn_step_f32(self.ptr(st), self.ptr(qq), self.ptr(kk), self.ptr(vv),
                                          self.ptr(bb), self.ptr(gg), self.ptr(out),
                                          L, B, Hk, Hv, dk, dv, up, nu)
        _check(rc, "oracle_gdn_step_f32")
        return st, out

    def prefill(self, state, q, k, v, beta, gate, units=None):
        """As Oracle.prefill, in float32 (returns float32 arrays)."""
        f = lambda a: np.ascontiguousarray(np.asarray(a, dtype=np.float32)).copy()
        st, qq, kk, vv, bb, gg = f(state), f(q), f(k), f(v), f(beta), f(gate)
        B, Hv, dv, dk = st.shape
        T, Hk = qq.shape[1], qq.shape[2]
        out = np.zeros((B, T, Hv, dv), dtype=np.float32)
        up, nu, _keep = _units(units)
        rc = self.lib.oracle_gdn_prefill_f32(self.ptr(st), self.ptr(qq), self.ptr(kk),
                                             self.ptr(vv), self.ptr(bb), self.ptr(gg),
                                             self.ptr(out), B, T, Hk, Hv, dk, dv, up, nu)
        _check(rc, "oracle_gdn_prefill_f32")
        return st, out


_DEFAULT_F32: Optional[OracleF32] = None


def load_f32() -> OracleF32:
    """The fp32 instantiation built from this directory's source."""
    global _DEFAULT_F32
    if _DEFAULT_F32 is None:
        _DEFAULT_F32 = OracleF32()
    return _DEFAULT_F32
