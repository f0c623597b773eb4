"""ctypes binding of ``libgdn.so`` (C ABI in ``include/gdn.h``).

Argument marshalling only: each function checks that the torch tensors are
float32, contiguous and on one CUDA device, passes their device pointers and
the current stream to the C entry point of the same name, and raises
``GdnError`` on a non-zero status. Every step of the computation runs in the
library's CUDA kernels. There is no CPU path: if the library is missing the
first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libgdn.so"

_VP = ctypes.c_void_p
_I64 = ctypes.c_int64
_F32 = ctypes.c_float

STATUS = {
    0: "GDN_OK", 1: "GDN_ERR_NULL", 2: "GDN_ERR_SHAPE", 3: "GDN_ERR_UNSUPPORTED",
    4: "GDN_ERR_ALIGN", 5: "GDN_ERR_OVERFLOW", 6: "GDN_ERR_CUDA", 7: "GDN_ERR_ALIAS",
}

# Every symbol that include/gdn.h declares.
EXPORTS = ("gdn_status_string", "gdn_last_error", "gdn_last_cuda_error", "gdn_step", "gdn_prefill", "gdn_pair",
           "gdn_layer_decode",
           "gdn_layer_pair", "gdn_linear_bf16", "gdn_linear_bf16_split_k",
           "gdn_forward_batch_workspace_size",
           "gdn_forward_batch", "gdn_forward_batch_noalloc", "gdn_short_conv_workspace_size",
           "gdn_short_conv_forward_batch", "gdn_short_conv_forward", "gdn_short_conv_pair",
           "gdn_kda_step", "gdn_kda_prefill", "gdn_selftest_bounded_wait",
           "gdn_selftest_grid_barrier")


class GdnError(RuntimeError):
    """A non-zero gdn_status from the library."""

    def __init__(self, func: str, status: int, detail: str):
        self.status = status
        self.code = STATUS.get(status, str(status))
        super().__init__(f"{func}: {self.code}: {detail}")


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return os.environ.get("GDN_LIBRARY", os.path.join(_PKG, _LIB_NAME))


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (once) and return the library; raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or library_path()
    if not os.path.exists(p):
        raise FileNotFoundError(
            f"{p} is missing: build it with `python -m linear_attention_recurrence_04_b200.build`"
            " (there is no CPU fallback)")
    lib = ctypes.CDLL(p)
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_status_string.argtypes = [ctypes.c_int]
    lib.gdn_last_error.restype = ctypes.c_char_p
    lib.gdn_last_error.argtypes = []
    lib.gdn_last_cuda_error.restype = ctypes.c_char_p
    lib.gdn_last_cuda_error.argtypes = []
    lib.gdn_step.restype = ctypes.c_int
    lib.gdn_step.argtypes = [_VP] * 7 + [_I64] * 6 + [_VP]
    lib.gdn_prefill.restype = ctypes.c_int
    lib.gdn_prefill.argtypes = [_VP] * 7 + [_I64] * 6 + [_VP, _VP]
    lib.gdn_pair.restype = ctypes.c_int
    lib.gdn_pair.argtypes = [_VP] * 8 + [_I64] * 6 + [_VP]
    lib.gdn_layer_decode.restype = ctypes.c_int
    lib.gdn_layer_decode.argtypes = [_VP] * 9 + [_F32, _F32] + [_VP, _VP] + [_I64] * 6 + [_VP]
    lib.gdn_layer_pair.restype = ctypes.c_int
    lib.gdn_layer_pair.argtypes = [_VP] * 9 + [_F32, _F32] + [_VP] * 4 + [_I64] * 6 + [_VP]
    lib.gdn_linear_bf16.restype = ctypes.c_int
    lib.gdn_linear_bf16.argtypes = [_VP, _VP, _VP, _I64, _I64, _I64, _VP, _VP]
    lib.gdn_linear_bf16_split_k.restype = ctypes.c_int
    lib.gdn_linear_bf16_split_k.argtypes = [_VP, _VP, _VP, _I64, _I64, _I64, _VP, _VP]
    lib.gdn_forward_batch_workspace_size.restype = ctypes.c_size_t
    lib.gdn_forward_batch_workspace_size.argtypes = [_I64] * 6
    lib.gdn_forward_batch.restype = ctypes.c_int
    lib.gdn_forward_batch.argtypes = ([_VP] * 10 + [_F32, _F32] + [_VP, _VP, _VP, ctypes.c_size_t]
                                      + [_I64] * 8 + [_VP, _VP])
    lib.gdn_forward_batch_noalloc.restype = ctypes.c_int
    lib.gdn_forward_batch_noalloc.argtypes = ([_VP] * 10 + [_F32, _F32] + [_VP, _VP]
                                              + [_I64] * 8 + [_VP, _VP])
    for name in ("gdn_kda_step", "gdn_kda_prefill"):
        getattr(lib, name).restype = ctypes.c_int
        getattr(lib, name).argtypes = [_VP] * 7 + [_I64] * 6 + [_VP]
    lib.gdn_selftest_bounded_wait.restype = ctypes.c_int
    lib.gdn_selftest_bounded_wait.argtypes = [_VP, ctypes.c_uint64, ctypes.c_int, _VP]
    lib.gdn_selftest_grid_barrier.restype = ctypes.c_int
    lib.gdn_selftest_grid_barrier.argtypes = [_VP, _VP, ctypes.c_uint64, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_uint64, _VP]
    lib.gdn_short_conv_workspace_size.restype = ctypes.c_size_t
    lib.gdn_short_conv_workspace_size.argtypes = [_I64] * 3
    lib.gdn_short_conv_forward_batch.restype = ctypes.c_int
    lib.gdn_short_conv_forward_batch.argtypes = ([_VP] * 7 + [ctypes.c_size_t] + [_I64] * 4
                                                 + [_VP, _VP])
    lib.gdn_short_conv_forward.restype = ctypes.c_int
    lib.gdn_short_conv_forward.argtypes = [_VP] * 7 + [ctypes.c_size_t] + [_I64] * 3 + [_VP, _VP]
    lib.gdn_short_conv_pair.restype = ctypes.c_int
    lib.gdn_short_conv_pair.argtypes = [_VP] * 8 + [ctypes.c_size_t] + [_I64] * 3 + [_VP, _VP]
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().gdn_status_string(int(status)).decode()


def _raise_on(func: str, status: int) -> None:
    if status != 0:
        lib = load_library()
        raise GdnError(func, status, lib.gdn_last_error().decode())


def _dev(tensors: Sequence[torch.Tensor], names: Sequence[str]) -> torch.device:
    device = tensors[0].device
    for t, n in zip(tensors, names):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{n} must be a torch.Tensor")
        if t.dtype is not torch.float32:
            raise TypeError(f"{n} must be float32, got {t.dtype}")
        if not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
        if t.device != device:
            raise ValueError(f"{n} is on {t.device}, expected {device}")
    return device


def _call(device: torch.device, fn, *args) -> int:
    """Call `fn` with `device` current (switching only when it is not)."""
    if torch.cuda.current_device() == device.index:
        return fn(*args)
    with torch.cuda.device(device):
        return fn(*args)


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr() if t.numel() else 0


def _stream(device: torch.device, stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def step(state, q, k, v, beta, gate, out=None, *, stream=None):
    """One decode token: state [L,B,Hv,128,128] (updated in place), q/k
    [L,B,Hk,128], v [L,B,Hv,128], beta/gate [L,B,Hv]. Returns out [L,B,Hv,128]."""
    if state.dim() != 5:
        raise ValueError("state must be [L, B, Hv, dv, dk]")
    L, B, Hv, dv, dk = state.shape
    Hk = q.shape[2]
    if out is None:
        out = torch.empty((L, B, Hv, dv), dtype=torch.float32, device=state.device)
    names = ("state", "q", "k", "v", "beta", "gate", "out")
    tensors = (state, q, k, v, beta, gate, out)
    device = _dev(tensors, names)
    expect = dict(q=(L, B, Hk, dk), k=(L, B, Hk, dk), v=(L, B, Hv, dv), beta=(L, B, Hv),
                  gate=(L, B, Hv), out=(L, B, Hv, dv))
    for n, t in zip(names[1:], tensors[1:]):
        if tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    st = _call(device, load_library().gdn_step, *(_ptr(t) for t in tensors), L, B, Hk, Hv, dk,
               dv, _stream(device, stream))
    _raise_on("gdn_step", st)
    return out


def pair(state, scratch_state, q, k, v, beta, gate, out=None, *, stream=None):
    """Two-position verify: state [L,B,Hv,128,128] (before position 0 ->
    after position 0, in place), scratch_state [L,B,Hv,128,128] (written:
    after position 1), q/k [L,B,2,Hk,128], v [L,B,2,Hv,128], beta/gate
    [L,B,2,Hv]. Returns out [L,B,2,Hv,128]."""
    if state.dim() != 5:
        raise ValueError("state must be [L, B, Hv, dv, dk]")
    L, B, Hv, dv, dk = state.shape
    Hk = q.shape[3]
    if out is None:
        out = torch.empty((L, B, 2, Hv, dv), dtype=torch.float32, device=state.device)
    names = ("state", "scratch_state", "q", "k", "v", "beta", "gate", "out")
    tensors = (state, scratch_state, q, k, v, beta, gate, out)
    device = _dev(tensors, names)
    expect = dict(scratch_state=(L, B, Hv, dv, dk), q=(L, B, 2, Hk, dk), k=(L, B, 2, Hk, dk),
                  v=(L, B, 2, Hv, dv), beta=(L, B, 2, Hv), gate=(L, B, 2, Hv),
                  out=(L, B, 2, Hv, dv))
    for n, t in zip(names[1:], tensors[1:]):
        if tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    st = _call(device, load_library().gdn_pair, *(_ptr(t) for t in tensors), L, B, Hk, Hv, dk,
               dv, _stream(device, stream))
    _raise_on("gdn_pair", st)
    return out


def prefill(state, q, k, v, beta, gate, out=None, *, status=None, stream=None):
    """T positions in order: state [B,Hv,128,128] (initial -> final, in place),
    q/k [B,T,Hk,128], v [B,T,Hv,128], beta/gate [B,T,Hv]. Returns out [B,T,Hv,128].
    `status`, if given, is a zero-initialised one-element int32 CUDA tensor that
    receives timeout bits (non-zero only if a bounded wait ever gave up)."""
    if state.dim() != 4:
        raise ValueError("state must be [B, Hv, dv, dk]")
    B, Hv, dv, dk = state.shape
    T, Hk = q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty((B, T, Hv, dv), dtype=torch.float32, device=state.device)
    names = ("state", "q", "k", "v", "beta", "gate", "out")
    tensors = (state, q, k, v, beta, gate, out)
    device = _dev(tensors, names)
    expect = dict(q=(B, T, Hk, dk), k=(B, T, Hk, dk), v=(B, T, Hv, dv), beta=(B, T, Hv),
                  gate=(B, T, Hv), out=(B, T, Hv, dv))
    for n, t in zip(names[1:], tensors[1:]):
        if tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    sp = None
    if status is not None:
        if status.dtype is not torch.int32 or status.device != device or status.numel() != 1:
            raise TypeError("status must be a one-element int32 tensor on the same device")
        sp = status.data_ptr()
    st = _call(device, load_library().gdn_prefill, *(_ptr(t) for t in tensors), B, T, Hk, Hv,
               dk, dv, sp, _stream(device, stream))
    _raise_on("gdn_prefill", st)
    return out


def layer_decode(mixed_qkv, z, a, b, conv_ring, conv_w, A_log, dt_bias, norm_w, state,
                 out=None, *, Hk: int, l2_eps: float = 1e-6, norm_eps: float = 1e-6,
                 stream=None):
    """Fused prestate + recurrence + gated RMSNorm for one token per sequence.

    mixed_qkv [B,C]; z [B,Hv*128]; a, b [B,Hv]; conv_ring [B,K-1,C] (in place);
    conv_w [C,K]; A_log, dt_bias [Hv]; norm_w [128]; state [B,Hv,128,128]
    (in place). Returns out [B,Hv*128]."""
    if state.dim() != 4:
        raise ValueError("state must be [B, Hv, dv, dk]")
    B, Hv, dv, dk = state.shape
    C, K = conv_w.shape
    if out is None:
        out = torch.empty((B, Hv * dv), dtype=torch.float32, device=state.device)
    names = ("mixed_qkv", "z", "a", "b", "conv_ring", "conv_w", "A_log", "dt_bias", "norm_w",
             "state", "out")
    tensors = (mixed_qkv, z, a, b, conv_ring, conv_w, A_log, dt_bias, norm_w, state, out)
    device = _dev(tensors, names)
    expect = dict(mixed_qkv=(B, C), z=(B, Hv * dv), a=(B, Hv), b=(B, Hv),
                  conv_ring=(B, K - 1, C), A_log=(Hv,), dt_bias=(Hv,), norm_w=(dv,),
                  out=(B, Hv * dv))
    for n, t in zip(names, tensors):
        if n in expect and tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    ptrs = [_ptr(t) for t in tensors]
    st = _call(device, load_library().gdn_layer_decode, *ptrs[:9], float(l2_eps),
               float(norm_eps), ptrs[9], ptrs[10], B, Hk, Hv, dk, dv, K, _stream(device, stream))
    _raise_on("gdn_layer_decode", st)
    return out


def layer_pair(mixed_qkv, z, a, b, conv_ring, conv_w, A_log, dt_bias, norm_w, state,
               scratch_ring=None, scratch_state=None, out=None, *, Hk: int, l2_eps: float = 1e-6,
               norm_eps: float = 1e-6, stream=None):
    """Two positions per sequence for speculative verification.

    Position 0 commits into conv_ring and state (in place); position 1's ring
    and state go to scratch_ring and scratch_state. Activations are
    [B, 2, ...]. Returns (out [B, 2, Hv*128], scratch_ring, scratch_state).
    """
    if state.dim() != 4:
        raise ValueError("state must be [B, Hv, dv, dk]")
    B, Hv, dv, dk = state.shape
    C, K = conv_w.shape
    if scratch_ring is None:
        scratch_ring = torch.empty_like(conv_ring)
    if scratch_state is None:
        scratch_state = torch.empty_like(state)
    if out is None:
        out = torch.empty((B, 2, Hv * dv), dtype=torch.float32, device=state.device)
    names = ("mixed_qkv", "z", "a", "b", "conv_ring", "conv_w", "A_log", "dt_bias", "norm_w",
             "state", "scratch_ring", "scratch_state", "out")
    tensors = (mixed_qkv, z, a, b, conv_ring, conv_w, A_log, dt_bias, norm_w, state,
               scratch_ring, scratch_state, out)
    device = _dev(tensors, names)
    expect = dict(mixed_qkv=(B, 2, C), z=(B, 2, Hv * dv), a=(B, 2, Hv), b=(B, 2, Hv),
                  conv_ring=(B, K - 1, C), A_log=(Hv,), dt_bias=(Hv,), norm_w=(dv,),
                  scratch_ring=(B, K - 1, C), scratch_state=(B, Hv, dv, dk), out=(B, 2, Hv * dv))
    for n, t in zip(names, tensors):
        if n in expect and tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    ptrs = [_ptr(t) for t in tensors]
    st = _call(device, load_library().gdn_layer_pair, *ptrs[:9], float(l2_eps), float(norm_eps),
               *ptrs[9:13], B, Hk, Hv, dk, dv, K, _stream(device, stream))
    _raise_on("gdn_layer_pair", st)
    return out, scratch_ring, scratch_state


def linear_bf16(x, w, y=None, *, status=None, stream=None, split_k=False):
    """y = x @ w.T on the tensor cores: x [M, K] bf16, w [N, K] bf16, y [M, N]
    fp32. `status`, if given, is a zero-initialised int32 CUDA tensor that
    receives timeout bits (see include/gdn.h). split_k=True calls
    gdn_linear_bf16_split_k (K split over a thread-block cluster when
    M <= 128)."""
    if x.dim() != 2 or w.dim() != 2 or x.shape[1] != w.shape[1]:
        raise ValueError("x must be [M, K] and w [N, K]")
    M, K = x.shape
    N = w.shape[0]
    for n, t in (("x", x), ("w", w)):
        if t.dtype is not torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous bfloat16 CUDA tensor")
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    device = _dev((y,), ("y",))
    if x.device != device or w.device != device:
        raise ValueError("x, w and y must be on one device")
    if tuple(y.shape) != (M, N):
        raise ValueError(f"y has shape {tuple(y.shape)}, expected {(M, N)}")
    sp = 0
    if status is not None:
        if status.dtype is not torch.int32 or status.device != device or status.numel() != 1:
            raise TypeError("status must be a one-element int32 tensor on the same device")
        sp = status.data_ptr()
    name = "gdn_linear_bf16_split_k" if split_k else "gdn_linear_bf16"
    st = _call(device, getattr(load_library(), name), _ptr(x), _ptr(w), _ptr(y), M, N, K, sp,
               _stream(device, stream))
    _raise_on(name, st)
    return y


def forward_batch_workspace_size(B: int, T: int, Hk: int = 16, Hv: int = 32) -> int:
    return int(load_library().gdn_forward_batch_workspace_size(B, T, Hk, Hv, 128, 128))


def forward_batch(hidden, w_qkv, w_z, w_ba, w_out, conv_ring, conv_w, A_log, dt_bias, norm_w,
                  state, out=None, workspace=None, *, Hk: int, l2_eps: float = 1e-6,
                  norm_eps: float = 1e-6, status=None, stream=None):
    """The layer over T positions with dense bf16 projections.

    hidden [B, T, D] bf16; w_qkv [C, D], w_z [Hv*128, D], w_ba [2*Hv, D],
    w_out [D, Hv*128] bf16; conv_ring [B, K-1, C] and state [B, Hv, 128, 128]
    are updated in place. `workspace` (uint8 CUDA tensor) is allocated here
    if not given. Returns out [B, T, D] fp32."""
    B, T, D = hidden.shape
    Hv = state.shape[1]
    C, K = conv_w.shape
    for n, t in (("hidden", hidden), ("w_qkv", w_qkv), ("w_z", w_z), ("w_ba", w_ba),
                 ("w_out", w_out)):
        if t.dtype is not torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous bfloat16 CUDA tensor")
    if out is None:
        out = torch.empty((B, T, D), dtype=torch.float32, device=hidden.device)
    names = ("conv_ring", "conv_w", "A_log", "dt_bias", "norm_w", "state", "out")
    tensors = (conv_ring, conv_w, A_log, dt_bias, norm_w, state, out)
    device = _dev(tensors, names)
    need = forward_batch_workspace_size(B, T, Hk, Hv)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    if workspace.dtype is not torch.uint8 or workspace.device != device:
        raise TypeError("workspace must be a uint8 tensor on the same device")
    expect = dict(w_qkv=(C, D), w_z=(Hv * 128, D), w_ba=(2 * Hv, D), w_out=(D, Hv * 128),
                  conv_ring=(B, K - 1, C), out=(B, T, D))
    for n, t in (("w_qkv", w_qkv), ("w_z", w_z), ("w_ba", w_ba), ("w_out", w_out),
                 ("conv_ring", conv_ring), ("out", out)):
        if tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    sp = status.data_ptr() if status is not None else 0
    st = _call(device, load_library().gdn_forward_batch, _ptr(hidden), _ptr(w_qkv), _ptr(w_z),
               _ptr(w_ba), _ptr(w_out), _ptr(conv_ring), _ptr(conv_w), _ptr(A_log),
               _ptr(dt_bias), _ptr(norm_w), float(l2_eps), float(norm_eps), _ptr(state),
               _ptr(out), workspace.data_ptr(), workspace.numel(), B, T, D, Hk, Hv, 128, 128, K,
               sp, _stream(device, stream))
    _raise_on("gdn_forward_batch", st)
    return out


def forward_batch_noalloc(hidden, w_qkv, w_z, w_ba, w_out, conv_ring, conv_w, A_log, dt_bias,
                          norm_w, state, out, *, Hk: int, l2_eps: float = 1e-6,
                          norm_eps: float = 1e-6, status=None, stream=None):
    """forward_batch with the library's built-in scratch instead of a
    workspace (see gdn_forward_batch_noalloc in include/gdn.h): for callers
    that cannot allocate device memory. `out` must be given; nothing is
    allocated here."""
    B, T, D = hidden.shape
    Hv = state.shape[1]
    C, K = conv_w.shape
    for n, t in (("hidden", hidden), ("w_qkv", w_qkv), ("w_z", w_z), ("w_ba", w_ba),
                 ("w_out", w_out)):
        if t.dtype is not torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous bfloat16 CUDA tensor")
    names = ("conv_ring", "conv_w", "A_log", "dt_bias", "norm_w", "state", "out")
    tensors = (conv_ring, conv_w, A_log, dt_bias, norm_w, state, out)
    device = _dev(tensors, names)
    if tuple(out.shape) != (B, T, D):
        raise ValueError(f"out has shape {tuple(out.shape)}, expected {(B, T, D)}")
    sp = status.data_ptr() if status is not None else 0
    st = _call(device, load_library().gdn_forward_batch_noalloc, _ptr(hidden), _ptr(w_qkv),
               _ptr(w_z), _ptr(w_ba), _ptr(w_out), _ptr(conv_ring), _ptr(conv_w), _ptr(A_log),
               _ptr(dt_bias), _ptr(norm_w), float(l2_eps), float(norm_eps), _ptr(state),
               _ptr(out), B, T, D, Hk, Hv, 128, 128, K, sp, _stream(device, stream))
    _raise_on("gdn_forward_batch_noalloc", st)
    return out


# -- KDA core ----------------------------------------------------------------

def kda_step(state, q, k, v, beta, g, out=None, *, stream=None):
    """One KDA decode token: state [L,B,Hv,128,128] (updated in place), q/k
    [L,B,Hk,128], v [L,B,Hv,128], beta [L,B,Hv], g [L,B,Hv,128] (log-decay per
    key channel). Returns out [L,B,Hv,128]."""
    if state.dim() != 5:
        raise ValueError("state must be [L, B, Hv, dv, dk]")
    L, B, Hv, dv, dk = state.shape
    Hk = q.shape[2]
    if out is None:
        out = torch.empty((L, B, Hv, dv), dtype=torch.float32, device=state.device)
    names = ("state", "q", "k", "v", "beta", "g", "out")
    tensors = (state, q, k, v, beta, g, out)
    device = _dev(tensors, names)
    expect = dict(q=(L, B, Hk, dk), k=(L, B, Hk, dk), v=(L, B, Hv, dv), beta=(L, B, Hv),
                  g=(L, B, Hv, dk), out=(L, B, Hv, dv))
    for n, t in zip(names[1:], tensors[1:]):
        if tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    st = _call(device, load_library().gdn_kda_step, *(_ptr(t) for t in tensors), L, B, Hk, Hv,
               dk, dv, _stream(device, stream))
    _raise_on("gdn_kda_step", st)
    return out


def kda_prefill(state, q, k, v, beta, g, out=None, *, stream=None):
    """T KDA positions in order: state [B,Hv,128,128] (initial -> final, in
    place), q/k [B,T,Hk,128], v [B,T,Hv,128], beta [B,T,Hv], g [B,T,Hv,128].
    Returns out [B,T,Hv,128]."""
    if state.dim() != 4:
        raise ValueError("state must be [B, Hv, dv, dk]")
    B, Hv, dv, dk = state.shape
    T, Hk = q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty((B, T, Hv, dv), dtype=torch.float32, device=state.device)
    names = ("state", "q", "k", "v", "beta", "g", "out")
    tensors = (state, q, k, v, beta, g, out)
    device = _dev(tensors, names)
    expect = dict(q=(B, T, Hk, dk), k=(B, T, Hk, dk), v=(B, T, Hv, dv), beta=(B, T, Hv),
                  g=(B, T, Hv, dk), out=(B, T, Hv, dv))
    for n, t in zip(names[1:], tensors[1:]):
        if tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    st = _call(device, load_library().gdn_kda_prefill, *(_ptr(t) for t in tensors), B, T, Hk,
               Hv, dk, dv, _stream(device, stream))
    _raise_on("gdn_kda_prefill", st)
    return out


# -- LFM2 short-convolution mixer ------------------------------------------

def short_conv_workspace_size(B: int, T: int, D: int) -> int:
    return int(load_library().gdn_short_conv_workspace_size(B, T, D))


def _short_conv_args(hidden, w_in, w_out, conv_ring, conv_w, out, workspace, T, npos_out):
    """Checks shared by the short-conv calls; returns (device, B, D, K, out, workspace)."""
    B, D = hidden.shape[0], hidden.shape[-1]
    K = conv_w.shape[1]
    for n, t in (("hidden", hidden), ("w_in", w_in), ("w_out", w_out)):
        if t.dtype is not torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous bfloat16 CUDA tensor")
    if out is None:
        out = torch.empty(npos_out, dtype=torch.float32, device=hidden.device)
    device = _dev((conv_ring, conv_w, out), ("conv_ring", "conv_w", "out"))
    if hidden.device != device or w_in.device != device or w_out.device != device:
        raise ValueError("all tensors must be on one device")
    expect = dict(w_in=(3 * D, D), w_out=(D, D), conv_ring=(B, K - 1, D), conv_w=(D, K),
                  out=tuple(npos_out))
    for n, t in (("w_in", w_in), ("w_out", w_out), ("conv_ring", conv_ring), ("conv_w", conv_w),
                 ("out", out)):
        if tuple(t.shape) != expect[n]:
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {expect[n]}")
    need = short_conv_workspace_size(B, T, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    if workspace.dtype is not torch.uint8 or workspace.device != device:
        raise TypeError("workspace must be a uint8 tensor on the same device")
    return device, B, D, K, out, workspace


def short_conv_forward_batch(hidden, w_in, w_out, conv_ring, conv_w, out=None, workspace=None,
                             *, status=None, stream=None):
    """T positions of the short-conv mixer: hidden [B, T, D] bf16, w_in
    [3D, D] and w_out [D, D] bf16, conv_ring [B, K-1, D] (updated in place),
    conv_w [D, K]. Returns out [B, T, D] fp32."""
    B, T, D = hidden.shape
    device, B, D, K, out, workspace = _short_conv_args(hidden, w_in, w_out, conv_ring, conv_w,
                                                       out, workspace, T, (B, T, D))
    sp = status.data_ptr() if status is not None else 0
    st = _call(device, load_library().gdn_short_conv_forward_batch, _ptr(hidden), _ptr(w_in),
               _ptr(w_out), _ptr(conv_ring), _ptr(conv_w), _ptr(out), workspace.data_ptr(),
               workspace.numel(), B, T, D, K, sp, _stream(device, stream))
    _raise_on("gdn_short_conv_forward_batch", st)
    return out


def short_conv_forward(hidden, w_in, w_out, conv_ring, conv_w, out=None, workspace=None, *,
                       status=None, stream=None):
    """One position per sequence: hidden [B, D] bf16. Returns out [B, D] fp32."""
    B, D = hidden.shape
    device, B, D, K, out, workspace = _short_conv_args(hidden, w_in, w_out, conv_ring, conv_w,
                                                       out, workspace, 1, (B, D))
    sp = status.data_ptr() if status is not None else 0
    st = _call(device, load_library().gdn_short_conv_forward, _ptr(hidden), _ptr(w_in),
               _ptr(w_out), _ptr(conv_ring), _ptr(conv_w), _ptr(out), workspace.data_ptr(),
               workspace.numel(), B, D, K, sp, _stream(device, stream))
    _raise_on("gdn_short_conv_forward", st)
    return out


def short_conv_pair(hidden, w_in, w_out, conv_ring, scratch_ring, conv_w, out=None,
                    workspace=None, *, status=None, stream=None):
    """Two-position verify: hidden [B, 2, D] bf16; conv_ring receives the ring
    after position 0, scratch_ring [B, K-1, D] the ring after position 1.
    Returns out [B, 2, D] fp32."""
    B, two, D = hidden.shape
    if two != 2:
        raise ValueError("hidden must be [B, 2, D]")
    device, B, D, K, out, workspace = _short_conv_args(hidden, w_in, w_out, conv_ring, conv_w,
                                                       out, workspace, 2, (B, 2, D))
    _dev((scratch_ring,), ("scratch_ring",))
    if tuple(scratch_ring.shape) != tuple(conv_ring.shape) or scratch_ring.device != device:
        raise ValueError("scratch_ring must match conv_ring in shape and device")
    sp = status.data_ptr() if status is not None else 0
    st = _call(device, load_library().gdn_short_conv_pair, _ptr(hidden), _ptr(w_in),
               _ptr(w_out), _ptr(conv_ring), _ptr(scratch_ring), _ptr(conv_w), _ptr(out),
               workspace.data_ptr(), workspace.numel(), B, D, K, sp, _stream(device, stream))
    _raise_on("gdn_short_conv_pair", st)
    return out


# -- failure detection -------------------------------------------------------

def selftest_bounded_wait(limit_ns: int, arrive: bool = False, *, device=None, stream=None):
    """Run the library's bounded mbarrier wait on a barrier that nothing
    arrives at (or, with arrive=True, one that completes at once). Returns
    (timed_out, microseconds_waited) after synchronising the stream."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    result = torch.zeros(2, dtype=torch.int32, device=device)
    st = _call(device, load_library().gdn_selftest_bounded_wait, result.data_ptr(), int(limit_ns),
               1 if arrive else 0, _stream(device, stream))
    _raise_on("gdn_selftest_bounded_wait", st)
    torch.cuda.synchronize(device)
    r = result.cpu().tolist()
    return bool(r[0]), int(r[1]) & 0xFFFFFFFF


def selftest_grid_barrier(word, tag: int, ctas: int, expect: int, limit_ns: int, *,
                          stream=None):
    """Run the one-kernel mixer's grid-wide barrier in `ctas` CTAs on `word`
    (a CUDA int64 tensor of one element) expecting `expect` arrivals. Returns
    (status bits per CTA, microseconds waited per CTA) after synchronising."""
    if word.dtype is not torch.int64 or not word.is_cuda or word.numel() != 1:
        raise TypeError("word must be a one-element int64 CUDA tensor")
    device = word.device
    result = torch.zeros(2 * ctas, dtype=torch.int32, device=device)
    st = _call(device, load_library().gdn_selftest_grid_barrier, word.data_ptr(),
               result.data_ptr(), int(tag), int(ctas), int(expect), int(limit_ns),
               _stream(device, stream))
    _raise_on("gdn_selftest_grid_barrier", st)
    torch.cuda.synchronize(device)
    r = result.cpu().tolist()
    return [x & 0xFFFFFFFF for x in r[:ctas]], [x & 0xFFFFFFFF for x in r[ctas:]]
