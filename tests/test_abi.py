"""The C ABI without a GPU: the library loads, exports every symbol that
include/gdn.h declares, and rejects bad arguments on the host before any
CUDA call (these calls never reach a launch)."""
import ctypes
import os
import re
import subprocess

import pytest

from linear_attention_recurrence_04_b200 import build as gdn_build
from linear_attention_recurrence_04_b200 import gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

OK, NULL, SHAPE, UNSUP, ALIGN, OVERFLOW, CUDA, ALIAS = range(8)


@pytest.fixture(scope="module")
def lib():
    gdn_build.build()
    return gdn.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(gdn.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.library_path()], check=True,
                         capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, f"{name} not exported"
        assert hasattr(lib, name)


def test_last_cuda_error_keeps_only_cuda_failures(lib):
    """gdn_last_cuda_error (the scope table's name for the CUDA error text)
    is exported, starts empty and is not touched by argument errors, which
    gdn_last_error reports instead."""
    lib.gdn_last_cuda_error.restype = ctypes.c_char_p
    before = lib.gdn_last_cuda_error()
    assert before == b""
    assert step_call(lib, dk=64) == UNSUP
    assert b"dk=64" in lib.gdn_last_error()
    assert lib.gdn_last_cuda_error() == before


def test_status_strings(lib):
    for code in range(8):
        assert gdn.status_string(code)
    assert gdn.status_string(99) == "unknown status"


# Fake, 16-byte aligned device addresses 4 GiB apart: never dereferenced,
# every call below fails its checks before any launch.
def fake(i):
    return (i + 1) << 32


A16, A16b, A16c = fake(0), fake(1), fake(2)


def step_call(lib, state=A16, q=A16b, k=A16c, v=fake(3), beta=fake(4), gate=fake(5),
              out=fake(6), L=1, B=1, Hk=16, Hv=32, dk=128, dv=128):
    return lib.gdn_step(state, q, k, v, beta, gate, out, L, B, Hk, Hv, dk, dv, None)


def test_step_argument_checks(lib):
    assert step_call(lib, L=-1) == SHAPE
    assert step_call(lib, Hv=24, Hk=16) == SHAPE
    assert step_call(lib, Hk=0) == SHAPE
    assert step_call(lib, dk=64) == UNSUP
    assert step_call(lib, dv=256) == UNSUP
    assert step_call(lib, q=0) == NULL
    assert step_call(lib, out=0) == NULL
    assert step_call(lib, state=A16 + 4) == ALIGN
    assert step_call(lib, beta=fake(4) + 2) == ALIGN
    assert step_call(lib, L=1 << 40, B=1 << 40) == OVERFLOW
    # out inside the state buffer; state overlapping q
    assert step_call(lib, out=A16 + 4096) == ALIAS
    assert step_call(lib, q=A16 + 1024) == ALIAS
    # read-only inputs may share memory
    assert step_call(lib, k=A16b, q=A16b, out=0) == NULL
    assert b"NULL" in lib.gdn_last_error() or lib.gdn_last_error()
    # empty problems succeed without touching the (null) pointers
    assert lib.gdn_step(0, 0, 0, 0, 0, 0, 0, 0, 5, 16, 32, 128, 128, None) == OK
    assert lib.gdn_step(0, 0, 0, 0, 0, 0, 0, 3, 0, 16, 32, 128, 128, None) == OK


def test_prefill_argument_checks(lib):
    f = lambda **kw: lib.gdn_prefill(kw.get("state", A16), A16b, A16c, fake(3), fake(4),
                                     fake(5), kw.get("out", fake(6)), kw.get("B", 1),
                                     kw.get("T", 4), kw.get("Hk", 16), kw.get("Hv", 32),
                                     128, 128, kw.get("status", None), None)
    assert f(T=-1) == SHAPE
    assert f(Hv=17) == SHAPE
    assert f(state=0) == NULL
    assert f(state=A16 + 8) == ALIGN
    assert f(status=fake(8) + 2) == ALIGN
    assert f(out=A16b) == ALIAS
    assert lib.gdn_prefill(0, 0, 0, 0, 0, 0, 0, 2, 0, 16, 32, 128, 128, None, None) == OK
    assert lib.gdn_prefill(0, 0, 0, 0, 0, 0, 0, 0, 9, 16, 32, 128, 128, None, None) == OK


def pair_call(lib, state=A16, scratch=fake(7), q=A16b, k=A16c, v=fake(3), beta=fake(4),
              gate=fake(5), out=fake(6), L=1, B=1, Hk=16, Hv=32, dk=128, dv=128):
    return lib.gdn_pair(state, scratch, q, k, v, beta, gate, out, L, B, Hk, Hv, dk, dv, None)


def test_pair_argument_checks(lib):
    assert pair_call(lib, B=-1) == SHAPE
    assert pair_call(lib, Hv=20, Hk=16) == SHAPE
    assert pair_call(lib, dk=64) == UNSUP
    assert pair_call(lib, scratch=0) == NULL
    assert pair_call(lib, gate=0) == NULL
    assert pair_call(lib, scratch=fake(7) + 8) == ALIGN
    assert pair_call(lib, gate=fake(5) + 2) == ALIGN
    assert pair_call(lib, L=1 << 40, B=1 << 40) == OVERFLOW
    # the scratch state inside the live state, over an input, over out
    assert pair_call(lib, scratch=A16 + 4096) == ALIAS
    assert pair_call(lib, scratch=fake(3) + 1024) == ALIAS
    assert pair_call(lib, scratch=fake(6) + 256) == ALIAS
    # out over the state; the state over q
    assert pair_call(lib, out=A16 + 16) == ALIAS
    assert pair_call(lib, q=A16 + 1024) == ALIAS
    # read-only inputs may share memory
    assert pair_call(lib, k=A16b, q=A16b, out=0) == NULL
    assert lib.gdn_pair(0, 0, 0, 0, 0, 0, 0, 0, 0, 4, 16, 32, 128, 128, None) == OK
    assert lib.gdn_pair(0, 0, 0, 0, 0, 0, 0, 0, 2, 0, 16, 32, 128, 128, None) == OK


def test_layer_argument_checks(lib):
    def f(B=1, Hk=16, Hv=32, K=4, state=A16, out=fake(10), ring=fake(5)):
        return lib.gdn_layer_decode(A16b, A16c, fake(3), fake(4), ring, fake(6), fake(7),
                                    fake(8), fake(9), ctypes.c_float(1e-6), ctypes.c_float(1e-6),
                                    state, out, B, Hk, Hv, 128, 128, K, None)
    assert f(B=-2) == SHAPE
    assert f(K=3) == UNSUP
    assert f(Hk=4, Hv=32) == UNSUP          # 8 value heads per key head: not compiled
    assert f(state=0) == NULL
    assert f(state=A16 + 4) == ALIGN
    assert f(out=A16b + 64) == ALIAS        # inside mixed_qkv
    assert f(ring=A16c + 16) == ALIAS       # conv ring overlapping z
    assert lib.gdn_layer_decode(0, 0, 0, 0, 0, 0, 0, 0, 0, ctypes.c_float(1e-6),
                                ctypes.c_float(1e-6), 0, 0, 0, 16, 32, 128, 128, 4, None) == OK


def test_binding_rejects_cpu_tensors():
    import torch
    st = torch.zeros(1, 1, 32, 128, 128)
    q = torch.zeros(1, 1, 16, 128)
    with pytest.raises(ValueError):
        gdn.step(st, q, q, torch.zeros(1, 1, 32, 128), torch.zeros(1, 1, 32),
                 torch.zeros(1, 1, 32), out=torch.zeros(1, 1, 32, 128))


def test_layer_pair_argument_checks(lib):
    def f(B=1, Hk=16, Hv=32, K=4, state=A16, sring=fake(11), sstate=fake(12), out=fake(10)):
        return lib.gdn_layer_pair(A16b, A16c, fake(3), fake(4), fake(5), fake(6), fake(7),
                                  fake(8), fake(9), ctypes.c_float(1e-6), ctypes.c_float(1e-6),
                                  state, sring, sstate, out, B, Hk, Hv, 128, 128, K, None)
    assert f(B=-1) == SHAPE
    assert f(K=5) == UNSUP
    assert f(sring=0) == NULL
    assert f(sstate=0) == NULL
    assert f(sstate=fake(12) + 8) == ALIGN
    assert f(sstate=A16 + 65536) == ALIAS           # scratch state inside the live state
    assert f(sring=fake(5) + 16) == ALIAS           # scratch ring inside the live ring
    assert f(out=A16b + 32768 + 64) == ALIAS        # out inside mixed_qkv [1][2][8192]
    assert lib.gdn_layer_pair(0, 0, 0, 0, 0, 0, 0, 0, 0, ctypes.c_float(1e-6),
                              ctypes.c_float(1e-6), 0, 0, 0, 0, 0, 16, 32, 128, 128, 4,
                              None) == OK


@pytest.mark.parametrize("name", ["gdn_linear_bf16", "gdn_linear_bf16_split_k"])
def test_linear_argument_checks(lib, name):
    fn = getattr(lib, name)
    f = lambda x=fake(1), w=fake(2), y=fake(3), M=4, N=4, K=16, st=0: fn(
        x, w, y, M, N, K, st, None)
    assert f(K=12) == UNSUP
    assert f(M=-1) == SHAPE
    assert f(x=0) == NULL
    assert f(y=fake(3) + 8) == ALIGN
    assert f(y=fake(1) + 16) == ALIAS
    assert f(M=1 << 30) == OVERFLOW
    assert f(st=fake(4) + 2) == ALIGN
    assert fn(0, 0, 0, 0, 7, 16, 0, None) == OK


def test_forward_batch_argument_checks(lib):
    ws = lib.gdn_forward_batch_workspace_size(2, 3, 16, 32, 128, 128)
    assert ws > 2 * 3 * (8192 + 4096 + 4096) * 4
    assert lib.gdn_forward_batch_workspace_size(2, 3, 16, 32, 64, 128) == 0

    def f(D=64, ws_bytes=ws, workspace=fake(20), K=4, out=fake(13)):
        return lib.gdn_forward_batch(fake(1), fake(2), fake(3), fake(4), fake(5), fake(6),
                                     fake(7), fake(8), fake(9), fake(10), ctypes.c_float(1e-6),
                                     ctypes.c_float(1e-6), fake(12), out, workspace, ws_bytes,
                                     2, 3, D, 16, 32, 128, 128, K, 0, None)
    assert f(D=60) == UNSUP
    assert f(K=2) == UNSUP
    assert f(ws_bytes=ws - 1) == SHAPE
    assert f(workspace=0) == NULL
    assert f(workspace=fake(20) + 16) == ALIGN
    assert f(out=fake(20) + 256) == ALIAS


def test_short_conv_argument_checks(lib):
    ws = lib.gdn_short_conv_workspace_size(2, 3, 64)
    assert ws >= 2 * 3 * 64 * (3 * 4 + 2)
    assert lib.gdn_short_conv_workspace_size(2, 3, 60) == 0
    assert lib.gdn_short_conv_workspace_size(70000, 1, 64) == 0

    def f(D=64, ws_bytes=ws, workspace=fake(20), K=3, out=fake(13), T=3, B=2):
        return lib.gdn_short_conv_forward_batch(fake(1), fake(2), fake(3), fake(4), fake(5), out,
                                                workspace, ws_bytes, B, T, D, K, 0, None)
    assert f(D=60) == UNSUP
    assert f(K=1) == UNSUP and f(K=5) == UNSUP
    assert f(T=-1) == SHAPE
    assert f(B=70000) == OVERFLOW
    assert f(ws_bytes=ws - 1) == SHAPE
    assert f(workspace=0) == NULL
    assert f(workspace=fake(20) + 16) == ALIGN
    assert f(out=fake(20) + 256) == ALIAS
    assert f(out=fake(4)) == ALIAS                      # out over the ring
    # one position and the two-position verify go through the same checks
    ws1 = lib.gdn_short_conv_workspace_size(2, 1, 64)
    assert lib.gdn_short_conv_forward(fake(1), fake(2), fake(3), fake(4), fake(5), fake(13),
                                      fake(20), ws1 - 1, 2, 64, 3, 0, None) == SHAPE
    ws2 = lib.gdn_short_conv_workspace_size(2, 2, 64)
    assert lib.gdn_short_conv_pair(fake(1), fake(2), fake(3), fake(4), 0, fake(5), fake(13),
                                   fake(20), ws2, 2, 64, 3, 0, None) == NULL
    assert lib.gdn_short_conv_pair(fake(1), fake(2), fake(3), fake(4), fake(4), fake(5), fake(13),
                                   fake(20), ws2, 2, 64, 3, 0, None) == ALIAS


def test_kda_argument_checks(lib):
    def step(g=fake(6), L=1, dk=128):
        return lib.gdn_kda_step(fake(1), fake(2), fake(3), fake(4), fake(5), g, fake(7), L, 2, 16,
                                32, dk, 128, None)
    assert step(dk=64) == UNSUP
    assert step(L=-1) == SHAPE
    assert step(g=0) == NULL
    assert step(g=fake(6) + 4) == ALIGN          # g is read 16 bytes at a time
    assert step(g=fake(1) + 16) == ALIAS         # g inside the state (updated in place)

    def pre(g=fake(6), T=3):
        return lib.gdn_kda_prefill(fake(1), fake(2), fake(3), fake(4), fake(5), g, fake(7), 2, T,
                                   16, 32, 128, 128, None)
    assert pre(T=-2) == SHAPE
    assert pre(g=0) == NULL
    assert pre(g=fake(6) + 8) == ALIGN


def test_tile_grid_limits(lib):
    """The conv kernels walk tiles of 32 positions in one grid dimension, so
    T above 65535 * 32 is refused before any launch."""
    T = 65535 * 32 + 1
    assert lib.gdn_forward_batch_workspace_size(1, T, 16, 32, 128, 128) == 0
    assert lib.gdn_short_conv_workspace_size(1, T, 64) == 0
    assert lib.gdn_forward_batch_workspace_size(1, T - 1, 16, 32, 128, 128) > 0
    assert lib.gdn_short_conv_forward_batch(fake(1), fake(2), fake(3), fake(4), fake(5), fake(13),
                                            fake(20), 1 << 40, 1, T, 64, 3, 0, None) == OVERFLOW


def test_selftest_bounded_wait_argument_checks(lib):
    assert lib.gdn_selftest_bounded_wait(0, 1000, 0, None) == NULL
    assert lib.gdn_selftest_bounded_wait(fake(1), 0, 0, None) == UNSUP
    assert lib.gdn_selftest_bounded_wait(fake(1), 2_000_000_001, 0, None) == UNSUP
    assert lib.gdn_selftest_bounded_wait(fake(1) + 2, 1000, 0, None) == ALIGN


def test_selftest_grid_barrier_argument_checks(lib):
    """Refused on the host before any launch: null pointers, sizes, a zero or
    over-wide tag, the limit, misalignment."""
    w, r = fake(1), fake(2)
    assert lib.gdn_selftest_grid_barrier(0, r, 5, 2, 2, 1000, None) == NULL
    assert lib.gdn_selftest_grid_barrier(w, 0, 5, 2, 2, 1000, None) == NULL
    assert lib.gdn_selftest_grid_barrier(w, r, 5, 0, 2, 1000, None) == UNSUP
    assert lib.gdn_selftest_grid_barrier(w, r, 5, 33, 2, 1000, None) == UNSUP
    assert lib.gdn_selftest_grid_barrier(w, r, 5, 2, 0, 1000, None) == UNSUP
    assert lib.gdn_selftest_grid_barrier(w, r, 5, 2, 65, 1000, None) == UNSUP
    assert lib.gdn_selftest_grid_barrier(w, r, 0, 2, 2, 1000, None) == UNSUP
    assert lib.gdn_selftest_grid_barrier(w, r, 1 << 48, 2, 2, 1000, None) == UNSUP
    assert lib.gdn_selftest_grid_barrier(w, r, 5, 2, 2, 0, None) == UNSUP
    assert lib.gdn_selftest_grid_barrier(w, r, 5, 2, 2, 2_000_000_001, None) == UNSUP
    assert lib.gdn_selftest_grid_barrier(w + 4, r, 5, 2, 2, 1000, None) == ALIGN
    assert lib.gdn_selftest_grid_barrier(w, r + 2, 5, 2, 2, 1000, None) == ALIGN
