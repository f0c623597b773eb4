"""gdn_linear_bf16 (tcgen05 + TMA projection GEMM) against an fp64 matmul of
the same bf16 values, through the C ABI."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_04_b200 import gdn

pytestmark = pytest.mark.gpu


def bf16_pair(M, N, K, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K, generator=g) * scale).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    return x, w


def check(x, w, y):
    xd = x.to(torch.float64).numpy()
    wd = w.to(torch.float64).numpy()
    ref = xd @ wd.T
    mag = np.abs(xd) @ np.abs(wd).T                 # sum of |products| per element
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    # fp32 accumulation of exact bf16 x bf16 products: a few units of fp32
    # rounding relative to the sum of magnitudes
    bound = 4e-7 * np.sqrt(x.shape[1]) * mag + 1e-30
    worst = float(np.max(err / bound)) if err.size else 0.0
    assert worst <= 1.0, f"error {worst:.2f} x bound (max abs {err.max():.3e})"
    return float(err.max())


@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (200, 300, 136), (1, 8, 8), (129, 257, 64),
                                   (256, 4096 + 64, 2048), (513, 2048, 4096)])
def test_linear_parity(M, N, K):
    x, w = bf16_pair(M, N, K, seed=M + N + K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = gdn.linear_bf16(x.cuda(), w.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check(x, w, y)


def test_linear_wide_tiles_ragged():
    """A product large enough for 256 x 256 tiles (at least one per SM) with M,
    N and K all off the tile grid: every element checked."""
    M, N, K = 3000, 3100, 200
    x, w = bf16_pair(M, N, K, seed=11)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = gdn.linear_bf16(x.cuda(), w.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check(x, w, y)


def test_linear_rows_independent_of_batch():
    """A row's result does not depend on the other rows of the call or on the
    tile shape chosen for it: rows of a 4096-row product (256 x 256 tiles)
    equal the same rows computed alone (narrow tiles), bit for bit."""
    M, N, K = 4096, 4096, 1024
    x, w = bf16_pair(M, N, K, seed=13)
    xc, wc = x.cuda(), w.cuda()
    y = gdn.linear_bf16(xc, wc)
    rows = [0, 255, 256, 4095]
    for r in rows:
        yr = gdn.linear_bf16(xc[r:r + 1].contiguous(), wc)
        torch.cuda.synchronize()
        assert torch.equal(yr[0], y[r]), f"row {r}"


def test_linear_large_sampled():
    """A projection-sized product (4096 x 8192 x 2048): sampled rows checked."""
    M, N, K = 4096, 8192, 2048
    x, w = bf16_pair(M, N, K, seed=7)
    y = gdn.linear_bf16(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    rows = torch.tensor([0, 1, 127, 128, 2049, 4095])
    check(x[rows], w, y[rows.cuda()])


def test_linear_k_zero_and_empty():
    x = torch.zeros(3, 0, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(5, 0, dtype=torch.bfloat16, device="cuda")
    y = torch.full((3, 5), 7.0, device="cuda")
    gdn.linear_bf16(x, w, y)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0
    e = gdn.linear_bf16(torch.zeros(0, 16, dtype=torch.bfloat16, device="cuda"),
                        torch.zeros(4, 16, dtype=torch.bfloat16, device="cuda"))
    assert e.shape == (0, 4)


# -- split-K form for decode-sized products (M <= 128) ----------------------

@pytest.mark.parametrize("M,N,K", [(64, 6144, 2048), (64, 2048, 2048), (1, 8, 8), (7, 384, 128),
                                   (100, 300, 136), (128, 257, 1000), (128, 6144 + 64, 2048),
                                   (33, 2048, 4096), (129, 512, 512)])
def test_linear_split_k_parity(M, N, K):
    """Every element against the fp64 matmul with the same bound as the
    persistent kernel: K chunks of whole and ragged 64-column steps, N off the
    tile grid, a single k-step (no split), and M = 129 (persistent kernel)."""
    x, w = bf16_pair(M, N, K, seed=3 * M + N + K)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = gdn.linear_bf16(x.cuda(), w.cuda(), status=status, split_k=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check(x, w, y)


def test_linear_split_k_rows_independent_of_batch():
    """The split depends on N and K alone: rows of a 128-row call equal the
    same rows of a 64-row call and computed alone, bit for bit."""
    M, N, K = 128, 6144, 2048
    x, w = bf16_pair(M, N, K, seed=17)
    xc, wc = x.cuda(), w.cuda()
    y = gdn.linear_bf16(xc, wc, split_k=True)
    y64 = gdn.linear_bf16(xc[64:].contiguous(), wc, split_k=True)
    torch.cuda.synchronize()
    assert torch.equal(y64, y[64:]), "rows 64..127"
    for r in (0, 63, 64, 127):
        yr = gdn.linear_bf16(xc[r:r + 1].contiguous(), wc, split_k=True)
        torch.cuda.synchronize()
        assert torch.equal(yr[0], y[r]), f"row {r}"


def test_linear_split_k_near_persistent_kernel():
    """The split form and the persistent kernel differ only by the grouping of
    the fp32 sum: within the accumulation bound of each other, and each within
    the bound of the exact product."""
    M, N, K = 64, 2048, 2048
    x, w = bf16_pair(M, N, K, seed=19, scale=4.0)
    xc, wc = x.cuda(), w.cuda()
    ys = gdn.linear_bf16(xc, wc, split_k=True)
    yp = gdn.linear_bf16(xc, wc)
    torch.cuda.synchronize()
    check(x, w, ys)
    check(x, w, yp)
    mag = (x.abs().double() @ w.abs().double().T).numpy()
    diff = (ys - yp).abs().double().cpu().numpy()
    assert np.all(diff <= 8e-7 * np.sqrt(K) * mag + 1e-30)
