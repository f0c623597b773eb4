"""The LFM2 short-conv mixer (gdn_short_conv_forward_batch / _forward / _pair)
on the GPU against the fp64 oracle, through the C ABI.

Tolerances. Both sides round y = cg * conv to bf16 before the output
projection; where the two unrounded values straddle a rounding boundary they
differ by one bf16 ulp on a few of the D terms of an output, which moves an
output of RMS ~0.4 by well under 1e-3: the bound is 2e-3 absolute (the one
the forward-batch tests use). A ring slot holds u = bg * xv, two outputs of
the fp32 input projection: its error is bounded by |xv| e_bg + |bg| e_xv plus
one fp32 rounding, where e_r is the projection's bound, a few fp32 units times
sqrt(D) relative to the sum of |h_i W_ri|. Slots carried over from the input
ring must be identical. Runs that must be elementwise identical (the same
positions in one call or in several) are compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_04_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

BF16 = ("hidden", "w_in", "w_out")
OUT_ABS = 2e-3


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def to_dev(d):
    t = {}
    for k, v in d.items():
        x = torch.from_numpy(np.ascontiguousarray(v)).cuda()
        t[k] = x.to(torch.bfloat16) if k in BF16 else x
    return t


def gpu_batch(t, hidden=None):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gdn.short_conv_forward_batch(t["hidden"] if hidden is None else hidden, t["w_in"],
                                       t["w_out"], t["conv_ring"], t["conv_w"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out


def check_out(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite"
    err = np.abs(gpu - ref)
    assert err.max() <= OUT_ABS, f"{what}: max abs {err.max():.3e} > {OUT_ABS}"


def check_ring(gpu_ring, ring_in, hidden, w_in, ref_ring, last, what):
    """Slot s of the ring holds the gated input of position last - (K-2) + s;
    positions before 0 come from `ring_in` unchanged."""
    h = hidden.astype(np.float64)
    W = w_in.astype(np.float64)
    D = h.shape[2]
    K1 = ref_ring.shape[1]
    gpu_ring = np.asarray(gpu_ring, np.float64)
    for slot in range(K1):
        t = last - (K1 - 1) + slot
        if t < 0:
            assert np.array_equal(gpu_ring[:, slot], ring_in[:, K1 + t]), f"{what}: carried slot"
            continue
        proj = h[:, t] @ W.T
        mag = np.abs(h[:, t]) @ np.abs(W).T
        e = 4e-7 * np.sqrt(D) * mag
        bg, xv = proj[:, :D], proj[:, 2 * D:]
        bound = np.abs(xv) * e[:, :D] + np.abs(bg) * e[:, 2 * D:] + e[:, :D] * e[:, 2 * D:] \
            + 2.0 ** -23 * np.abs(bg * xv) + 1e-30
        err = np.abs(gpu_ring[:, slot] - ref_ring[:, slot])
        assert np.all(err <= bound), f"{what}: slot {slot} error {np.max(err / bound):.2f} x bound"


@pytest.mark.parametrize("B,T,D,K", [(3, 1, 64, 3), (2, 5, 256, 2), (2, 37, 64, 4),
                                     (3, 70, 256, 3), (1, 33, 320, 3)])
def test_forward_batch_matches_oracle(o, B, T, D, K):
    d = inputs.short_conv_inputs(B, T, D=D, K=K, seed=1400 + T)
    t = to_dev(d)
    out = gpu_batch(t)
    ref_out, ref_ring = o.short_conv_forward_batch(d["hidden"], d["w_in"], d["w_out"],
                                                   d["conv_ring"], d["conv_w"])
    check_out(out.cpu().numpy(), ref_out, f"B{B} T{T} D{D} K{K} out")
    check_ring(t["conv_ring"].cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_ring,
               T - 1, f"B{B} T{T} D{D} K{K} ring")


def test_chunks_and_single_positions_are_elementwise_identical():
    """20 + 30 positions, and 50 single-position calls, give exactly the
    outputs and ring of one 50-position call."""
    B, T, D, K = 2, 50, 128, 3
    d = inputs.short_conv_inputs(B, T, D=D, K=K, seed=1450)
    whole = to_dev(d)
    out_whole = gpu_batch(whole)
    parts = to_dev(d)
    o1 = gpu_batch(parts, parts["hidden"][:, :20].contiguous())
    o2 = gpu_batch(parts, parts["hidden"][:, 20:].contiguous())
    assert torch.equal(torch.cat([o1, o2], dim=1), out_whole), "chunked outputs"
    assert torch.equal(parts["conv_ring"], whole["conv_ring"]), "chunked ring"
    single = to_dev(d)
    outs = []
    for s in range(T):
        outs.append(gdn.short_conv_forward(single["hidden"][:, s].contiguous(), single["w_in"],
                                           single["w_out"], single["conv_ring"],
                                           single["conv_w"]))
    torch.cuda.synchronize()
    assert torch.equal(torch.stack(outs, dim=1), out_whole), "single-position outputs"
    assert torch.equal(single["conv_ring"], whole["conv_ring"]), "single-position ring"


@pytest.mark.parametrize("B,T,D", [(3, 5, 1024), (2, 1, 1088), (7, 9, 1088)])
def test_wide_hidden_matches_oracle(o, B, T, D):
    """Hidden sizes of 16 and 17 k-steps of 64 (17 64-channel tiles for the
    fused projection-and-gate kernel), one position and several."""
    d = inputs.short_conv_inputs(B, T, D=D, K=3, seed=1480 + D + T)
    t = to_dev(d)
    out = gpu_batch(t)
    ref_out, ref_ring = o.short_conv_forward_batch(d["hidden"], d["w_in"], d["w_out"],
                                                   d["conv_ring"], d["conv_w"])
    check_out(out.cpu().numpy(), ref_out, f"B{B} T{T} D{D} out")
    check_ring(t["conv_ring"].cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_ring,
               T - 1, f"B{B} T{T} D{D} ring")


@pytest.mark.parametrize("K", [2, 3, 4])
def test_pair_matches_oracle(o, K):
    B, D = 5, 192
    d = inputs.short_conv_inputs(B, 2, D=D, K=K, seed=1460 + K)
    t = to_dev(d)
    scratch = torch.full_like(t["conv_ring"], float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gdn.short_conv_pair(t["hidden"], t["w_in"], t["w_out"], t["conv_ring"], scratch,
                              t["conv_w"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_out, ref_ring, ref_scratch = o.short_conv_pair(d["hidden"], d["w_in"], d["w_out"],
                                                       d["conv_ring"], d["conv_w"])
    check_out(out.cpu().numpy(), ref_out, f"pair K{K} out")
    check_ring(t["conv_ring"].cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_ring, 0,
               f"pair K{K} committed ring")
    check_ring(scratch.cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_scratch, 1,
               f"pair K{K} scratch ring")
    # the pair's outputs are those of a two-position batch, bit for bit
    t2 = to_dev(d)
    out2 = gpu_batch(t2)
    assert torch.equal(out, out2), "pair vs two-position batch"
    assert torch.equal(scratch, t2["conv_ring"]), "scratch ring vs two-position batch ring"


@pytest.mark.parametrize("B,T,D,K", [(3, 5, 200, 3), (2, 1, 1096, 4), (64, 1, 200, 2),
                                     (4, 30, 200, 3)])
def test_ragged_channel_tiles_match_oracle(o, B, T, D, K):
    """Hidden sizes off the 64-channel tile of the fused projection-and-gate
    kernel that calls of at most 128 rows take (200 = 3 x 64 + 8,
    1096 = 17 x 64 + 8); B*T of 15, 2, 64 and 120 rows."""
    d = inputs.short_conv_inputs(B, T, D=D, K=K, seed=1490 + D + T)
    t = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gdn.short_conv_forward_batch(t["hidden"], t["w_in"], t["w_out"], t["conv_ring"],
                                       t["conv_w"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_out, ref_ring = o.short_conv_forward_batch(d["hidden"], d["w_in"], d["w_out"],
                                                   d["conv_ring"], d["conv_w"])
    check_out(out.cpu().numpy(), ref_out, f"B{B} T{T} D{D} K{K} out")
    check_ring(t["conv_ring"].cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_ring,
               T - 1, f"B{B} T{T} D{D} K{K} ring")


def test_pair_ragged_channel_tile_matches_oracle(o):
    B, D, K = 6, 200, 4
    d = inputs.short_conv_inputs(B, 2, D=D, K=K, seed=1495)
    t = to_dev(d)
    scratch = torch.full_like(t["conv_ring"], float("nan"))
    out = gdn.short_conv_pair(t["hidden"], t["w_in"], t["w_out"], t["conv_ring"], scratch,
                              t["conv_w"])
    torch.cuda.synchronize()
    ref_out, ref_ring, ref_scratch = o.short_conv_pair(d["hidden"], d["w_in"], d["w_out"],
                                                       d["conv_ring"], d["conv_w"])
    check_out(out.cpu().numpy(), ref_out, "pair D200 out")
    check_ring(t["conv_ring"].cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_ring, 0,
               "pair D200 committed ring")
    check_ring(scratch.cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_scratch, 1,
               "pair D200 scratch ring")


def test_rows_of_calls_up_to_128_rows_are_batch_invariant():
    """Calls of at most 128 rows share one split of K (fixed by D): the
    sequences of a 64-sequence decode equal the same sequences decoded in a
    call of their own, bit for bit (outputs and rings)."""
    B, D = 64, 2048
    d = inputs.short_conv_inputs(B, 1, D=D, K=3, seed=1497)
    whole = to_dev(d)
    out_all = gdn.short_conv_forward(whole["hidden"][:, 0].contiguous(), whole["w_in"],
                                     whole["w_out"], whole["conv_ring"], whole["conv_w"])
    for b in (0, 37, 63):
        one = to_dev({k: (v[b:b + 1] if k in ("hidden", "conv_ring") else v)
                      for k, v in d.items()})
        o1 = gdn.short_conv_forward(one["hidden"][:, 0].contiguous(), one["w_in"], one["w_out"],
                                    one["conv_ring"], one["conv_w"])
        torch.cuda.synchronize()
        assert torch.equal(o1[0], out_all[b]), f"sequence {b} output"
        assert torch.equal(one["conv_ring"][0], whole["conv_ring"][b]), f"sequence {b} ring"


def test_empty_batch_is_a_no_op():
    d = inputs.short_conv_inputs(2, 1, D=64, seed=1470)
    t = to_dev(d)
    ring0 = t["conv_ring"].clone()
    out = gdn.short_conv_forward_batch(t["hidden"][:, :0].contiguous(), t["w_in"], t["w_out"],
                                       t["conv_ring"], t["conv_w"])
    torch.cuda.synchronize()
    assert out.shape == (2, 0, 64)
    assert torch.equal(t["conv_ring"], ring0)


def test_decode_b64_full_size(o):
    """The benchmark's decode launch (64 sequences, D = 2048, K = 3), every
    sequence against the oracle."""
    w = inputs.SHORT_CONV_WORKLOADS["short_conv_decode_b64"]
    d = w.draw()
    t = to_dev(d)
    out = gdn.short_conv_forward(t["hidden"][:, 0].contiguous(), t["w_in"], t["w_out"],
                                 t["conv_ring"], t["conv_w"])
    torch.cuda.synchronize()
    ref_out, ref_ring = o.short_conv_forward_batch(d["hidden"], d["w_in"], d["w_out"],
                                                   d["conv_ring"], d["conv_w"])
    check_out(out.cpu().numpy(), ref_out[:, 0], "decode_b64 out")
    check_ring(t["conv_ring"].cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_ring, 0,
               "decode_b64 ring")


def test_batch_b4_t4096_full_size_sampled(o):
    """The benchmark's 4 x 4096-position launch. Sequence 0's first 40
    positions against the oracle from the true ring; for every sequence the
    last 12 positions against the oracle started 12 positions early from an
    arbitrary ring (after K-1 positions the window no longer reaches it), and
    the final rings."""
    w = inputs.SHORT_CONV_WORKLOADS["short_conv_batch_b4_t4096"]
    d = w.draw()
    t = to_dev(d)
    out = gpu_batch(t).cpu().numpy()
    B, T, D = d["hidden"].shape
    K = d["conv_w"].shape[1]
    head = {k: (v[:1, :40] if k == "hidden" else v[:1] if k == "conv_ring" else v)
            for k, v in d.items()}
    ref_head, _ = o.short_conv_forward_batch(head["hidden"], d["w_in"], d["w_out"],
                                             head["conv_ring"], d["conv_w"])
    check_out(out[:1, :40], ref_head, "batch_b4_t4096 head")
    tail_h = d["hidden"][:, T - 12:]
    ref_tail, ref_ring = o.short_conv_forward_batch(tail_h, d["w_in"], d["w_out"],
                                                    np.zeros_like(d["conv_ring"]), d["conv_w"])
    check_out(out[:, T - 12 + (K - 1):], ref_tail[:, K - 1:], "batch_b4_t4096 tail")
    check_ring(t["conv_ring"].cpu().numpy(), None, tail_h, d["w_in"], ref_ring, 11,
               "batch_b4_t4096 ring")


def test_pair_b64_full_size(o):
    """The benchmark's verify launch (64 sequences, D = 2048, K = 3), every
    sequence against the oracle: outputs, committed and scratch rings."""
    d = inputs.SHORT_CONV_WORKLOADS["short_conv_pair_b64"].draw()
    t = to_dev(d)
    scratch = torch.full_like(t["conv_ring"], float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gdn.short_conv_pair(t["hidden"], t["w_in"], t["w_out"], t["conv_ring"], scratch,
                              t["conv_w"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_out, ref_ring, ref_scratch = o.short_conv_pair(d["hidden"], d["w_in"], d["w_out"],
                                                       d["conv_ring"], d["conv_w"])
    check_out(out.cpu().numpy(), ref_out, "pair_b64 out")
    check_ring(t["conv_ring"].cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_ring, 0,
               "pair_b64 committed ring")
    check_ring(scratch.cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"], ref_scratch, 1,
               "pair_b64 scratch ring")


def check_word(ws, need, D):
    """The barrier word: (48-bit tag << 16) | count, count = CTAs of the grid."""
    w = int.from_bytes(bytes(ws[need - 256:need - 248].cpu().numpy()), "little")
    count, tag = w & 0xFFFF, w >> 16
    tiles = D // 64
    assert tag != 0 and count >= 2 * tiles and count % tiles == 0, f"barrier word {w:#x}"


def test_one_kernel_decode_graph_replay_and_stale_workspace():
    """Calls of one position with D = 2048 run the whole mixer as one kernel
    whose grid-wide barrier lives in the workspace's last 256 bytes. A
    workspace full of stale bytes works from the first call, every call
    leaves the barrier word holding its tag and a count of the whole grid
    (64-channel tiles times K chunks), and a CUDA graph replayed three times
    (the same call, so the same tag, each replay finding the previous one's
    complete count) gives the outputs and ring of three eager calls bit for
    bit."""
    B, D, K, steps = 64, 2048, 3, 3
    d = inputs.short_conv_inputs(B, steps, D=D, K=K, seed=1498)
    need = gdn.short_conv_workspace_size(B, 1, D)
    ws = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda")
    eager = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for s in range(steps):
        outs.append(gdn.short_conv_forward(eager["hidden"][:, s].contiguous(), eager["w_in"],
                                           eager["w_out"], eager["conv_ring"], eager["conv_w"],
                                           workspace=ws, status=status))
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        check_word(ws, need, D)
    ref_out, _ = oracle.load().short_conv_forward_batch(d["hidden"], d["w_in"], d["w_out"],
                                                        d["conv_ring"], d["conv_w"])
    check_out(torch.stack(outs, dim=1).cpu().numpy(), ref_out, "eager decode steps")

    g = to_dev(d)
    h_in = torch.empty_like(g["hidden"][:, 0]).contiguous()
    out_g = torch.empty(B, D, dtype=torch.float32, device="cuda")
    ws.fill_(0x5A)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            gdn.short_conv_forward(h_in, g["w_in"], g["w_out"], g["conv_ring"], g["conv_w"],
                                   out=out_g, workspace=ws, status=status)
    torch.cuda.synchronize()
    for s in range(steps):
        h_in.copy_(g["hidden"][:, s])
        graph.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out_g, outs[s]), f"replay {s} output"
    assert torch.equal(g["conv_ring"], eager["conv_ring"]), "ring after the replays"
    check_word(ws, need, D)
    del graph


@pytest.mark.parametrize("T", [1, 2])
def test_one_kernel_and_two_kernel_paths_are_bit_identical(monkeypatch, T):
    """GDN_SHORT_CONV_ONE_KERNEL=0 selects the two-kernel path for decode and
    verify calls; both paths give the same outputs and rings bit for bit
    (64 sequences, D = 2048, K = 3)."""
    B, D, K = 64, 2048, 3
    d = inputs.short_conv_inputs(B, T, D=D, K=K, seed=1499 + T)
    runs = {}
    for flag in ("1", "0"):
        monkeypatch.setenv("GDN_SHORT_CONV_ONE_KERNEL", flag)
        t = to_dev(d)
        need = gdn.short_conv_workspace_size(B, T, D)
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        if T == 1:
            out = gdn.short_conv_forward(t["hidden"][:, 0].contiguous(), t["w_in"], t["w_out"],
                                         t["conv_ring"], t["conv_w"], workspace=ws,
                                         status=status)
            scratch = None
        else:
            scratch = torch.full_like(t["conv_ring"], float("nan"))
            out = gdn.short_conv_pair(t["hidden"], t["w_in"], t["w_out"], t["conv_ring"],
                                      scratch, t["conv_w"], workspace=ws, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        word = int.from_bytes(bytes(ws[need - 256:need - 248].cpu().numpy()), "little")
        runs[flag] = (out, t["conv_ring"], scratch, word)
    one, two = runs["1"], runs["0"]
    assert one[3] != 0 and two[3] == 0, "the barrier word shows which path ran"
    assert torch.equal(one[0], two[0]), "outputs"
    assert torch.equal(one[1], two[1]), "committed ring"
    if T == 2:
        assert torch.equal(one[2], two[2]), "scratch ring"


@pytest.mark.parametrize("K", [3, 4])
def test_decode_b128_full_rows_matches_oracle(o, monkeypatch, K):
    """128 sequences, one position: the largest call of the split forms. With
    K = 3 it runs as one kernel (all 128 rows of every partial and y box
    real) and equals the two-kernel path bit for bit; with K = 4 the rings of
    a CTA's channels no longer fit its shared-memory cache and the call takes
    the two kernels. Both against the oracle."""
    B, D = 128, 2048
    d = inputs.short_conv_inputs(B, 1, D=D, K=K, seed=1510 + K)
    ref_out, ref_ring = o.short_conv_forward_batch(d["hidden"], d["w_in"], d["w_out"],
                                                   d["conv_ring"], d["conv_w"])
    results = {}
    for flag in ("1", "0"):
        monkeypatch.setenv("GDN_SHORT_CONV_ONE_KERNEL", flag)
        t = to_dev(d)
        need = gdn.short_conv_workspace_size(B, 1, D)
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = gdn.short_conv_forward(t["hidden"][:, 0].contiguous(), t["w_in"], t["w_out"],
                                     t["conv_ring"], t["conv_w"], workspace=ws, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        word = int.from_bytes(bytes(ws[need - 256:need - 248].cpu().numpy()), "little")
        results[flag] = (out, t["conv_ring"], word)
        check_out(out.cpu().numpy(), ref_out[:, 0], f"decode_b128 K{K} out ({flag})")
        check_ring(t["conv_ring"].cpu().numpy(), d["conv_ring"], d["hidden"], d["w_in"],
                   ref_ring, 0, f"decode_b128 K{K} ring ({flag})")
    one, two = results["1"], results["0"]
    assert two[2] == 0
    assert (one[2] != 0) == (K == 3), "one kernel for K = 3 only"
    assert torch.equal(one[0], two[0]) and torch.equal(one[1], two[1])
