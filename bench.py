"""Benchmark of the Gated DeltaNet recurrent-state update on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one batched decode token through ``gdn_step`` over the B = 64
workload (64 sequences x 32 value heads x 128 x 128 fp32 state, one layer).
The timed region holds exactly K steps, bracketed by a barrier and a device
synchronisation on both sides and timed with CUDA events on the launching
stream; with N ranks each rank runs its own B = 64 batch (weak scaling, no
collective on the data path) and the slowest rank's time is used. Without a
launcher, ``--gpus N`` (N > 1) starts N ranks itself through torchrun; under
a launcher, N must equal WORLD_SIZE.

The metric is state GB/s: each value head's 64 KiB state read once and
written once per token, counted the same way in every figure (the GPU step,
the end-to-end leg, the CPU baselines and the reference arm).

Printed (rank 0, one JSON line): state GB/s over all ranks, layer-tokens/s,
the roofline of the step kernel against the measured HBM copy bandwidth, an
end-to-end figure through the C ABI with the per-step inputs copied from
pinned host memory and the output copied back (graph-replayed and eager),
NVML clock samples taken during the timed region, the CPU oracle timed on
this host as a reported baseline (its literal fp32 instantiation, and the
fp64 parity oracle beside it), and (N = 1) the other workloads (36-layer and
B = 1 decode, prefill, fused layer and verify, batched forward, KDA core,
short-conv mixer) measured the same way, each with its roofline.

``--impl reference`` times the CPU oracle alone on the same workload and
metric (rank 0 only; other ranks exit at once).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time
from typing import Dict, List, Optional

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gdn_step state GB/s and % of HBM peak; layer-tokens/s at B=64 decode"
UNIT = "GB/s"
HEADLINE = "decode_l1_b64"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
STATE_BYTES_PER_HEAD = 128 * 128 * 4
E2E_SLOTS = 2            # device buffer slots of the end-to-end pipeline

# Algorithmic bytes of one value-head token of gdn_step: state read + write,
# v in, out, beta and gate, and q/k of its key head shared by Hv / Hk value heads.
def step_bytes(L: int, B: int, Hk: int = 16, Hv: int = 32, d: int = 128) -> int:
    heads = L * B * Hv
    return heads * (2 * d * d * 4 + 2 * d * 4 + 2 * 4) + L * B * Hk * 2 * d * 4


def state_rw_bytes(L: int, B: int, Hv: int = 32, d: int = 128) -> int:
    """State bytes one decode token moves: every value head's d x d fp32 state
    read once and written once. The headline metric (state GB/s) is this
    figure per second, in every arm: the GPU step, the end-to-end leg, the
    CPU oracle baselines and the reference arm."""
    return 2 * L * B * Hv * d * d * 4


def state_gb_s(units: int, seconds: float, n_ranks: int = 1, d: int = 128) -> float:
    """State GB/s of `units` value-head tokens per rank over `seconds` (the
    slowest rank's time): read + write of each unit's d x d fp32 state."""
    return throughput(units * 2 * d * d * 4 / 1e9, n_ranks, seconds)


def pair_bytes(L: int, B: int, Hk: int = 16, Hv: int = 32, d: int = 128) -> int:
    """gdn_pair: each state row read once and written twice (committed and
    scratch), and two positions of q/k, v, out, beta and gate."""
    heads = L * B * Hv
    return heads * (3 * d * d * 4 + 2 * (2 * d * 4 + 2 * 4)) + L * B * 2 * Hk * 2 * d * 4


def prefill_bytes(B: int, T: int, Hk: int = 16, Hv: int = 32, d: int = 128) -> int:
    return (2 * B * Hv * d * d * 4 + B * T * (Hk * 2 * d * 4 + Hv * (2 * d * 4 + 2 * 4)))


def prefill_flops(B: int, T: int, Hv: int = 32, d: int = 128) -> int:
    # per state element and position: decay (1), sk (2), update (2), output (2)
    return 7 * B * T * Hv * d * d


def layer_bytes(B: int, Hk: int = 16, Hv: int = 32, d: int = 128, K: int = 4) -> int:
    C = 2 * Hk * d + Hv * d
    return (B * Hv * d * d * 4 * 2 + B * (K - 1) * C * 4 * 2 + B * C * 4 + B * Hv * d * 4 * 2
            + B * Hv * 4 * 2 + C * K * 4 + Hv * 4 * 2 + d * 4)


def layer_pair_bytes(B: int, Hk: int = 16, Hv: int = 32, d: int = 128, K: int = 4) -> int:
    """State read once and written twice (committed + scratch), ring likewise,
    and two positions of activations and outputs."""
    C = 2 * Hk * d + Hv * d
    return (B * Hv * d * d * 4 * 3 + B * (K - 1) * C * 4 * 3
            + 2 * (B * C * 4 + B * Hv * d * 4 * 2 + B * Hv * 4 * 2)
            + C * K * 4 + Hv * 4 * 2 + d * 4)


def kda_step_bytes(L: int, B: int, Hk: int = 16, Hv: int = 32, d: int = 128) -> int:
    """gdn_step's bytes with the scalar gate replaced by a log-decay per key
    channel (d floats per value head)."""
    return step_bytes(L, B, Hk, Hv, d) + L * B * Hv * (d - 1) * 4


def short_conv_bytes(B: int, T: int, D: int = 2048, K: int = 3, pair: bool = False) -> int:
    """One launch of the short-conv mixer: both weight matrices (bf16) once,
    hidden in and out, the ring read and written (twice for the verify's
    committed and scratch rings), the conv weight."""
    rings = 3 if pair else 2
    return (3 * D * D * 2 + D * D * 2 + B * T * D * 2 + B * T * D * 4
            + rings * B * (K - 1) * D * 4 + D * K * 4)


def short_conv_flops(B: int, T: int, D: int = 2048) -> int:
    return 2 * B * T * D * 3 * D + 2 * B * T * D * D


# --------------------------------------------------------------------------
# host-side helpers (no GPU needed; covered by the CPU tests)
# --------------------------------------------------------------------------
def dist_env() -> Dict[str, int]:
    return dict(rank=int(os.environ.get("RANK", 0)), world=int(os.environ.get("WORLD_SIZE", 1)),
                local_rank=int(os.environ.get("LOCAL_RANK", 0)))


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling): distinct, reproducible seeds."""
    return base + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(units_per_rank: float, n_ranks: int, seconds: float) -> float:
    """Whole-job throughput: units processed by all ranks over the slowest rank's time."""
    return units_per_rank * n_ranks / seconds if seconds > 0 else float("nan")


def measured_peaks() -> Dict[str, object]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS, source="fallback")


def kernel_source_digest(names: List[str]) -> str:
    """Short hash of kernel sources; a stored ncu traffic figure is used only
    while the source it was taken from is unchanged."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "linear_attention_recurrence_04_b200", "csrc", n), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, digest: str) -> Optional[float]:
    """DRAM bytes per launch from the committed ncu summary, if still current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_digest") != digest:
        return None
    return float(rec["dram_bytes_per_launch"])


REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


def decode_reasons(mask: int) -> List[str]:
    return [name for bit, name in REASON_BITS.items() if mask & bit]


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples: List[int] = []
        self.reasons = 0
        self.max_mhz: Optional[int] = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        self._handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nvml = pynvml
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self._handle = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self._handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = int(pynvml.nvmlDeviceGetMaxClockInfo(self._handle,
                                                                pynvml.NVML_CLOCK_SM))
        except Exception:
            self._nvml = None

    def _sample(self):
        p = self._nvml
        self.samples.append(int(p.nvmlDeviceGetClockInfo(self._handle, p.NVML_CLOCK_SM)))
        try:
            mask = p.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
        except AttributeError:
            mask = p.nvmlDeviceGetCurrentClocksThrottleReasons(self._handle)
        self.reasons |= int(mask)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                break
            self._stop.wait(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
            if not self.samples:
                self._sample()

    def summary(self) -> Dict[str, object]:
        if self._nvml is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvml_unavailable"], samples=0)
        med = float(np.median(self.samples)) if self.samples else None
        reasons = [r for r in decode_reasons(self.reasons) if r != "gpu_idle"]
        return dict(sm_mhz=med, sm_max_mhz=self.max_mhz, reasons=reasons,
                    samples=len(self.samples))


# --------------------------------------------------------------------------
# GPU measurement
# --------------------------------------------------------------------------
def _to_dev(d: Dict[str, np.ndarray], device) -> Dict[str, "torch.Tensor"]:
    import torch
    return {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in d.items()}


def step_footprint(L: int, B: int, Hk: int = 16, Hv: int = 32, d: int = 128) -> int:
    """Bytes of one decode input set (state, q, k, v, beta, gate) and its
    output, the unit the timed launches rotate over."""
    return (L * B * Hv * d * d * 4 + 2 * L * B * Hk * d * 4 + 2 * L * B * Hv * d * 4
            + 2 * L * B * Hv * 4)


def _sets_for(bytes_per_set: int) -> int:
    """Rotating input sets so the sets together exceed 4x the L2."""
    return max(1, min(64, math.ceil(4 * L2_BYTES / max(bytes_per_set, 1))))


def capture(launches, device):
    """A CUDA graph holding the given launches (callables), in order."""
    import torch
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    with torch.cuda.graph(g, stream=side):
        for fn in launches:
            fn()
    return g


def time_launches(launch, n_sets: int, steps: int, warmup: int, stream,
                  graph: bool = False) -> float:
    """Run `launch(i)` for warmup + steps iterations, rotating input set
    i % n_sets; return the device seconds of the timed steps. With
    graph=True the timed steps are captured once into a CUDA graph and
    replayed, so host launch overhead does not enter the timing."""
    import torch
    for i in range(warmup):
        launch(i % n_sets)
    torch.cuda.synchronize()
    g = None
    if graph and steps > 0:
        g = capture([(lambda j=j: launch((warmup + j) % n_sets)) for j in range(steps)],
                    stream.device)
        torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    if g is not None:
        g.replay()
    else:
        for i in range(steps):
            launch((warmup + i) % n_sets)
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / 1e3


def bench_step_workload(name: str, steps: int, warmup: int, device, seed_offset: int = 0,
                        graph: bool = True):
    import torch
    from linear_attention_recurrence_04_b200 import gdn, inputs
    w = inputs.WORKLOADS[name]
    L, B = w.sizes["L"], w.sizes["B"]
    d = inputs.decode_inputs(L, B, seed=w.seed + seed_offset)
    base = _to_dev(d, device)
    nbytes = step_bytes(L, B)
    footprint = step_footprint(L, B)
    assert footprint == sum(v.nbytes for v in d.values()) + d["v"].nbytes   # inputs + out
    n_sets = _sets_for(footprint)
    sets = [base] + [{k: v.clone() for k, v in base.items()} for _ in range(n_sets - 1)]
    outs = [torch.empty_like(s["v"]) for s in sets]
    stream = torch.cuda.current_stream(device)

    def launch(i):
        s = sets[i]
        gdn.step(s["state"], s["q"], s["k"], s["v"], s["beta"], s["gate"], outs[i])

    secs = time_launches(launch, n_sets, steps, warmup, stream, graph=graph)
    return dict(seconds=secs, bytes=nbytes, units=L * B * 32, state_rw=state_rw_bytes(L, B),
                layer_tokens=L * B, n_sets=n_sets, set_bytes=footprint, sets=sets, outs=outs,
                d=d)


def bench_e2e(d: Dict[str, np.ndarray], steps: int, warmup: int, device):
    """gdn_step through the C ABI with each step's q, k, v, beta, gate copied
    from pinned host memory and the output copied back to pinned host memory,
    all inside the timed region. The recurrent state stays resident on the
    device, as a decode cache does.

    The per-step inputs are packed in one pinned buffer (one host-to-device
    copy per step). Copy-in, compute and copy-out run on three streams with
    two device buffer slots, so step i+1's inputs travel while step i
    computes and step i-1's output travels back; events order every reuse of
    a slot. The same K-step loop is timed twice:
      - graph: the K steps (each one's copy-in, gdn_step call through the C
        ABI and copy-out) captured once into a CUDA graph and replayed, as a
        serving loop would, so host-side issue does not pace the GPU;
      - eager: the K steps issued from Python, each one a ctypes call of
        gdn_step with the library's argument checks and launch on the host.
    Each timed region runs from before the first copy-in to after the last
    copy-out. Returns (graph_seconds, eager_seconds, h2d_bytes, d2h_bytes)."""
    import torch
    from linear_attention_recurrence_04_b200 import gdn
    names = ("q", "k", "v", "beta", "gate")
    sizes = [int(np.prod(d[n].shape)) for n in names]
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
    packed = np.concatenate([np.ascontiguousarray(d[n], dtype=np.float32).ravel() for n in names])
    host_in = torch.from_numpy(packed).pin_memory()
    n_slots = E2E_SLOTS
    dev_in = [torch.empty_like(host_in, device=device) for _ in range(n_slots)]
    views = [{n: dev_in[sl][offs[i]:offs[i + 1]].view(d[n].shape) for i, n in enumerate(names)}
             for sl in range(n_slots)]
    dev_out = [torch.empty(d["v"].shape, dtype=torch.float32, device=device) for _ in range(n_slots)]
    host_out = [torch.empty(d["v"].shape, dtype=torch.float32).pin_memory() for _ in range(n_slots)]
    state_bytes = d["state"].nbytes
    n_sets = _sets_for(state_bytes)
    states = [torch.from_numpy(d["state"]).to(device) for _ in range(n_sets)]
    s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_ready = [ev() for _ in range(n_slots)]
    comp_done = [ev() for _ in range(n_slots)]
    out_done = [ev() for _ in range(n_slots)]
    used = [False] * n_slots

    def step(i):
        sl = i % n_slots
        with torch.cuda.stream(s_in):
            if used[sl]:
                s_in.wait_event(comp_done[sl])           # slot's inputs no longer read
            dev_in[sl].copy_(host_in, non_blocking=True)
            in_ready[sl].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_ready[sl])
            if used[sl]:
                s_comp.wait_event(out_done[sl])          # slot's output already copied out
            v = views[sl]
            gdn.step(states[i % n_sets], v["q"], v["k"], v["v"], v["beta"], v["gate"],
                     dev_out[sl], stream=s_comp)
            comp_done[sl].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[sl])
            host_out[sl].copy_(dev_out[sl], non_blocking=True)
            out_done[sl].record(s_out)
        used[sl] = True

    def loop(origin):
        # the three streams fork from `origin` and join it again at the end
        for s in (s_in, s_comp, s_out):
            s.wait_stream(origin)
        for i in range(steps):
            step(warmup + i)
        for s in (s_in, s_comp, s_out):
            origin.wait_stream(s)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    # graph: slot reuse inside the graph waits only on events recorded inside it
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device)
    used[:] = [False] * n_slots
    with torch.cuda.graph(graph, stream=cap):
        loop(cap)
    torch.cuda.synchronize()
    replay = torch.cuda.current_stream(device)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(replay)
    graph.replay()
    end.record(replay)
    torch.cuda.synchronize()
    graph_secs = start.elapsed_time(end) / 1e3
    del graph
    # eager: the same loop issued call by call
    used[:] = [False] * n_slots
    start.record(replay)
    loop(replay)
    end.record(replay)
    torch.cuda.synchronize()
    eager_secs = start.elapsed_time(end) / 1e3
    h2d = host_in.numel() * host_in.element_size()
    d2h = host_out[0].numel() * host_out[0].element_size()
    return graph_secs, eager_secs, h2d, d2h


def bench_prefill(steps: int, warmup: int, device):
    """Each launch starts from the zero state (restored outside the timed
    interval); the launches alone are timed, one event pair each."""
    import torch
    from linear_attention_recurrence_04_b200 import gdn, inputs
    w = inputs.WORKLOADS["prefill_b4_t4096"]
    B, T = w.sizes["B"], w.sizes["T"]
    t = _to_dev(w.draw(), device)
    out = torch.empty_like(t["v"])
    state0 = t["state"].clone()
    stream = torch.cuda.current_stream(device)
    total = 0.0
    for i in range(warmup + steps):
        t["state"].copy_(state0)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        gdn.prefill(t["state"], t["q"], t["k"], t["v"], t["beta"], t["gate"], out)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= warmup:
            total += a.elapsed_time(b) / 1e3
    return dict(seconds=total, launches=steps, bytes=prefill_bytes(B, T),
                flops=prefill_flops(B, T), tokens=B * T)


def _bf16_dev(d: Dict[str, np.ndarray], bf16_names, device) -> Dict[str, "torch.Tensor"]:
    import torch
    return {k: (torch.from_numpy(v).to(device).to(torch.bfloat16) if k in bf16_names
                else torch.from_numpy(v).to(device)) for k, v in d.items()}


def build_case(name: str, device):
    """(launch(i), meta) for one named workload on seeded synthetic inputs
    resident on `device`; `launch` issues one call of the library on the
    current stream. Used by the benchmark legs and by --profile-case."""
    import torch
    from linear_attention_recurrence_04_b200 import gdn, inputs
    if name in inputs.WORKLOADS and inputs.WORKLOADS[name].kind == "step":
        w = inputs.WORKLOADS[name]
        t = _to_dev(w.draw(), device)
        out = torch.empty_like(t["v"])
        return (lambda i: gdn.step(t["state"], t["q"], t["k"], t["v"], t["beta"], t["gate"],
                                   out)), dict(tensors=t)
    if name == "decode_l1_b64_rotated":
        # the benchmark's rotation: launch i uses input set i % n_sets, so a
        # run of launches shows each one's DRAM traffic in steady state (the
        # write-backs a launch leaves in L2 are paid by the ones after it)
        r = bench_step_workload("decode_l1_b64", 0, 0, device)
        sets, outs = r["sets"], r["outs"]
        return (lambda i: gdn.step(sets[i % len(sets)]["state"], sets[i % len(sets)]["q"],
                                   sets[i % len(sets)]["k"], sets[i % len(sets)]["v"],
                                   sets[i % len(sets)]["beta"], sets[i % len(sets)]["gate"],
                                   outs[i % len(sets)])), dict(n_sets=len(sets))
    if name == "pair_l1_b64":
        # two input sets of 256 MiB of state each, so a launch's state rows
        # are not still in L2 from the one before
        w = inputs.PAIR_WORKLOAD
        first = _to_dev(w.draw(), device)
        sets = []
        for si in range(2):
            t = first if si == 0 else {n: x.clone() for n, x in first.items()}
            sets.append((t, torch.empty_like(t["state"]), torch.empty_like(t["v"])))

        def launch(i):
            t, scratch, out = sets[i % len(sets)]
            gdn.pair(t["state"], scratch, t["q"], t["k"], t["v"], t["beta"], t["gate"], out)
        return launch, dict(sizes=w.sizes)
    if name == "prefill_b4_t4096":
        w = inputs.WORKLOADS[name]
        t = _to_dev(w.draw(), device)
        out = torch.empty_like(t["v"])
        return (lambda i: gdn.prefill(t["state"], t["q"], t["k"], t["v"], t["beta"], t["gate"],
                                      out)), dict(tensors=t, B=w.sizes["B"], T=w.sizes["T"])
    order = ("mixed_qkv", "z", "a", "b", "conv_ring", "conv_w", "A_log", "dt_bias", "norm_w",
             "state")
    if name == "layer_decode_b256":
        w = inputs.WORKLOADS[name]
        t = _to_dev(w.draw(), device)
        out = torch.empty_like(t["z"])
        return (lambda i: gdn.layer_decode(*(t[n] for n in order), out, Hk=16)), \
            dict(B=w.sizes["B"])
    if name == "layer_pair_b256":
        B = 256
        d = inputs.layer_inputs(B, seed=1005)
        d2 = inputs.layer_inputs(B, seed=1006)
        for n in ("mixed_qkv", "z", "a", "b"):
            d[n] = np.stack([d[n], d2[n]], axis=1)
        t = _to_dev(d, device)
        sring = torch.empty_like(t["conv_ring"])
        sstate = torch.empty_like(t["state"])
        out = torch.empty((B, 2, 32 * 128), dtype=torch.float32, device=device)
        return (lambda i: gdn.layer_pair(*(t[n] for n in order), sring, sstate, out, Hk=16)), \
            dict(B=B)
    if name == "forward_batch_b4_t4096":
        w = inputs.FORWARD_WORKLOAD
        B, T = w.sizes["B"], w.sizes["T"]
        t = _bf16_dev(w.draw(), ("hidden", "w_qkv", "w_z", "w_ba", "w_out"), device)
        D = t["hidden"].shape[2]
        out = torch.empty((B, T, D), dtype=torch.float32, device=device)
        ws = torch.empty(gdn.forward_batch_workspace_size(B, T), dtype=torch.uint8,
                         device=device)

        def launch(i):
            gdn.forward_batch(t["hidden"], t["w_qkv"], t["w_z"], t["w_ba"], t["w_out"],
                              t["conv_ring"], t["conv_w"], t["A_log"], t["dt_bias"],
                              t["norm_w"], t["state"], out, ws, Hk=16)
        return launch, dict(B=B, T=T, D=D)
    if name in inputs.KDA_WORKLOADS:
        w = inputs.KDA_WORKLOADS[name]
        t = _to_dev(w.draw(), device)
        out = torch.empty_like(t["v"])
        fn = gdn.kda_step if w.kind == "kda_step" else gdn.kda_prefill
        return (lambda i: fn(t["state"], t["q"], t["k"], t["v"], t["beta"], t["g"], out)), \
            dict(sizes=w.sizes, tensors=t)
    if name in inputs.SHORT_CONV_WORKLOADS:
        w = inputs.SHORT_CONV_WORKLOADS[name]
        B, T, D, K = (w.sizes[k] for k in ("B", "T", "D", "K"))
        t = _bf16_dev(w.draw(), ("hidden", "w_in", "w_out"), device)
        meta = dict(B=B, T=T, D=D, K=K, sets=1)
        if T <= 2:
            # decode-sized calls stream the weights: copies of them, together
            # over 4x the L2, rotate from launch to launch (a layer's weights
            # are not in L2 when its next token comes)
            n = _sets_for(t["w_in"].nbytes + t["w_out"].nbytes)
            w_in = [t["w_in"]] + [t["w_in"].clone() for _ in range(n - 1)]
            w_out = [t["w_out"]] + [t["w_out"].clone() for _ in range(n - 1)]
            meta["sets"] = n
        if name == "short_conv_pair_b64":
            out = torch.empty((B, 2, D), dtype=torch.float32, device=device)
            ws = torch.empty(gdn.short_conv_workspace_size(B, 2, D), dtype=torch.uint8,
                             device=device)
            sring = torch.empty_like(t["conv_ring"])
            return (lambda i: gdn.short_conv_pair(t["hidden"], w_in[i % len(w_in)], w_out[i % len(w_out)],
                                                  t["conv_ring"], sring, t["conv_w"], out,
                                                  ws)), meta
        out = torch.empty((B, T, D), dtype=torch.float32, device=device)
        ws = torch.empty(gdn.short_conv_workspace_size(B, T, D), dtype=torch.uint8,
                         device=device)
        if T == 1:
            h1, o1 = t["hidden"][:, 0], out[:, 0]
            return (lambda i: gdn.short_conv_forward(h1, w_in[i % len(w_in)], w_out[i % len(w_out)], t["conv_ring"],
                                                     t["conv_w"], o1, ws)), meta
        return (lambda i: gdn.short_conv_forward_batch(t["hidden"], t["w_in"], t["w_out"],
                                                       t["conv_ring"], t["conv_w"], out,
                                                       ws)), meta
    if name == "linear_bf16_m16384_n8192_k2048":
        M, N, K = 16384, 8192, 2048
        r = np.random.default_rng(1010)
        x = torch.from_numpy(inputs.to_bf16_values(r.normal(size=(M, K)))).to(device)
        wt = torch.from_numpy(inputs.to_bf16_values(r.normal(0, K ** -0.5, (N, K)))).to(device)
        x, wt = x.to(torch.bfloat16), wt.to(torch.bfloat16)
        y = torch.empty((M, N), dtype=torch.float32, device=device)
        return (lambda i: gdn.linear_bf16(x, wt, y)), dict(flops=2 * M * N * K)
    raise KeyError(f"unknown case {name!r}")


PROFILE_CASES = ("decode_l1_b1", "decode_l1_b64", "decode_l1_b64_rotated", "decode_l36_b16",
                 "pair_l1_b64",
                 "prefill_b4_t4096", "layer_decode_b256", "layer_pair_b256", "forward_batch_b4_t4096",
                 "linear_bf16_m16384_n8192_k2048", "short_conv_decode_b64", "short_conv_pair_b64",
                 "short_conv_batch_b4_t4096", "kda_decode_b64", "kda_prefill_b4_t4096")


CUBLAS_SHAPES = ((16384, 8192, 2048), (16384, 4096, 2048), (16384, 2048, 4096), (16384, 64, 2048),
                 (8192, 8192, 8192), (64, 6144, 2048), (64, 2048, 2048))


def run_cublas_compare(reps: int = 20) -> int:
    """gdn_linear_bf16 (and, for at most 128 rows, its split-K form) against
    cuBLAS (torch.mm with bf16 inputs and fp32 output) on the layer's
    projection shapes, each graph-replayed `reps` times between CUDA events;
    products of at most 128 rows rotate 16 weight sets (more than the L2).
    Prints one JSON line per shape with both times and the largest absolute
    difference of the two outputs."""
    import torch
    from linear_attention_recurrence_04_b200 import gdn
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev).manual_seed(1011)

    def timed(fn, n_sets):
        for i in range(3):
            fn(i % n_sets)
        torch.cuda.synchronize()
        g = capture([(lambda j=j: fn(j % n_sets)) for j in range(reps)], dev)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps * 1e3

    for M, N, K in CUBLAS_SHAPES:
        n_sets = 16 if M <= 128 else 1
        x = torch.randn(M, K, device=dev, generator=gen).to(torch.bfloat16)
        ws = [torch.randn(N, K, device=dev, generator=gen).mul(K ** -0.5).to(torch.bfloat16)
              for _ in range(n_sets)]
        y = torch.empty(M, N, device=dev, dtype=torch.float32)
        yc = torch.empty_like(y)
        line = {"M": M, "N": N, "K": K,
                "gdn_linear_bf16_us": timed(lambda i: gdn.linear_bf16(x, ws[i], y), n_sets)}
        if M <= 128:
            line["gdn_linear_bf16_split_k_us"] = timed(
                lambda i: gdn.linear_bf16(x, ws[i], y, split_k=True), n_sets)
        line["cublas_us"] = timed(lambda i: torch.mm(x, ws[i].t(), out_dtype=torch.float32,
                                                      out=yc), n_sets)
        ours = min(line["gdn_linear_bf16_us"], line.get("gdn_linear_bf16_split_k_us", float("inf")))
        line["ours_tflops"] = 2.0 * M * N * K / ours / 1e6
        line["cublas_tflops"] = 2.0 * M * N * K / line["cublas_us"] / 1e6
        line["ours_over_cublas_time"] = ours / line["cublas_us"]
        line["max_abs_diff"] = float((y - yc).abs().max())
        print(json.dumps(line), flush=True)
    return 0


def run_profile_case(name: str, launches: int) -> int:
    """Run `launches` calls of one case and exit (no timing): the program
    that ncu captures for the summaries kept with the sources."""
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    device = torch.device("cuda", 0)
    launch, _ = build_case(name, device)
    for i in range(launches):
        launch(i)
    torch.cuda.synchronize()
    print(f"ok {name} x{launches}")
    return 0


def bench_layer(steps: int, warmup: int, device):
    import torch
    launch, meta = build_case("layer_decode_b256", device)
    stream = torch.cuda.current_stream(device)
    secs = time_launches(launch, 1, steps, warmup, stream, graph=True)
    return dict(seconds=secs, launches=steps, bytes=layer_bytes(meta["B"]), tokens=meta["B"])


def bench_layer_pair(steps: int, warmup: int, device):
    import torch
    launch, meta = build_case("layer_pair_b256", device)
    stream = torch.cuda.current_stream(device)
    secs = time_launches(launch, 1, steps, warmup, stream, graph=True)
    B = meta["B"]
    return dict(seconds=secs, launches=steps, bytes=layer_pair_bytes(B), tokens=2 * B)


def bench_forward_batch(steps: int, warmup: int, device):
    """The layer over B = 4 x T = 4096 positions with dense bf16 projections
    (D = 2048), graph-replayed; the ring and state advance from call to call."""
    import torch
    launch, meta = build_case("forward_batch_b4_t4096", device)
    B, T, D = meta["B"], meta["T"], meta["D"]
    stream = torch.cuda.current_stream(device)
    secs = time_launches(launch, 1, steps, warmup, stream, graph=True)
    C, HD, Hv = 8192, 4096, 32
    gemm_flops = 2 * B * T * D * (C + HD + 2 * Hv) + 2 * B * T * HD * D
    return dict(seconds=secs, launches=steps, tokens=B * T, gemm_flops=gemm_flops,
                rec_flops=prefill_flops(B, T))


def forward_batch_roofline(fb, seconds: float, peaks, alu_peak: float) -> Dict[str, object]:
    """The stages of the batched forward run one after another, so its ideal
    time is the sum of each stage's own bound: the projection GEMMs at the
    bf16 tensor peak, the recurrence at the FP32 ALU peak, and the conv
    (read + write of the qkv activations), the q/k norms (read + write of q
    and k) and the tail (o and z in, bf16 y out) at the HBM peak."""
    BT, C, HD, QK = fb["tokens"], 8192, 4096, 4096
    hbm_bytes = BT * (2 * C * 4 + 2 * QK * 4 + 2 * HD * 4 + HD * 2)
    parts = {"gemm_ms": fb["gemm_flops"] / (peaks["bf16_tflops"] * 1e12) * 1e3,
             "recurrence_ms": fb["rec_flops"] / (alu_peak * 1e12) * 1e3,
             "elementwise_ms": hbm_bytes / (peaks["hbm_gbs"] * 1e9) * 1e3}
    ideal = sum(parts.values())
    return {"bound": "sum of stage bounds (tensor + alu + hbm)", "ideal_ms": ideal,
            "frac": ideal / (seconds * 1e3), **parts}


def bench_short_conv(name: str, steps: int, warmup: int, device, peaks):
    """One short-conv workload, graph-replayed; HBM roofline for the decode
    and verify launches (weight streaming), tensor roofline for the batch."""
    import torch
    launch, m = build_case(name, device)
    stream = torch.cuda.current_stream(device)
    secs = time_launches(launch, m["sets"], steps, warmup, stream, graph=True)
    per = secs / steps
    B, T, D, K = m["B"], m["T"], m["D"], m["K"]
    r = {"ms_per_launch": per * 1e3, "tokens_per_s": B * T / per,
         "l2": f"rotating {m['sets']} weight sets" if m["sets"] > 1
         else "inputs larger than L2"}
    if T <= 2:
        gbs = short_conv_bytes(B, T, D, K, pair=(name == "short_conv_pair_b64")) / per / 1e9
        r.update(gb_s=gbs, roofline={"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": gbs / peaks["hbm_gbs"]})
    else:
        tf = short_conv_flops(B, T, D) / per / 1e12
        r.update(tflops=tf, roofline={"bound": "tensor", "peak": peaks["bf16_tflops"],
                                      "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"]})
    return r


def bench_pair(steps: int, device, peaks):
    """gdn_pair for 64 sequences (HBM roofline), graph-replayed over two
    input sets."""
    import torch
    stream = torch.cuda.current_stream(device)
    launch, m = build_case("pair_l1_b64", device)
    per = time_launches(launch, 1, steps, 10, stream, graph=True) / steps
    L, B = m["sizes"]["L"], m["sizes"]["B"]
    gbs = pair_bytes(L, B) / per / 1e9
    return {"ms_per_launch": per * 1e3, "layer_tokens_per_s": 2 * L * B / per, "gb_s": gbs,
            "l2": "rotating 2 input sets",
            "roofline": {"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"]}}


def bench_kda(steps_decode: int, steps_prefill: int, device, peaks, alu_peak):
    """The KDA core: the B = 64 decode token (HBM roofline) and the
    4 x 4096-position prefill (fp32 ALU roofline), graph-replayed; the
    prefill's state carries over from launch to launch, which changes no
    work per launch."""
    import torch
    stream = torch.cuda.current_stream(device)
    launch, m = build_case("kda_decode_b64", device)
    per = time_launches(launch, 1, steps_decode, 10, stream, graph=True) / steps_decode
    L, B = m["sizes"]["L"], m["sizes"]["B"]
    gbs = kda_step_bytes(L, B) / per / 1e9
    res = {"kda_decode_b64": {
        "ms_per_launch": per * 1e3, "layer_tokens_per_s": L * B / per, "gb_s": gbs,
        "roofline": {"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"]}}}
    del launch, m
    torch.cuda.empty_cache()
    launch, m = build_case("kda_prefill_b4_t4096", device)
    per = time_launches(launch, 1, steps_prefill, 3, stream, graph=True) / steps_prefill
    B, T = m["sizes"]["B"], m["sizes"]["T"]
    tf = prefill_flops(B, T) / per / 1e12
    res["kda_prefill_b4_t4096"] = {
        "ms_per_launch": per * 1e3, "tokens_per_s": B * T / per, "fp32_tflops": tf,
        "roofline": {"bound": "alu", "peak": alu_peak, "unit": "TFLOP/s", "frac": tf / alu_peak}}
    return res


class OracleDecode:
    """The C oracle's decode entry on one decode workload, with the inputs
    converted once (outside any timing) to the instantiation's type:
    precision "f32" is the literal fp32 instantiation (``gdn_oracle_f32.c``,
    the pages' F32 CPU step), "f64" the double parity oracle. `run(units)`
    advances the listed (layer, sequence, head) units by one token in place;
    calls on disjoint unit lists may run from several threads at once
    (ctypes releases the GIL during the call)."""

    def __init__(self, name: str, precision: str = "f32"):
        import ctypes
        import oracle
        from linear_attention_recurrence_04_b200 import inputs
        w = inputs.WORKLOADS[name]
        d = inputs.decode_inputs(w.sizes["L"], w.sizes["B"], seed=w.seed)
        if precision == "f32":
            lib, ctype, dt = oracle.load_f32().lib, ctypes.c_float, np.float32
            self._fn = lib.oracle_gdn_step_f32
        elif precision == "f64":
            lib, ctype, dt = oracle.load().lib, ctypes.c_double, np.float64
            self._fn = lib.oracle_gdn_step
        else:
            raise ValueError(precision)
        self.precision = precision
        self.a = {k: np.array(v, dtype=dt, order="C") for k, v in d.items()}
        self.out = np.zeros(self.a["v"].shape, dtype=dt)
        self.L, self.B, self.Hv, self.dv, self.dk = self.a["state"].shape
        self.Hk = self.a["q"].shape[2]
        self.total_units = self.L * self.B * self.Hv
        self._pt = ctypes.POINTER(ctype)
        self._pi = ctypes.POINTER(ctypes.c_int64)

    def run(self, units: np.ndarray) -> None:
        u = np.ascontiguousarray(units, dtype=np.int64)
        p = lambda x: x.ctypes.data_as(self._pt)
        a = self.a
        rc = self._fn(p(a["state"]), p(a["q"]), p(a["k"]), p(a["v"]), p(a["beta"]),
                      p(a["gate"]), p(self.out), self.L, self.B, self.Hk, self.Hv, self.dk,
                      self.dv, u.ctypes.data_as(self._pi), int(u.size))
        if rc != 0:
            raise RuntimeError(f"oracle decode entry returned {rc}")


def _label(precision: str) -> str:
    return ("the fp32 instantiation of the C oracle (literal F32 step)" if precision == "f32"
            else "the fp64 C oracle")


def cpu_oracle_baseline(name: str, budget_s: float, max_units: Optional[int] = None,
                        precision: str = "f32"):
    """Time the oracle as it stands, on one thread, over a bounded sample of
    the workload: whole decode steps over the first `units` (layer, sequence,
    head) units, repeated until `budget_s` has elapsed (at least once). The
    inputs are converted once, before timing."""
    od = OracleDecode(name, precision)
    units = np.arange(od.total_units if max_units is None else
                      min(max_units, od.total_units), dtype=np.int64)
    reps, elapsed = 0, 0.0
    while reps == 0 or elapsed < budget_s:
        t0 = time.perf_counter()
        od.run(units)
        elapsed += time.perf_counter() - t0
        reps += 1
    return dict(value=state_gb_s(reps * len(units), elapsed), unit=UNIT, cores=1,
                kind="oracle", precision=precision,
                sample=(f"{reps} pass(es) of {_label(precision)} over {len(units)} of "
                        f"{od.total_units} value-head units of {name}, single thread, inputs "
                        f"converted once before timing, {elapsed:.1f} s"),
                seconds=elapsed, units=int(len(units)), reps=reps)


def cpu_oracle_baseline_parallel(name: str, budget_s: float, precision: str = "f32"):
    """The same oracle entry on every host core this process may use: called
    from one thread per core on disjoint unit lists, over inputs converted
    once and shared. Whole decode steps over all units, repeated until
    `budget_s` has elapsed (at least once); half the budget times the same
    calls on one thread."""
    from concurrent.futures import ThreadPoolExecutor
    od = OracleDecode(name, precision)
    n = max(1, len(os.sched_getaffinity(0)))
    chunks = [c for c in np.array_split(np.arange(od.total_units, dtype=np.int64), n) if c.size]

    def timed(threads, budget):
        reps, elapsed = 0, 0.0
        with ThreadPoolExecutor(threads) as ex:
            while reps == 0 or elapsed < budget:
                t0 = time.perf_counter()
                if threads == 1:
                    for c in chunks:
                        od.run(c)
                else:
                    list(ex.map(od.run, chunks))
                elapsed += time.perf_counter() - t0
                reps += 1
        return reps, elapsed, state_gb_s(reps * od.total_units, elapsed)

    r1, e1, v1 = timed(1, budget_s / 2)
    rn, en, vn = timed(len(chunks), budget_s / 2)
    return dict(value=vn, unit=UNIT, cores=len(chunks), kind="oracle", precision=precision,
                value_one_thread=v1,
                sample=(f"{rn} pass(es) of {_label(precision)} over all {od.total_units} "
                        f"value-head units of {name}, {len(chunks)} threads on disjoint units, "
                        f"inputs converted once and shared, {en:.1f} s; the same calls on one "
                        f"thread: {r1} pass(es), {e1:.1f} s"))


def cpu_oracle_prefill_parallel(budget_s: float, precision: str = "f32"):
    """The oracle's prefill entry on prefill_b4_t4096, parallel over
    (sequence, value head) units: one thread per host core, each running
    whole units through all T positions, over inputs converted once. Repeats
    passes over a sample of one unit per thread until `budget_s` has elapsed
    (at least once); reports tokens/s of the workload (a token is one
    position of one sequence, all 32 heads) and the arithmetic rate."""
    import ctypes
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    from linear_attention_recurrence_04_b200 import inputs
    if precision == "f32":
        fn, ctype, dt = oracle.load_f32().lib.oracle_gdn_prefill_f32, ctypes.c_float, np.float32
    else:
        fn, ctype, dt = oracle.load().lib.oracle_gdn_prefill, ctypes.c_double, np.float64
    w = inputs.WORKLOADS["prefill_b4_t4096"]
    a = {k: np.array(v, dtype=dt, order="C") for k, v in w.draw().items()}
    B, Hv, dv, dk = a["state"].shape
    T, Hk = a["q"].shape[1], a["q"].shape[2]
    n = max(1, min(len(os.sched_getaffinity(0)), B * Hv))
    units = [np.array([u], dtype=np.int64) for u in range(n)]
    states = [a["state"].copy() for _ in range(n)]
    outs = [np.zeros((B, T, Hv, dv), dtype=dt) for _ in range(n)]
    pt, pi = ctypes.POINTER(ctype), ctypes.POINTER(ctypes.c_int64)
    p = lambda x: x.ctypes.data_as(pt)

    def work(j):
        rc = fn(p(states[j]), p(a["q"]), p(a["k"]), p(a["v"]), p(a["beta"]), p(a["gate"]),
                p(outs[j]), B, T, Hk, Hv, dk, dv, units[j].ctypes.data_as(pi), 1)
        if rc != 0:
            raise RuntimeError(f"oracle prefill entry returned {rc}")

    reps, elapsed = 0, 0.0
    with ThreadPoolExecutor(n) as ex:
        while reps == 0 or elapsed < budget_s:
            t0 = time.perf_counter()
            list(ex.map(work, range(n)))
            elapsed += time.perf_counter() - t0
            reps += 1
    unit_positions = reps * n * T
    return dict(value=unit_positions / Hv / elapsed, unit="tokens/s", cores=n, kind="oracle",
                precision=precision,
                gflops=unit_positions * 7 * dk * dv / elapsed / 1e9,
                sample=(f"{reps} pass(es) of {_label(precision)} over {n} of the {B * Hv} "
                        f"(sequence, head) units of prefill_b4_t4096, each through all {T} "
                        f"positions, one unit per thread, {n} threads, {elapsed:.1f} s"))


# --------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------
def config_block() -> Dict[str, object]:
    """The headline workload, identical in both arms."""
    n_sets = _sets_for(step_footprint(1, 64))
    return {"workload": HEADLINE, "L": 1, "B": 64, "Hk": 16, "Hv": 32, "dk": 128, "dv": 128,
            "state_bytes": 64 * 32 * STATE_BYTES_PER_HEAD,
            "l2": f"rotating {n_sets} input sets of {step_footprint(1, 64) / 2**20:.0f} MiB "
                  f"(> 4x the 126 MB L2)",
            "parallelism": "independent batches per rank"}


def run_reference(args) -> int:
    """The oracle as the reference arm: the fp32 instantiation of the C
    oracle's decode step (the pages' F32 CPU path), one host thread, each
    step a bounded sample of the headline workload's units, sized so that
    the whole run stays within about two minutes."""
    env = dist_env()
    if env["rank"] != 0:
        return 0
    n_steps = args.steps + args.warmup
    od = OracleDecode(HEADLINE, "f32")
    probe = np.arange(64, dtype=np.int64)
    t0 = time.perf_counter()
    od.run(probe)
    per_unit = (time.perf_counter() - t0) / probe.size
    units = int(max(1, min(od.total_units, 120.0 / max(n_steps, 1) / per_unit)))
    sel = np.arange(units, dtype=np.int64)
    for _ in range(args.warmup):
        od.run(sel)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        od.run(sel)
    secs = time.perf_counter() - t0
    value = state_gb_s(args.steps * units, secs)
    sample = (f"each step: {_label('f32')} over {units} of {od.total_units} value-head units "
              f"of {HEADLINE}, single thread, inputs converted once before timing")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": env["world"],
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / max(args.steps, 1) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_block(), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args) -> int:
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from linear_attention_recurrence_04_b200 import gdn

    env = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU path)")
    torch.cuda.set_device(env["local_rank"])
    device = torch.device("cuda", env["local_rank"])
    gdn.load_library()
    if env["world"] > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=device)

    def barrier():
        if env["world"] > 1:
            dist.barrier(device_ids=[env["local_rank"]])

    # ---- headline: device-resident gdn_step, B = 64 -------------------
    res = bench_step_workload(HEADLINE, 0, args.warmup, device,
                              seed_offset=rank_seed(0, env["rank"]))
    sets, outs = res["sets"], res["outs"]
    n_sets = res["n_sets"]
    stream = torch.cuda.current_stream(device)

    def launch(i):
        s = sets[i]
        gdn.step(s["state"], s["q"], s["k"], s["v"], s["beta"], s["gate"], outs[i])

    # the K timed launches, captured once into a CUDA graph (no host launch
    # overhead inside the timed region); the same K launches eager, for reference
    graph = capture([(lambda j=j: launch(j % n_sets)) for j in range(args.steps)], device)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(env["local_rank"]) as clocks:
        start.record(stream)
        graph.replay()
        end.record(stream)
        torch.cuda.synchronize()
    barrier()
    secs = max_over_ranks(start.elapsed_time(end) / 1e3, device)
    del graph
    eager_secs = max_over_ranks(time_launches(launch, n_sets, args.steps, 3, stream), device)
    per_launch = secs / max(args.steps, 1)
    value = state_gb_s(res["units"] * args.steps, secs, env["world"])
    tokens_per_s = throughput(res["layer_tokens"] * args.steps, env["world"], secs)
    peaks = measured_peaks()
    achieved = res["bytes"] / per_launch / 1e9
    digest = kernel_source_digest(["gdn_step.cu", "gdn_common.cuh"])

    # ---- end to end through the C ABI with host buffers --------------
    e2e_steps = max(args.steps, 1)
    barrier()
    e2e_secs, e2e_eager_secs, h2d, d2h = bench_e2e(res["d"], e2e_steps, args.warmup, device)
    e2e_secs = max_over_ranks(e2e_secs, device)
    e2e_eager_secs = max_over_ranks(e2e_eager_secs, device)
    e2e_value = state_gb_s(res["units"] * e2e_steps, e2e_secs, env["world"])
    e2e_eager = state_gb_s(res["units"] * e2e_steps, e2e_eager_secs, env["world"])
    del sets, outs, res["sets"], res["outs"]
    torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": env["world"],
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_launch * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded numpy draws: state N(0,0.05^2), unit q/k, v N(0,1), "
                "beta sigmoid(N(0,1)), gate U(-1,0))",
        "config": config_block(),
        "layer_tokens_per_s": tokens_per_s,
        "timing": "CUDA graph of the K launches, replayed once between CUDA events",
        "eager_ms_per_step": eager_secs / max(args.steps, 1) * 1e3,
        "hbm_frac_of_measured": achieved / peaks["hbm_gbs"],
        "hbm_frac_of_8tbs_nominal": achieved / 8000.0,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "peak_source": peaks["source"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "traffic": stored_traffic("gdn_step", digest),
                     "algorithmic_bytes_per_launch": res["bytes"],
                     "kernel": "gdn::step_kernel", "kernel_source_digest": digest},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_secs / e2e_steps * 1e3,
                "timing": "K pipelined steps (pinned copy-in, gdn_step through the C ABI, "
                          "copy-out to pinned memory) captured in one CUDA graph, replayed "
                          "between CUDA events",
                "eager": {"value": e2e_eager, "unit": UNIT,
                          "ms_per_step": e2e_eager_secs / e2e_steps * 1e3,
                          "timing": "the same K steps issued from Python, one ctypes call of "
                                    "gdn_step per step, between CUDA events"}},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }

    if env["world"] == 1 and not args.no_extras:
        extras = {}
        r0 = bench_step_workload("decode_l1_b1", 2000, 50, device)
        extras["decode_l1_b1"] = _step_extra(r0, 2000, peaks)
        del r0
        r2 = bench_step_workload("decode_l36_b16", 20, 3, device)
        extras["decode_l36_b16"] = _step_extra(r2, 20, peaks)
        del r2
        torch.cuda.empty_cache()
        extras["pair_l1_b64"] = bench_pair(400, device, peaks)
        torch.cuda.empty_cache()
        p = bench_prefill(5, 3, device)
        alu_peak = 148 * 128 * 2 * (line["clocks"]["sm_max_mhz"] or 1965) * 1e6 / 1e12
        extras["prefill_b4_t4096"] = {
            "ms_per_launch": p["seconds"] / p["launches"] * 1e3,
            "tokens_per_s": p["tokens"] * p["launches"] / p["seconds"],
            "gb_s": p["bytes"] * p["launches"] / p["seconds"] / 1e9,
            "fp32_tflops": p["flops"] * p["launches"] / p["seconds"] / 1e12,
            "roofline": {"bound": "alu", "peak": alu_peak, "unit": "TFLOP/s",
                         "frac": p["flops"] * p["launches"] / p["seconds"] / 1e12 / alu_peak},
        }
        torch.cuda.empty_cache()
        lay = bench_layer(20, 3, device)
        gbs = lay["bytes"] * lay["launches"] / lay["seconds"] / 1e9
        extras["layer_decode_b256"] = {
            "ms_per_launch": lay["seconds"] / lay["launches"] * 1e3,
            "layer_tokens_per_s": lay["tokens"] * lay["launches"] / lay["seconds"],
            "gb_s": gbs, "roofline": {"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                      "frac": gbs / peaks["hbm_gbs"]},
        }
        pr = bench_layer_pair(20, 3, device)
        gbs = pr["bytes"] * pr["launches"] / pr["seconds"] / 1e9
        extras["layer_pair_b256"] = {
            "ms_per_launch": pr["seconds"] / pr["launches"] * 1e3,
            "layer_tokens_per_s": pr["tokens"] * pr["launches"] / pr["seconds"],
            "gb_s": gbs, "roofline": {"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                      "frac": gbs / peaks["hbm_gbs"]},
        }
        torch.cuda.empty_cache()
        fb = bench_forward_batch(5, 2, device)
        per = fb["seconds"] / fb["launches"]
        extras["forward_batch_b4_t4096"] = {
            "ms_per_launch": per * 1e3,
            "tokens_per_s": fb["tokens"] / per,
            "projection_tflops": fb["gemm_flops"] / per / 1e12,
            "roofline": forward_batch_roofline(fb, per, peaks, alu_peak),
            "note": "D=2048 bf16 projections on tcgen05 + conv + sequential recurrence + tail",
        }
        torch.cuda.empty_cache()
        for name in ("short_conv_decode_b64", "short_conv_pair_b64"):
            extras[name] = bench_short_conv(name, 200, 10, device, peaks)
        extras["short_conv_batch_b4_t4096"] = bench_short_conv("short_conv_batch_b4_t4096", 10, 3,
                                                               device, peaks)
        torch.cuda.empty_cache()
        extras.update(bench_kda(200, 5, device, peaks, alu_peak))
        line["workloads"] = extras

    if env["rank"] == 0 and env["world"] == 1 and not args.no_cpu_baseline:
        budget = args.cpu_budget
        cb = cpu_oracle_baseline(HEADLINE, budget / 2, precision="f32")
        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        # the same instantiation on every host core (independent units, no exchange)
        line["cpu_baseline_all_cores"] = cpu_oracle_baseline_parallel(HEADLINE, budget / 2,
                                                                      precision="f32")
        # the double parity oracle, for reference
        c64 = cpu_oracle_baseline(HEADLINE, budget / 4, precision="f64")
        line["cpu_baseline_fp64"] = {
            "one_thread": {k: c64[k] for k in ("value", "unit", "cores", "sample")},
            "all_cores": cpu_oracle_baseline_parallel(HEADLINE, budget / 4, precision="f64")}
        if "prefill_b4_t4096" in line.get("workloads", {}):
            line["workloads"]["prefill_b4_t4096"]["cpu_baseline_all_cores"] = \
                cpu_oracle_prefill_parallel(budget / 3, precision="f32")

    if env["world"] > 1:
        barrier()
        dist.destroy_process_group()
    if env["rank"] == 0:
        print(json.dumps(line), flush=True)
    return 0


def _step_extra(r, steps, peaks):
    per = r["seconds"] / steps
    gbs = r["bytes"] / per / 1e9
    return {"ms_per_launch": per * 1e3, "state_gb_s": state_gb_s(r["units"], per),
            "layer_tokens_per_s": r["layer_tokens"] / per, "gb_s": gbs,
            "roofline": {"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"]},
            "l2": f"rotating {r['n_sets']} input sets"}


def launcher_command(argv: List[str], n_gpus: int, port: int) -> List[str]:
    """torchrun command that starts one rank of this script per GPU."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n_gpus}", "--master-addr", "127.0.0.1",
            "--master-port", str(port), os.path.abspath(__file__), *argv]


def world_mismatch(gpus: int, environ) -> Optional[str]:
    """Why `--gpus` and the launcher's WORLD_SIZE disagree, or None."""
    world = int(environ.get("WORLD_SIZE", 1))
    if world != gpus:
        return (f"--gpus {gpus} but this process is one of WORLD_SIZE={world} ranks: run "
                f"`bench.py --gpus N` without a launcher (it starts N ranks itself) or "
                f"under torchrun with --nproc-per-node N")
    return None


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of CPU time for the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=PROFILE_CASES, default=None,
                    help="run --launches calls of one case without timing (for ncu) and exit")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--cublas-compare", action="store_true",
                    help="time the projection kernels against cuBLAS on the layer's shapes and exit")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other four workloads (headline only)")
    args = ap.parse_args(argv)
    if args.profile_case:
        return run_profile_case(args.profile_case, args.launches)
    if args.cublas_compare:
        return run_cublas_compare()
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # not under a launcher: one rank per GPU, started here
        import socket
        import subprocess
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        argv = sys.argv[1:] if argv is None else list(argv)
        return subprocess.call(launcher_command(argv, args.gpus, port))
    why = world_mismatch(args.gpus, os.environ)
    if why:
        ap.error(why)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
