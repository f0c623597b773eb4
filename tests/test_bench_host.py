"""Host-side logic of bench.py, without a GPU: the N > 1 path with two gloo
ranks on the CPU (max over ranks, weak-scaling throughput, per-rank seeds),
the reference arm's rank handling, and the roofline bookkeeping."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        env = bench.dist_env()
        t = bench.max_over_ranks(0.5 + rank)              # rank 1 is the slow one
        v = bench.throughput(100.0, env["world"], t)
        q.put((rank, env, t, v, bench.rank_seed(1001, rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, env0, t0, v0, s0), (r1, env1, t1, v1, s1) = results
    assert env0["world"] == env1["world"] == 2 and env1["rank"] == 1
    assert t0 == t1 == 1.5                                 # both see the slowest rank
    assert v0 == v1 == pytest.approx(2 * 100.0 / 1.5)     # all ranks' units / max time
    assert s0 != s1                                        # each rank draws its own batch


def test_max_over_ranks_without_group_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_algorithmic_bytes():
    # per value-head token: 2 x 64 KiB state + v + out + beta + gate, q/k per key head
    assert bench.step_bytes(1, 1) == 32 * (131072 + 1024 + 8) + 16 * 1024
    assert bench.step_bytes(1, 64) == 271_597_568
    assert bench.step_bytes(36, 16) == 2_444_378_112
    assert bench.prefill_bytes(4, 4096) == 826_277_888
    assert bench.prefill_flops(4, 4096) == 60_129_542_144
    assert bench.layer_bytes(256) == 1_141_048_064


def test_clock_reason_decoding():
    assert bench.decode_reasons(0x4 | 0x40) == ["sw_power_cap", "hw_thermal_slowdown"]
    assert bench.decode_reasons(0) == []


def test_traffic_record_tracks_the_kernel_source():
    dig = bench.kernel_source_digest(["gdn_step.cu", "gdn_common.cuh"])
    assert bench.stored_traffic("gdn_step", "not-the-digest") is None
    t = bench.stored_traffic("gdn_step", dig)
    assert t is None or t > 1e8


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["metric"] == bench.METRIC and line["steps"] == 3
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_cpu_baselines_time_the_oracle():
    """One pass each: the single-thread leg and the all-cores leg (the oracle's
    C entry on disjoint units from one thread per core) both report the state
    bandwidth of the headline workload."""
    one = bench.cpu_oracle_baseline(bench.HEADLINE, 0.0, max_units=64)
    assert one["cores"] == 1 and one["kind"] == "oracle" and one["value"] > 0
    allc = bench.cpu_oracle_baseline_parallel(bench.HEADLINE, 0.0)
    assert allc["kind"] == "oracle" and allc["unit"] == bench.UNIT
    assert 1 <= allc["cores"] <= len(os.sched_getaffinity(0))
    assert allc["value"] > 0 and allc["value_one_thread"] > 0
    pre = bench.cpu_oracle_prefill_parallel(0.0)
    assert pre["unit"] == "tokens/s" and pre["value"] > 0 and pre["fp64_gflops"] > 0
    assert 1 <= pre["cores"] <= len(os.sched_getaffinity(0))
