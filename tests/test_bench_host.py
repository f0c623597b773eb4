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
                        "--gpus", "2", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=120)
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
    assert line["config"] == bench.config_block()      # the same workload as the GPU arm


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
    assert pre["unit"] == "tokens/s" and pre["value"] > 0 and pre["gflops"] > 0
    assert 1 <= pre["cores"] <= len(os.sched_getaffinity(0))
    f64 = bench.cpu_oracle_baseline(bench.HEADLINE, 0.0, max_units=16, precision="f64")
    assert f64["precision"] == "f64" and f64["value"] > 0


def test_state_bandwidth_counts_read_and_write_in_every_arm():
    """The headline metric counts each head's 64 KiB state read once and
    written once per token. The GPU arm, the end-to-end leg, the CPU
    baselines and the reference arm all go through state_gb_s."""
    assert bench.state_rw_bytes(1, 64) == 2 * 134_217_728
    assert bench.state_rw_bytes(36, 16) == 2 * 1_207_959_552
    assert bench.state_gb_s(64 * 32, 1e-3) == pytest.approx(bench.state_rw_bytes(1, 64) / 1e-3 / 1e9)
    assert bench.state_gb_s(2048, 2.0, n_ranks=4) == pytest.approx(4 * bench.state_gb_s(2048, 2.0))
    one = bench.cpu_oracle_baseline(bench.HEADLINE, 0.0, max_units=8)
    expect = one["reps"] * one["units"] * 2 * 128 * 128 * 4 / one["seconds"] / 1e9
    assert one["value"] == pytest.approx(expect)
    src = open(os.path.join(ROOT, "bench.py")).read()
    # no figure of the metric is formed from the one-way state size
    assert "state_bytes\"] * " not in src and "STATE_BYTES_PER_HEAD * 2" not in src


def test_fp32_oracle_instantiation_matches_the_parity_oracle():
    """The timed CPU baseline's fp32 instantiation agrees with the fp64
    oracle within the library tolerance on the headline workload."""
    import oracle
    from linear_attention_recurrence_04_b200 import inputs
    from parity import assert_parity
    d = inputs.WORKLOADS[bench.HEADLINE].draw()
    args = (d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    s64, o64 = oracle.load().step(*args)
    s32, o32 = oracle.load_f32().step(*args)
    assert_parity(o32, o64, "fp32 oracle out")
    assert_parity(s32, s64, "fp32 oracle state")
    p = inputs.prefill_inputs(2, 200, seed=71, state_std=0.05)
    pargs = (p["state"], p["q"], p["k"], p["v"], p["beta"], p["gate"])
    s64, o64 = oracle.load().prefill(*pargs)
    s32, o32 = oracle.load_f32().prefill(*pargs)
    assert_parity(o32, o64, "fp32 oracle prefill out")
    assert_parity(s32, s64, "fp32 oracle prefill state")


def test_gpus_flag_must_match_the_launcher():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--impl", "reference", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 2 and "WORLD_SIZE=1" in r.stderr
    assert bench.world_mismatch(4, {"WORLD_SIZE": "4"}) is None
    assert bench.world_mismatch(1, {}) is None
    assert "WORLD_SIZE=2" in bench.world_mismatch(8, {"WORLD_SIZE": "2"})


def test_launcher_command_starts_one_rank_per_gpu():
    cmd = bench.launcher_command(["--gpus", "4", "--steps", "5"], 4, 29500)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "29500" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"] and cmd[-5].endswith("bench.py")
