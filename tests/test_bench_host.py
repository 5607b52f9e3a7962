"""Host logic of bench.py on the CPU: the N-rank timing reduction (max over ranks, gloo with
two ranks) and the all-rank agreement on retaking a clock-rejected timing region, the
reference arm's rank-0-only rule, and the clock-sample rejection rules."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, values, out_q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    got = bench.max_over_ranks(values[rank], dist, torch, "cpu")
    # a clock rejection seen on one rank only: both ranks retake the timing region
    agree = bench.any_over_ranks(rank == 1, dist, torch, "cpu")
    none = bench.any_over_ranks(False, dist, torch, "cpu")
    dist.barrier()
    out_q.put((rank, (got, agree, none)))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    values = [12.5, 40.25]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: (40.25, True, False), 1: (40.25, True, False)}


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, torch, "cpu") == 3.5


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_bench_rejects_short_warmup():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "1"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0


def _sampler(samples, max_mhz=1965):
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.samples = samples
    c.max_mhz = max_mhz
    return c


def test_clock_rules():
    ok = _sampler([(1800, 0x0, 900.0), (1750, 0x4, 1000.0)])
    assert not ok.rejected()
    assert ok.summary()["reasons"] == ["sw_power_cap"]
    assert _sampler([(1800, 0x8, 900.0)]).rejected()           # hw_slowdown
    assert _sampler([(1800, 0x40, 900.0)]).rejected()          # hw thermal
    assert _sampler([(1800, 0x20, 900.0)]).rejected()          # sw thermal
    assert _sampler([(900, 0x0, 300.0), (900, 0x0, 300.0)]).rejected()   # stuck low, no reason
    assert not _sampler([(900, 0x4, 1000.0)]).rejected()       # low under the power cap: kept
    assert _sampler([]).summary()["reasons"] == ["unavailable"]


def test_reference_arm_json_line_cpu():
    """The reference arm (the oracle on the host cores) prints one JSON line of the contract."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--workload", "small_4k",
                        "--ref-step-seconds", "1"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in line
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_backward_times_the_oracle_gradients():
    """For a backward workload the reference arm times the oracle's gradients (a one-head
    causal sample) under the workload's backward name."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--workload", "llama8b_32k_bwd",
                        "--ref-step-seconds", "1"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"]["workload"].endswith("_backward")
    assert "gradients" in line["cpu_baseline"]["sample"]


def test_multi_gpu_step_splits_heads_or_falls_back():
    """bench --gpus N runs the Ulysses step across N GPUs when the workload's query heads
    and sequence divide over N (the driver's 1, 2, 4, 8), otherwise independent replicas."""
    import bench
    from sequence_parallelism_attn_b200 import synth
    w = synth.ULYSSES_128K
    assert [n for n in (1, 2, 3, 4, 5, 8, 16) if bench.DistUlyssesPath.splits(w, n)] == \
        [1, 2, 4, 8, 16]
    # the hybrid workload (head groups fewer than ranks) keeps replicas
    assert not bench.DistUlyssesPath.splits(synth.USP_128K, 2)
