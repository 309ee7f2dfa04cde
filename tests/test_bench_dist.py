"""The multi-process path of bench.py on the CPU: gloo ranks, world size 2.

bench.py runs one process per GPU; every rank processes its own batch (no
data-path collective) and the step time is the slowest rank's. These tests
run the rank reduction and the whole-job rate with real gloo process groups,
and check that the reference arm leaves ranks other than 0 without work.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(times[rank])
        out.put((rank, t, bench.whole_job_rate(1000, world, t)))
    finally:
        dist.destroy_process_group()


def _run_ranks(times):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    world = len(times)
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_step_time_is_the_slowest_rank_and_rate_counts_all_ranks():
    res = _run_ranks([0.5, 2.0])
    for rank, t, rate in res:
        assert t == 2.0, (rank, t)
        assert rate == pytest.approx(1000 * 2 / 2.0)


def test_reduction_is_order_independent():
    res = _run_ranks([3.0, 1.0])
    assert [t for _, t, _ in res] == [3.0, 3.0]


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25) == 1.25
    assert bench.whole_job_rate(32768, 1, 0.5) == 65536


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_keeps_the_contract():
    """Rank 0 of the reference arm (the fp64 oracle on the host cores) prints
    one JSON line with the bench contract's keys, the same metric, unit and
    config as the GPU arm, impl "reference", a cpu_baseline describing the
    run and an e2e object with no host copies."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--cpu-seconds", "2"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"] == bench._reference_config()
    assert d["config"] == bench.workload_config(1, 32, 8, 32768, 128)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
