"""The multi-GPU bench path (independent replicas, one per rank) on CPU:
world-size-2 gloo ranks check the max-over-ranks timing and the whole-job
throughput, and that the reference arm runs on rank 0 only and prints one
contract line."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank(rank, world, port, times, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _load_bench()
        t = b.max_over_ranks(times[rank], "cpu")
        out[rank] = (t, b.job_throughput(32, 200, world, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world, times = 2, [17.5, 23.25]
    port = 29500 + os.getpid() % 1000
    with mp.get_context("spawn").Manager() as m:   # no fork of a threaded process
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, times, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == max(times)
    # 2 replicas x 32 sequences x 200 steps in the slowest replica's 23.25 ms
    assert res[0][1] == pytest.approx(2 * 32 * 200 / 0.02325)


def test_single_process_needs_no_process_group():
    b = _load_bench()
    assert b.max_over_ranks(4.0, "cpu") == 4.0
    assert b.job_throughput(8, 10, 1, 2.0) == pytest.approx(40000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_contract_line():
    """The reference arm alone (one process): one JSON line with the same
    metric, unit and workload as the library's arm, the oracle's timing as
    its value, a cpu_baseline describing that run and an e2e with no host
    copies."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["unit"] == "tok/s" and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"] == "csa_decode_128k_b32" and d["config"]["batch"] == 32
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
