"""Host logic of bench.py for N > 1 ranks, on CPU with the gloo backend.

The path has no collective: ranks run independent replicas of the decode step
and only the timing is combined (max over ranks). These tests run two gloo ranks
as child processes on 127.0.0.1."""
import os
import time
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
torch = pytest.importorskip("torch")
import bench  # noqa: E402

WORKER = r'''
import datetime, os, sys
sys.path.insert(0, os.environ["ROOT"])
import torch.distributed as dist
import bench
dist.init_process_group("gloo", rank=int(os.environ["RANK"]), world_size=2,
                        timeout=datetime.timedelta(seconds=60))
rank = dist.get_rank()
ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")   # rank 1 is the slow one
value = bench.replica_throughput(100, dist.get_world_size(), ms)
dist.barrier()
print(f"rank={rank} ms={ms} value={value}", flush=True)
dist.destroy_process_group()
'''


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_agree_on_the_max_time():
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, ROOT=ROOT, RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(out.strip())
    # both ranks see the slower replica's time; 2 x 100 tokens in 15 ms
    assert outs[0] == "rank=0 ms=15.0 value=13333.333333333334"
    assert outs[1] == "rank=1 ms=15.0 value=13333.333333333334"


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.replica_throughput(1, 1, 2.0) == 500.0


def test_reference_arm_on_a_nonzero_rank_does_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line_with_the_contract_keys():
    import json
    t0 = time.time()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "7",
                        "--warmup", "3", "--ref-budget", "6"], env=dict(os.environ, RANK="0", WORLD_SIZE="1"),
                       capture_output=True, text=True, timeout=600)
    wall = time.time() - t0
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["metric"] == bench.METRIC
    # the line describes what was timed: its steps fit the run, and it names the GPU arm's workload
    assert d["ms_per_step"] * d["steps"] / 1e3 <= wall
    wl = bench.synth.full_step(n_layers=32)
    assert d["config"] == bench.step_config(wl, 32, 1, 1)


def test_bench_refuses_fewer_than_three_warmup_steps():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                       text=True, timeout=120)
    assert r.returncode != 0 and "warmup" in r.stderr
