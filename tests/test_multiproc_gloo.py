"""The multi-rank path of bench.py on CPU: two gloo ranks exercise the host logic
that a multi-GPU run uses (per-rank batches, the max-over-ranks time, the
whole-job rate), and the reference arm's rank-0-only rule.  No GPU needed."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        t = bench.max_over_ranks(local_ms, dist, "cpu")
        x = np.arange(12, dtype=np.uint16).reshape(6, 2)
        b = bench.rank_batch(x, rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, b.tolist())
        out[rank] = (t, bench.whole_job_rate(1e9, world, t), gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_batches():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        t, rate, gathered = res[rank]
        assert t == 15.0                                  # the max of 10 ms and 15 ms on every rank
        assert rate == pytest.approx(2 * 1e9 / 15e-3)     # both ranks' units over the slowest time
        assert gathered[0] != gathered[1]                 # each rank has its own batch
        assert sorted(map(tuple, gathered[0])) == sorted(map(tuple, gathered[1]))


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_json_line():
    """Rank 0 of the reference arm prints one JSON line with the contract's keys, its
    cpu_baseline describing the run and an e2e block with no host-device bytes."""
    import json
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config"):
        assert k in d, k
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["config"]["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
