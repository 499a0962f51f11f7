"""The multi-GPU (N > 1) host logic of bench.py on CPU: two gloo ranks, each
timing its own replica of the workload, agree on the slowest rank's time and
on the whole-job value; the reference arm runs on rank 0 only."""

import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(my_ms, dist, "cpu")
        v = bench.whole_job_value(world, 1_638_400, 100, ms * 1e-3, 1e-9)
        out[rank] = (ms, v)
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_max_and_value():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    ms, v = res[0]
    assert ms == 5.0
    assert v == pytest.approx(2 * 1_638_400 * 100 / 5e-3 * 1e-9)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "1"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_matches_our_arm():
    """Rank 0 of the reference arm prints one JSON line carrying the contract's
    keys, the same metric and workload identity as our arm, and its own
    description as cpu_baseline and e2e (no host<->device bytes)."""
    import json
    import bench
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1"], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["warmup"] >= 3 and d["steps"] == 1 and d["n_gpus"] == 1
    ident = bench.workload_identity("decode")
    assert {k: d["config"][k] for k in ident} == ident
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
