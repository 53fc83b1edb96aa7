"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The decode step shards trivially: every rank runs its own replica of the
workload, with no collective on the data path.  What crosses ranks is the
timing (max over ranks) and the barriers around the timed region; the
reference arm runs on rank 0 alone.  These tests run that logic as real
ranks on 127.0.0.1 without a GPU.
"""

import json
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, loc = bench._dist()
    bench._init_pg(w, "gloo")
    bench._barrier(w)
    m = bench._max_over_ranks(float(10 * (rank + 1)), w, torch.device("cpu"))
    bench._barrier(w)
    q.put((r, loc, w, m))
    dist.destroy_process_group()


def test_dist_env_defaults(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench._dist() == (1, 0, 0)
    assert bench._max_over_ranks(3.5, 1, None) == 3.5      # no process group at N = 1
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "3")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench._dist() == (4, 3, 1)


def test_max_over_ranks_and_barriers_world_size_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == [0, 1]
    assert [g[1] for g in got] == [0, 1]
    assert all(g[2] == 2 for g in got)
    assert all(g[3] == 20.0 for g in got)      # every rank reports the slowest rank's time


def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched like the multi-GPU bench: rank 0
    prints exactly one JSON line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--ref-budget-s", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["metric"] == "fused 3-bit logits HBM GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_percentiles_nearest_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench._percentiles(range(1, 11)) == {"p10": 1, "p50": 5, "p90": 9, "n": 10}
    assert bench._percentiles([2.5]) == {"p10": 2.5, "p50": 2.5, "p90": 2.5, "n": 1}
    s = bench._percentiles([4, 1, 3, 2])
    assert (s["p10"], s["p50"], s["p90"]) == (1, 2, 4)
