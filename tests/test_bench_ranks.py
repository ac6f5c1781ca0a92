"""The multi-rank plumbing of bench.py (one process per GPU, launched by
torch.distributed.run; here two CPU ranks over gloo): every rank joins the
barrier, and the timed region's device times reduce to their element-wise
maximum over ranks, which every rank then holds."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.rank_env()
    dev = torch.device("cpu")
    bench.init_ranks(w, dev, backend="gloo")
    bench.barrier(w)
    got = bench.max_over_ranks([1.0 + r, 10.0 - r, 0.5 * r], w, dev)
    bench.close_ranks(w)
    q.put((r, got))


def test_max_over_ranks_with_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = dict(q.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
    assert res[0] == res[1] == [2.0, 10.0, 0.5]
    assert all(p.exitcode == 0 for p in procs)


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    w, r, local = bench.rank_env()
    assert (w, r, local) == (1, 0, 0)
    bench.init_ranks(w, torch.device("cpu"))  # no process group for one rank
    bench.barrier(w)
    assert bench.max_over_ranks([3.0, 4.0], w, torch.device("cpu")) == [3.0, 4.0]
    bench.close_ranks(w)


def test_gpus_flag_starts_one_rank_per_gpu():
    """`bench.py --gpus 2` with no launcher environment starts two ranks under
    torch.distributed.run itself; both join and rank 0 reports n_gpus 2."""
    import json
    import subprocess
    import sys

    import bench
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    res = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--gpus", "2", "--check-ranks"],
                         capture_output=True, text=True, timeout=300, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["ranks_joined"] == 2
    cmd = bench.spawn_command(4, ["--steps", "3"])
    assert "--nproc-per-node=4" in cmd and cmd[-2:] == ["--steps", "3"] and "127.0.0.1" in cmd
