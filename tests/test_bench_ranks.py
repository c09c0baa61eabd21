"""bench.py's multi-rank logic on CPU: two gloo ranks (world size 2).

The ranks run independent replicas; the only exchanges are the barrier and
the max of the ranks' timed totals, which every rank must agree on.  The
reference arm prints from rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    r, w, _, pg = bench.dist_setup(world, backend="gloo")
    try:
        bench.barrier(pg)
        mx = bench.max_over_ranks(10.0 + 5.0 * r, pg)       # rank-dependent "timed total"
        passes = bench.max_over_ranks_vec([1.0 + r, 5.0 - r, 3.0], pg)   # per-pass times, element-wise
        bench.barrier(pg)
        q.put((r, w, mx, tuple(passes)))
    finally:
        pg.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_agree_on_the_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 2, 15.0, (2.0, 5.0, 3.0)), (1, 2, 15.0, (2.0, 5.0, 3.0))]


def test_world_size_must_match_gpus(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.dist_setup(1, backend="gloo")


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_from_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), VGQA_REF_BUDGET_S="2")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--workload", "tiny",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 1:
        assert lines == []
    else:
        res = json.loads(lines[-1])
        assert res["impl"] == "reference" and res["value"] > 0
        assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["cpu_baseline"]["kind"] == "oracle"
