"""Context-parallel decode: the exchange logic over two and three gloo ranks on
CPU.

Each rank shards every sequence's keys (varlen_gqa_split_b200.context_parallel),
attends over its shard and joins the all-gather of the (out, lse) pairs; the
merged result must equal attention over all keys.  The local attention and
the merge are the fp64 oracle's here (no GPU on this machine); the GPU suite
runs the library's kernels for both."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _batch():
    sys.path.insert(0, ROOT)
    import workloads as W
    sh = W.Shape("cp", B=6, Hq=8, Hkv=2, D=64, max_q=1, s_max=500)
    lk = [500, 3, 0, 1, 64, 129]
    return sh, W.make_batch(sh, [1] * sh.B, lk, seed=21)


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    import workloads as W
    from varlen_gqa_split_b200 import context_parallel as cp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sh, batch = _batch()
        cu_k = torch.from_numpy(batch.cu_k)
        cu_q = torch.from_numpy(batch.cu_q)
        k_loc, v_loc, cu_loc = cp.shard_kv(batch.k, batch.v, cu_k, rank, world)

        def attend(q_, k_, v_, cq, ck):
            o, l = oracle.attention(W.bits(q_), W.bits(k_), W.bits(v_), cq.numpy(), ck.numpy(), B=sh.B, Hq=sh.Hq,
                                    Hkv=sh.Hkv, D=sh.D)
            return torch.from_numpy(o), torch.from_numpy(l)

        def merge(outs, lses, cq):
            o, l = oracle.merge_lse(outs.numpy(), lses.numpy())
            return torch.from_numpy(o), torch.from_numpy(l)

        out, lse = cp.decode_step(None, batch.q, k_loc, v_loc, cu_q, cu_loc, attend=attend, merge=merge)
        q.put((rank, int(k_loc.shape[0]), out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_decode_over_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    import oracle
    import workloads as W
    sh, batch = _batch()
    ref_o, ref_l = oracle.attention(W.bits(batch.q), W.bits(batch.k), W.bits(batch.v), batch.cu_q, batch.cu_k,
                                    B=sh.B, Hq=sh.Hq, Hkv=sh.Hkv, D=sh.D)
    assert sum(g[1] for g in got) == int(batch.cu_k[-1])           # the shards tile the keys
    for _, _, o, l in got:                                          # every rank holds the merged result
        assert np.abs(o - ref_o).max() < 1e-12
        assert np.array_equal(np.isneginf(l), np.isneginf(ref_l))
        fin = np.isfinite(ref_l)
        assert np.abs(l[fin] - ref_l[fin]).max() < 1e-12


def test_shard_bounds_tile_each_sequence_in_rank_order():
    sys.path.insert(0, ROOT)
    from varlen_gqa_split_b200.context_parallel import shard_bounds
    cu = torch.tensor([0, 10, 10, 13, 1000], dtype=torch.int32)
    for world in (1, 2, 3, 8):
        prev_hi = cu[:-1].to(torch.int64)
        for r in range(world):
            lo, hi = shard_bounds(cu, r, world)
            assert torch.equal(lo, prev_hi)
            assert bool((hi >= lo).all())
            prev_hi = hi
        assert torch.equal(prev_hi, cu[1:].to(torch.int64))
