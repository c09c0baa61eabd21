"""attn_merge_lse on the GPU: results over disjoint key ranges, computed by
the library's kernels and merged by its merge kernel, against the fp64
oracle over all keys (needs a B200)."""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_helpers import (ATOL_LSE, ATOL_OUT, BF16_NAN_BITS, compare_full, covered_rows, oracle_full, plan_for,
                         sentinel_lse, sentinel_out)
import varlen_gqa_split_b200 as vg
from varlen_gqa_split_b200 import context_parallel as cp

pytestmark = pytest.mark.gpu

SIMT, MMA, TC = vg.ATTN_VARIANT_SIMT, vg.ATTN_VARIANT_MMA, vg.ATTN_VARIANT_TC


@pytest.fixture(scope="module", autouse=True)
def _built():
    from varlen_gqa_split_b200 import build
    build.build()
    torch.cuda.init()


def _parts(plan, batch, n):
    q = batch.q.cuda()
    k, v = batch.k.cuda(), batch.v.cuda()
    cu_q = torch.from_numpy(batch.cu_q).cuda()
    cu_k = torch.from_numpy(batch.cu_k).cuda()
    outs, lses = [], []
    for r in range(n):
        k_r, v_r, cu_r = cp.shard_kv(k, v, cu_k, r, n)
        o, l = plan.run(q, k_r, v_r, cu_q, cu_r)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    assert plan.check_error() == 0
    return torch.stack(outs).contiguous(), torch.stack(lses).contiguous(), cu_q


@pytest.mark.parametrize("n", [1, 2, 3, 8])
@pytest.mark.parametrize("variant,D", [(MMA, 128), (SIMT, 64), (TC, 128)])
def test_merged_key_ranges_equal_the_whole(n, variant, D):
    sh = W.Shape("cp", B=7, Hq=16, Hkv=2, D=D, max_q=1, s_max=3000)
    lk = [3000, 5, 0, 1, 64, 129, 2047]
    batch = W.make_batch(sh, [1] * sh.B, lk, seed=5, gen_device="cuda")
    plan = plan_for(sh, variant=variant)
    outs, lses, cu_q = _parts(plan, batch, n)
    T = outs.shape[1] + 3                           # rows past cu_q[B_max] stay untouched
    out = sentinel_out(T, sh.Hq, sh.D)
    lse = sentinel_lse(T, sh.Hq)
    pad_o = torch.zeros(n, T, sh.Hq, sh.D, dtype=torch.bfloat16, device="cuda")
    pad_l = torch.zeros(n, T, sh.Hq, dtype=torch.float32, device="cuda")
    pad_o[:, :outs.shape[1]] = outs
    pad_l[:, :outs.shape[1]] = lses
    vg.merge_lse(pad_o, pad_l, cu_q, out=out, lse=lse)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_full(batch)
    cov = np.zeros(T, dtype=bool)
    cov[: int(batch.cu_q[-1])] = True
    ro = np.zeros((T, sh.Hq, sh.D))
    rl = np.zeros((T, sh.Hq))
    ro[: ref_o.shape[0]] = ref_o
    rl[: ref_l.shape[0]] = ref_l
    compare_full(out.cpu(), lse.cpu(), ro, rl, cov)


def test_one_part_passes_through_unchanged():
    sh = W.Shape("cp1", B=3, Hq=8, Hkv=1, D=128, max_q=1, s_max=700)
    batch = W.make_batch(sh, [1, 1, 1], [700, 0, 33], seed=9, gen_device="cuda")
    plan = plan_for(sh)
    outs, lses, cu_q = _parts(plan, batch, 1)
    out, lse = vg.merge_lse(outs, lses, cu_q)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), outs[0].view(torch.int16))
    fin = torch.isfinite(lses[0])
    assert torch.equal(torch.isneginf(lse), torch.isneginf(lses[0]))
    assert (lse[fin] - lses[0][fin]).abs().max().item() < 1e-6


def test_merge_rejects_bad_arguments():
    lib = vg.lib()
    t = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(64, dtype=torch.float32, device="cuda")
    cu = torch.zeros(2, dtype=torch.int32, device="cuda")
    args = dict(outs=t.data_ptr(), lses=f.data_ptr(), cu=cu.data_ptr(), out=t.data_ptr(), lse=f.data_ptr())

    def call(n=2, T=2, B=1, Hq=4, D=128, **kw):
        a = dict(args, **kw)
        return lib.attn_merge_lse(n, a["outs"], a["lses"], T, a["cu"], B, Hq, D, a["out"], a["lse"], None)

    assert call() == 0
    assert call(D=96) == -2                 # head dim
    assert call(n=0) == -1
    assert call(outs=None) == -3
    assert call(outs=t.data_ptr() + 2) == -4
    torch.cuda.synchronize()
