"""Paged K/V cache (attn_run_paged) vs the fp64 oracle (needs a B200).

The keys and values of a packed batch are scattered into a paged cache with
a shuffled page order; every slot no key uses holds NaN and every block-table
entry past a sequence's pages holds an invalid index, so a kernel that lets a
stale slot into its result, or reads a table entry it should not, fails.  The
oracle runs on the packed bytes of the same batch.
"""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_helpers import (ATOL_LSE, ATOL_OUT, check_values, compare_full, covered_rows, oracle_full, plan_for, sample_rows,
                         sentinel_lse, sentinel_out)
import varlen_gqa_split_b200 as vg

pytestmark = pytest.mark.gpu

SIMT, MMA, TC = vg.ATTN_VARIANT_SIMT, vg.ATTN_VARIANT_MMA, vg.ATTN_VARIANT_TC


@pytest.fixture(scope="module", autouse=True)
def _built():
    from varlen_gqa_split_b200 import build
    build.build()
    torch.cuda.init()


def _edge_batch(Hq, max_q, s_max=600, seed=31):
    """Lengths around page and tile edges, zero and full, plus random ones."""
    Hkv, D = 4, 128
    lk = [0, 1, 7, 8, 9, 63, 64, 65, 127, 128, 129, s_max, 300, 511]
    rng = np.random.default_rng(seed)
    lk = np.array(lk + list(rng.integers(0, s_max, 6)), dtype=np.int64)
    lq = rng.integers(1, max_q, lk.size, endpoint=True)
    lq = np.minimum(lq, np.maximum(lk, 1))
    sh = W.Shape("paged", B=lk.size + 2, Hq=Hq, Hkv=Hkv, D=D, max_q=max_q, s_max=s_max)
    lq = np.concatenate([lq, [0, 0]])
    lk = np.concatenate([lk, [0, 0]])
    return sh, W.make_batch(sh, lq, lk, seed=seed, gen_device="cuda")


def _run_paged(plan, batch, pc):
    sh = batch.shape
    q = batch.q.cuda()
    cu_q = torch.from_numpy(batch.cu_q).cuda()
    cu_k = torch.from_numpy(batch.cu_k).cuda()
    out = sentinel_out(q.shape[0], sh.Hq, sh.D)
    lse = sentinel_lse(q.shape[0], sh.Hq)
    plan.run_paged(q, pc.k_cache, pc.v_cache, pc.block_table, cu_q, cu_k, out, lse)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("page_size", [8, 16, 64, 256])
@pytest.mark.parametrize("variant,Hq,max_q", [(MMA, 16, 1), (MMA, 16, 4), (TC, 32, 8), (TC, 32, 40), (SIMT, 16, 2)])
def test_paged_parity(variant, Hq, max_q, page_size):
    sh, batch = _edge_batch(Hq, max_q)
    pc = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, page_size, sh.s_max, seed=page_size, extra_cols=2)
    plan = plan_for(sh, variant=variant)
    out, lse = _run_paged(plan, batch, pc)
    assert plan.check_error() == 0           # no table entry past a sequence's pages was read
    ref_o, ref_l = oracle_full(batch)
    compare_full(out.cpu(), lse.cpu(), ref_o, ref_l, covered_rows(batch))


@pytest.mark.parametrize("variant", [MMA, TC, SIMT])
def test_paged_fused_cache_layout(variant):
    """K and V as the two halves of one [pages, 2, page_size, Hkv, D] buffer
    (page stride 2 * page_size * Hkv * D)."""
    Hq, max_q = (16, 1) if variant == MMA else (32, 4)
    sh, batch = _edge_batch(Hq, max_q, seed=37)
    pc = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, 32, sh.s_max, seed=3, fused=True)
    assert not pc.k_cache.is_contiguous()
    plan = plan_for(sh, variant=variant)
    out, lse = _run_paged(plan, batch, pc)
    assert plan.check_error() == 0
    ref_o, ref_l = oracle_full(batch)
    compare_full(out.cpu(), lse.cpu(), ref_o, ref_l, covered_rows(batch))


@pytest.mark.parametrize("variant", [MMA, TC])
def test_paged_split_units_and_block_counts(variant):
    """Few blocks over long sequences: units cut across blocks, run-time
    claims, the slot combine and (tcgen05) the fused merge, all through the
    page table."""
    Hq, max_q = (16, 1) if variant == MMA else (32, 8)
    sh = W.Shape("paged_long", B=3, Hq=Hq, Hkv=4, D=128, max_q=max_q, s_max=9000)
    batch = W.make_batch(sh, [1, max_q, min(2, max_q)], [9000, 4097, 3001], seed=41, gen_device="cuda")
    pc = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, 16, sh.s_max, seed=5)
    ref_o, ref_l = oracle_full(batch)
    kws = [{"ctas": 7}, {"ctas": 7, "deterministic": 1}, {"ctas": 7, "deterministic": -1}, {}]
    if variant == TC:
        # the fused merge (the block holding each cut unit's last part merges it) on pages
        kws.append({"ctas": 7, "combine": vg.ATTN_COMBINE_FUSED})
    for kw in kws:
        plan = plan_for(sh, variant=variant, **kw)
        out, lse = _run_paged(plan, batch, pc)
        assert plan.check_error() == 0
        compare_full(out.cpu(), lse.cpu(), ref_o, ref_l, covered_rows(batch))


def test_paged_ragged_workload_sampled():
    """The ragged decode workload (64 sequences, Lk ~ U{0..8192}) in 16-key
    pages, checked on sampled rows."""
    batch = W.workload("ragged", gen_device="cuda")
    sh = batch.shape
    pc = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, 16, sh.s_max, seed=9)
    plan = plan_for(sh)
    out, lse = _run_paged(plan, batch, pc)
    assert plan.check_error() == 0
    rng = np.random.default_rng(2)
    rows = sample_rows(batch, 200, rng)
    import oracle
    ro, rl = oracle.attention_rows(W.bits(batch.q), W.bits(batch.k), W.bits(batch.v), batch.cu_q, batch.cu_k,
                                   rows, B=sh.B, Hq=sh.Hq, Hkv=sh.Hkv, D=sh.D)
    tok = batch.cu_q[rows[:, 0]] + rows[:, 1]
    o = out.cpu()[tok, rows[:, 2]].float().numpy()
    l = lse.cpu()[tok, rows[:, 2]].numpy()
    check_values(o, l, ro, rl)


@pytest.mark.parametrize("variant", [MMA, TC, SIMT])
def test_paged_bad_table_entry_is_flagged_and_stays_in_bounds(variant):
    """A table entry past the cache sets ATTN_DEV_ERR_PAGE; the keys it names
    read as zeros (no access outside the cache), and the other sequences'
    rows still match the oracle."""
    Hq, max_q = (16, 1) if variant == MMA else (32, 4)
    sh, batch = _edge_batch(Hq, max_q, seed=43)
    pc = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, 64, sh.s_max, seed=8)
    bad_b = int(np.argmax(batch.lens_k))              # a sequence with several pages
    pc.block_table[bad_b, 1] = pc.k_cache.shape[0] + 1000
    plan = plan_for(sh, variant=variant)
    out, lse = _run_paged(plan, batch, pc)
    assert plan.check_error() & vg.ATTN_DEV_ERR_PAGE
    ref_o, ref_l = oracle_full(batch)
    cov = covered_rows(batch)
    q0, q1 = int(batch.cu_q[bad_b]), int(batch.cu_q[bad_b + 1])
    cov[q0:q1] = False
    o = out.cpu().float().numpy()
    l = lse.cpu().numpy()
    check_values(o[cov], l[cov], ref_o[cov], ref_l[cov])
    # a clean call afterwards on the same plan is exact again
    pc2 = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, 64, sh.s_max, seed=8)
    out, lse = _run_paged(plan, batch, pc2)
    assert plan.check_error() == 0
    compare_full(out.cpu(), lse.cpu(), ref_o, ref_l, covered_rows(batch))


def test_paged_graph_replay_with_new_tables():
    """Captured once, replayed with the block table and lengths rewritten in
    place (the decode-step pattern of a paged cache)."""
    sh = W.Shape("paged_graph", B=8, Hq=32, Hkv=4, D=128, max_q=1, s_max=2048)
    rng = np.random.default_rng(5)
    cols = sh.s_max // 16
    q = torch.empty(sh.B, sh.Hq, sh.D, dtype=torch.bfloat16, device="cuda")
    cu_q = torch.from_numpy(W.cu_from_lengths(np.ones(sh.B, np.int64))).cuda()
    cu_k = torch.zeros(sh.B + 1, dtype=torch.int32, device="cuda")
    n_pages = sh.B * cols + 4
    kc = torch.full((n_pages, 16, sh.Hkv, sh.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    bt = torch.full((sh.B, cols), -1, dtype=torch.int32, device="cuda")
    out = sentinel_out(sh.B, sh.Hq, sh.D)
    lse = sentinel_lse(sh.B, sh.Hq)
    plan = plan_for(sh)
    graph = None
    for step in range(4):
        lk = rng.integers(0, sh.s_max, sh.B, endpoint=True)
        batch = W.make_batch(sh, np.ones(sh.B, np.int64), lk, seed=100 + step, gen_device="cuda")
        pc = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, 16, sh.s_max, seed=step,
                        spare_pages=n_pages - int(((lk + 15) // 16).sum()))
        kc.copy_(pc.k_cache)
        vc.copy_(pc.v_cache)
        bt.copy_(pc.block_table)
        cu_k.copy_(torch.from_numpy(batch.cu_k))
        q.copy_(batch.q)
        if graph is None:
            plan.run_paged(q, kc, vc, bt, cu_q, cu_k, out, lse)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, capture_error_mode="global"):
                plan.run_paged(q, kc, vc, bt, cu_q, cu_k, out, lse)
        graph.replay()
        torch.cuda.synchronize()
        assert plan.check_error() == 0
        ref_o, ref_l = oracle_full(batch)
        compare_full(out.cpu(), lse.cpu(), ref_o, ref_l, covered_rows(batch))
    del graph


def test_paged_rejects_bad_arguments():
    import ctypes
    sh = W.Shape("paged_bad", B=2, Hq=8, Hkv=2, D=64, max_q=1, s_max=64)
    plan = plan_for(sh)
    lib = vg.lib()
    t = torch.zeros(1 << 16, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    bt = torch.zeros(2, 8, dtype=torch.int32, device="cuda")
    lse = torch.zeros(16, dtype=torch.float32, device="cuda")
    tok = sh.Hkv * sh.D

    def call(page_stride, token_stride, page_size, num_pages, bt_stride):
        return lib.attn_run_paged(plan._h, t.data_ptr(), t.data_ptr(), t.data_ptr(), page_stride, token_stride,
                                  page_size, num_pages, bt.data_ptr(), bt_stride, cu.data_ptr(), cu.data_ptr(),
                                  t.data_ptr(), lse.data_ptr(), None)

    assert call(8 * tok, tok, 8, 4, 8) == 0                 # accepted
    assert call(16 * tok, tok, 12, 4, 8) == -1              # page size not a power of two
    assert call(4 * tok, tok, 4, 4, 16) == -1               # page size below 8
    assert call(8 * tok, tok, 8, 0, 8) == -1                # no pages
    assert call(8 * tok, tok, 8, 4, 7) == -1                # table row shorter than s_max / page_size
    assert call(8 * tok, tok - 8, 8, 4, 8) == -1            # token stride below Hkv * D
    assert call(8 * tok + 4, tok, 8, 4, 8) == -1            # page stride not 16-byte aligned
    assert call(7 * tok, tok, 8, 4, 8) == -1                # pages overlap
    assert lib.attn_run_paged(plan._h, t.data_ptr(), t.data_ptr(), t.data_ptr(), 8 * tok, tok, 8, 4, None, 8,
                              cu.data_ptr(), cu.data_ptr(), t.data_ptr(), lse.data_ptr(), None) == -3
    torch.cuda.synchronize()
    assert plan.check_error() == 0
