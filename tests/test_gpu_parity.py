"""CUDA path vs the fp64 oracle on the same seeded inputs (needs a B200).

Every call goes through the C ABI (libvgqa.so via the ctypes binding).
Tolerances: max-abs 2e-2 on the bf16 output, 1e-3 on the fp32 lse, -inf lse
and zero output matched exactly, and cu_seqlens placement bit-exact (every
covered row written, every other row keeps its NaN sentinel).
"""
import itertools

import numpy as np
import pytest
import torch

import workloads as W
from gpu_helpers import (ATOL_LSE, ATOL_OUT, BF16_NAN_BITS, check_values, compare_full, compare_rows, covered_rows, oracle_full,
                         plan_for, run_gpu, sample_rows, sentinel_lse, sentinel_out, to_device)
import varlen_gqa_split_b200 as vg

pytestmark = pytest.mark.gpu

SIMT, MMA, TC = vg.ATTN_VARIANT_SIMT, vg.ATTN_VARIANT_MMA, vg.ATTN_VARIANT_TC


@pytest.fixture(scope="module", autouse=True)
def _built():
    from varlen_gqa_split_b200 import build
    build.build()
    torch.cuda.init()


def _gen_device(name):
    return "cpu" if name == "tiny" else "cuda"


# ------------------------------------------------------------ the five workloads

@pytest.mark.parametrize("variant", [0, SIMT, MMA, TC])
@pytest.mark.parametrize("name", ["tiny", "long", "ragged"])
def test_decode_workloads_full_parity(name, variant):
    batch = W.workload(name, gen_device=_gen_device(name))
    plan = plan_for(batch.shape, variant=variant)
    out, lse = run_gpu(plan, batch, extra_q_rows=3)
    ref_o, ref_l = oracle_full(batch)
    cov = covered_rows(batch)
    compare_full(out, lse, ref_o, ref_l, cov)


@pytest.mark.parametrize("variant", [0, SIMT, TC])
def test_short_query_workload_full_parity(variant):
    batch = W.workload("shortq", gen_device="cuda")
    plan = plan_for(batch.shape, variant=variant)
    out, lse = run_gpu(plan, batch, extra_q_rows=5)
    ref_o, ref_l = oracle_full(batch)
    compare_full(out, lse, ref_o, ref_l, covered_rows(batch))


def test_continuous_batching_one_graph_many_steps():
    """One CUDA graph captured once (global capture mode: any host sync or
    pageable copy inside attn_run would break the capture) and replayed for
    100 steps while the lengths change in place; each step is checked against
    the oracle on sampled rows."""
    sh = W.SHAPES["continuous"]
    steps = W.lengths("continuous", seed=0)
    cap = max(int(lk.sum()) for _, lk in steps)
    g = W.make_generator(0, "cuda")
    k = W.bf16_normal((cap, sh.Hkv, sh.D), g, "cuda")
    v = W.bf16_normal((cap, sh.Hkv, sh.D), g, "cuda")
    qpool = W.bf16_normal((len(steps), sh.B, sh.Hq, sh.D), g, "cuda")
    q = torch.empty(sh.B, sh.Hq, sh.D, dtype=torch.bfloat16, device="cuda")
    cu_q = torch.from_numpy(W.cu_from_lengths(np.ones(sh.B, np.int64))).cuda()
    cu_k = torch.zeros(sh.B + 1, dtype=torch.int32, device="cuda")
    out = sentinel_out(sh.B, sh.Hq, sh.D)
    lse = sentinel_lse(sh.B, sh.Hq)
    plan = plan_for(sh)
    cu_k.copy_(torch.from_numpy(W.cu_from_lengths(steps[0][1])))
    q.copy_(qpool[0])
    plan.run(q, k, v, cu_q, cu_k, out, lse)          # warm-up outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="global"):
        plan.run(q, k, v, cu_q, cu_k, out, lse)
    kb, vb = W.bits(k), W.bits(v)
    rng = np.random.default_rng(0)
    for s, (lq, lk) in enumerate(steps):
        cu_k.copy_(torch.from_numpy(W.cu_from_lengths(lk)))
        q.copy_(qpool[s])
        graph.replay()
        torch.cuda.synchronize()
        batch = W.Batch(sh, q.cpu(), None, None, W.cu_from_lengths(lq), W.cu_from_lengths(lk), lq, lk)
        rows = sample_rows(batch, 24, rng)
        import oracle
        ro, rl = oracle.attention_rows(W.bits(batch.q), kb, vb, batch.cu_q, batch.cu_k, rows, B=sh.B,
                                       Hq=sh.Hq, Hkv=sh.Hkv, D=sh.D)
        oc = out.cpu()[rows[:, 0], rows[:, 2]].float().numpy()
        lc = lse.cpu()[rows[:, 0], rows[:, 2]].numpy()
        check_values(oc, lc, ro, rl)
    assert plan.check_error() == 0
    del graph


# ------------------------------------------------------------ split-count invariance

@pytest.mark.parametrize("combine", [vg.ATTN_COMBINE_FUSED, vg.ATTN_COMBINE_KERNEL])
def test_nsplit_invariance_simt(combine):
    sh = W.Shape("mid", B=4, Hq=64, Hkv=8, D=128, max_q=1, s_max=4096)
    batch = W.make_batch(sh, [1, 1, 1, 1], [4096, 1000, 77, 0], seed=3, gen_device="cuda")
    ref_o, ref_l = oracle_full(batch)
    cov = covered_rows(batch)
    outs = []
    for ns in (1, 2, 3, 8, 32, 64):
        plan = plan_for(sh, variant=SIMT, nsplit=ns, combine=combine)
        assert plan.info["nsplit"] == ns
        assert plan.info["combine"] == (0 if ns == 1 else combine)
        out, lse = run_gpu(plan, batch)
        compare_full(out, lse, ref_o, ref_l, cov)
        outs.append(out.float().numpy())
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2 * ATOL_OUT


@pytest.mark.parametrize("stages,det", [(0, 0), (0, 1), (2, 0), (3, 1)])
def test_block_count_invariance_mma(stages, det):
    """The persistent tensor-core path at 1 .. 2 x SM-count blocks: from one
    block that finishes every unit itself to shares that cut every unit many
    times (several partials per unit, merged by the last block to finish)."""
    sh = W.Shape("mid", B=4, Hq=64, Hkv=8, D=128, max_q=1, s_max=4096)
    batch = W.make_batch(sh, [1, 1, 1, 1], [4096, 1000, 77, 0], seed=3, gen_device="cuda")
    ref_o, ref_l = oracle_full(batch)
    cov = covered_rows(batch)
    outs = []
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for ctas in (1, 2, 3, 7, 37, sms, 2 * sms):
        plan = plan_for(sh, variant=MMA, ctas=ctas, stages=stages, deterministic=det)
        assert plan.info["ctas"] == ctas and plan.info["nsplit"] == 0
        out, lse = run_gpu(plan, batch)
        compare_full(out, lse, ref_o, ref_l, cov)
        outs.append(out.float().numpy())
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2 * ATOL_OUT


@pytest.mark.parametrize("stages,det", [(0, -1), (0, 1), (2, -1), (3, 0)])
def test_block_count_invariance_tc(stages, det):
    """The tcgen05 path at 1 .. 2 x SM-count blocks on a short-query batch:
    whole units, units cut into many parts, a unit without keys, and rows
    that see no key under the tail-aligned causal mask (Lq > Lk)."""
    sh = W.Shape("midq", B=5, Hq=32, Hkv=4, D=128, max_q=16, s_max=2048)
    batch = W.make_batch(sh, [16, 3, 9, 1, 12], [2048, 700, 5, 0, 130], seed=13, gen_device="cuda")
    ref_o, ref_l = oracle_full(batch)
    cov = covered_rows(batch)
    outs = []
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for ctas in (1, 2, 3, 7, 37, sms, 2 * sms):
        plan = plan_for(sh, variant=TC, ctas=ctas, stages=stages, deterministic=det)
        assert plan.info["ctas"] == ctas and plan.info["variant"] == TC
        out, lse = run_gpu(plan, batch, extra_q_rows=2)
        compare_full(out, lse, ref_o, ref_l, cov)
        outs.append(out.float().numpy()[:len(cov)][cov])
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2 * ATOL_OUT


@pytest.mark.parametrize("Hq,Hkv,D,max_q", [(64, 4, 128, 8), (24, 4, 64, 5), (12, 12, 128, 128),
                                            (16, 2, 64, 16), (40, 8, 128, 3)])
def test_tc_row_layouts(Hq, Hkv, D, max_q):
    """Query boxes of G heads x max_q tokens for several G (odd ones
    included), both head dims, and the 128-row limit (G * max_q = 128)."""
    rng = np.random.default_rng(Hq * 7 + max_q)
    B = 9
    lq = rng.integers(1, max_q, B, endpoint=True)
    lk = np.array([rng.integers(0, 700) for _ in lq])
    lk[0], lq[0] = 0, max_q
    lk[1] = max(1, int(lq[1]) - 1)
    sh = W.Shape("rows", B=B + 1, Hq=Hq, Hkv=Hkv, D=D, max_q=max_q, s_max=700)
    batch = W.make_batch(sh, lq, lk, seed=21, gen_device="cuda")
    ref_o, ref_l = oracle_full(batch)
    for combine in (vg.ATTN_COMBINE_KERNEL, vg.ATTN_COMBINE_FUSED):
        plan = plan_for(sh, variant=TC, ctas=11, combine=combine)
        assert plan.info["combine"] == combine
        out, lse = run_gpu(plan, batch, extra_q_rows=3)
        compare_full(out, lse, ref_o, ref_l, covered_rows(batch))


def test_variants_agree():
    batch = W.workload("ragged", gen_device="cuda")
    a, la = run_gpu(plan_for(batch.shape, variant=SIMT), batch)
    b, lb = run_gpu(plan_for(batch.shape, variant=MMA), batch)
    cov = covered_rows(batch)
    fa, fb = a.float().numpy()[cov], b.float().numpy()[cov]
    assert np.abs(fa - fb).max() <= 2 * ATOL_OUT
    l1, l2 = la.numpy()[cov], lb.numpy()[cov]
    fin = np.isfinite(l1)
    assert np.array_equal(fin, np.isfinite(l2))
    assert np.abs(l1[fin] - l2[fin]).max() <= 2 * ATOL_LSE


@pytest.mark.parametrize("kw", [{"deterministic": 1}, {"variant": TC, "deterministic": 1}, {"variant": TC},
                                {"variant": TC, "combine": vg.ATTN_COMBINE_FUSED},
                                {"variant": TC, "combine": vg.ATTN_COMBINE_KERNEL},
                                {"variant": SIMT, "nsplit": 8, "combine": vg.ATTN_COMBINE_FUSED},
                                {"variant": SIMT, "nsplit": 8, "combine": vg.ATTN_COMBINE_KERNEL}])
def test_repeat_runs_bitwise_equal(kw):
    # a deterministic plan repeats bit for bit: fixed tile shares and a fixed
    # merge order, whichever block finishes last
    batch = W.workload("long", gen_device="cuda")
    plan = plan_for(batch.shape, **kw)
    assert plan.info["deterministic"] == 1
    runs = [run_gpu(plan, batch) for _ in range(3)]
    for o, l in runs[1:]:
        assert torch.equal(o.view(torch.int16), runs[0][0].view(torch.int16))
        assert torch.equal(l.view(torch.int32), runs[0][1].view(torch.int32))


def test_dynamic_balance_repeats_within_rounding():
    # with run-time balancing inside cut units, repeated calls agree with each
    # other and with the oracle within the tolerance, not bit for bit
    batch = W.workload("long", gen_device="cuda")
    plan = plan_for(batch.shape)
    assert plan.info["deterministic"] == 0 and plan.info["variant"] == MMA
    ref_o, ref_l = oracle_full(batch)
    cov = covered_rows(batch)
    runs = [run_gpu(plan, batch) for _ in range(4)]
    for o, l in runs:
        compare_full(o, l, ref_o, ref_l, cov)
    for o, _ in runs[1:]:
        assert (o.float() - runs[0][0].float()).abs().max().item() <= 2 * ATOL_OUT


# ------------------------------------------------------------ strided K/V (views into larger buffers)

@pytest.mark.parametrize("variant,Hq,max_q", [(MMA, 16, 1), (TC, 32, 8), (SIMT, 16, 2)])
@pytest.mark.parametrize("layout", ["fused_kv", "wide_heads"])
def test_strided_kv_views(variant, Hq, max_q, layout):
    """K and V as views with a token stride: the halves of a fused [T, 2, Hkv, D]
    cache, or Hkv heads out of a buffer with more heads per token.  The
    oracle gets packed copies of the same bytes."""
    Hkv, D = 4, 128
    rng = np.random.default_rng(17)
    B = 7
    lq = rng.integers(1, max_q, B, endpoint=True)
    lk = rng.integers(0, 600, B)
    lk[0] = 0
    sh = W.Shape("strided", B=B + 1, Hq=Hq, Hkv=Hkv, D=D, max_q=max_q, s_max=600)
    batch = W.make_batch(sh, lq, lk, seed=23, gen_device="cuda")
    T = batch.k.shape[0]
    if layout == "fused_kv":
        buf = torch.empty(T, 2, Hkv, D, dtype=torch.bfloat16, device="cuda")
        buf[:, 0] = batch.k
        buf[:, 1] = batch.v
        kv, vv = buf[:, 0], buf[:, 1]
    else:
        buf_k = torch.zeros(T, Hkv + 3, D, dtype=torch.bfloat16, device="cuda")
        buf_v = torch.zeros(T, Hkv + 5, D, dtype=torch.bfloat16, device="cuda")
        buf_k[:, 2:2 + Hkv] = batch.k
        buf_v[:, 1:1 + Hkv] = batch.v
        kv, vv = buf_k[:, 2:2 + Hkv], buf_v[:, 1:1 + Hkv]
    assert not kv.is_contiguous()
    plan = plan_for(sh, variant=variant)
    q = batch.q.cuda()
    cu_q = torch.from_numpy(batch.cu_q).cuda()
    cu_k = torch.from_numpy(batch.cu_k).cuda()
    out = sentinel_out(q.shape[0], Hq, D)
    lse = sentinel_lse(q.shape[0], Hq)
    plan.run(q, kv, vv, cu_q, cu_k, out, lse)
    torch.cuda.synchronize()
    assert plan.check_error() == 0
    ref_o, ref_l = oracle_full(batch)
    compare_full(out.cpu(), lse.cpu(), ref_o, ref_l, covered_rows(batch))


def test_strided_kv_rejects_bad_strides():
    import ctypes
    sh = W.Shape("strided_bad", B=2, Hq=8, Hkv=2, D=64, max_q=1, s_max=64)
    plan = plan_for(sh)
    lib = vg.lib()
    t = torch.zeros(256, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    lse = torch.zeros(16, dtype=torch.float32, device="cuda")
    args = [plan._h, t.data_ptr(), t.data_ptr(), t.data_ptr(), cu.data_ptr(), cu.data_ptr(), t.data_ptr(),
            lse.data_ptr()]
    for ks, vs in ((64, 128), (128, 132), (128, 1 << 40)):       # below Hkv*D, not a multiple of 8, too large
        assert lib.attn_run_strided(*args, ks, vs, None) == -1     # ATTN_E_INVALID_ARG
    assert lib.attn_run_strided(*args, 136, 128, None) == 0        # wider, aligned: accepted
    torch.cuda.synchronize()


# ------------------------------------------------------------ placement and edge cases

def _packed_cases(B, values):
    lq, lk = [], []
    for lens_q in itertools.product(values, repeat=B):
        for lens_k in itertools.product(values, repeat=B):
            lq.extend(lens_q)
            lk.extend(lens_k)
    return lq, lk


@pytest.mark.parametrize("G,D", [(4, 64), (8, 128), (16, 128)])
def test_direct_one_block_per_unit(G, D):
    """Units of at most two tiles that fit one wave: the warp-MMA plan gives
    block c unit c whole and launches no merge.  Every length edge of such a
    plan (Lq 0, 1 and 2 with Lk 0, 1, 63, 64, 65, 127, 128, Lq > Lk, and
    zero-length sequences padding B_max) against the oracle, with NaN
    sentinels in the rows past cu_q."""
    lq = [1, 1, 0, 2, 1, 2, 1, 1, 2, 0, 1, 0, 0]
    lk = [0, 1, 5, 1, 63, 64, 65, 127, 128, 0, 128, 0, 0]
    max_q = 2 if G <= 8 else 1
    lq = [min(x, max_q) for x in lq]
    sh = W.Shape("direct", B=len(lq), Hq=2 * G, Hkv=2, D=D, max_q=max_q, s_max=128)
    batch = W.make_batch(sh, lq, lk, seed=53, gen_device="cuda")
    plan = plan_for(sh)
    assert plan.info["variant"] == MMA and plan.info["combine"] == 0 and plan.info["ctas"] == 2 * len(lq)
    ref_o, ref_l = oracle_full(batch)
    for _ in range(2):                                   # and a second call on the same plan
        out, lse = run_gpu(plan, batch, extra_q_rows=3)
        compare_full(out, lse, ref_o, ref_l, covered_rows(batch))


@pytest.mark.parametrize("variant", [SIMT, MMA, TC])
def test_exhaustive_small_lengths_placement(variant):
    """Every (Lq, Lk) combination with lengths in [0, 4] for 3 sequences (the
    exhaustive method of TransformerEngine PR #24, section Equivalence), packed
    into one batch and padded with zero-length sequences to B_max; causal tail
    alignment with Lq > Lk included."""
    lq, lk = _packed_cases(3, range(5))
    B_max = len(lq) + 7
    sh = W.Shape("placement", B=B_max, Hq=4, Hkv=1, D=64, max_q=4, s_max=4)
    batch = W.make_batch(sh, lq, lk, seed=11, gen_device="cuda")
    plan = plan_for(sh, variant=variant)
    out, lse = run_gpu(plan, batch, extra_q_rows=2)
    ref_o, ref_l = oracle_full(batch)
    compare_full(out, lse, ref_o, ref_l, covered_rows(batch))


@pytest.mark.parametrize("kw", [{"variant": SIMT, "nsplit": 1}, {"variant": SIMT, "nsplit": 3},
                                {"variant": SIMT, "nsplit": 3, "combine": vg.ATTN_COMBINE_KERNEL},
                                {"variant": MMA, "ctas": 1}, {"variant": MMA, "ctas": 5},
                                {"variant": MMA, "ctas": 64}, {"variant": MMA},
                                {"variant": MMA, "ctas": 64, "deterministic": 1},
                                {"variant": TC, "ctas": 1}, {"variant": TC, "ctas": 5}, {"variant": TC},
                                {"variant": TC, "ctas": 64, "deterministic": 1},
                                {"variant": TC, "ctas": 5, "deterministic": -1},
                                {"variant": TC, "ctas": 64, "deterministic": -1}])
def test_ragged_multi_tile_placement(kw):
    """Lengths spanning several 64-key tiles, units cut across blocks, short
    sequences whose tile starts before the buffer (negative TMA
    coordinates), sequences without keys or queries, Lq up to 2."""
    rng = np.random.default_rng(5 + len(kw))
    B = 40
    lq = rng.integers(0, 3, B)
    lk = rng.integers(0, 330, B)
    lk[:3] = [1, 63, 64]
    lk[3:6] = [65, 0, 129]
    lq[6] = 0
    sh = W.Shape("ragged_mt", B=B + 2, Hq=16, Hkv=2, D=128, max_q=2, s_max=330)
    batch = W.make_batch(sh, lq, lk, seed=7, gen_device="cuda")
    plan = plan_for(sh, **kw)
    out, lse = run_gpu(plan, batch, extra_q_rows=1)
    ref_o, ref_l = oracle_full(batch)
    compare_full(out, lse, ref_o, ref_l, covered_rows(batch))


@pytest.mark.parametrize("variant", [SIMT, MMA, TC])
def test_single_key_returns_v_exactly(variant):
    sh = W.Shape("one", B=5, Hq=8, Hkv=2, D=128, max_q=1, s_max=64)
    batch = W.make_batch(sh, [1] * 5, [1] * 5, seed=2, gen_device="cuda")
    plan = plan_for(sh, variant=variant)
    out, lse = run_gpu(plan, batch)
    G = sh.Hq // sh.Hkv
    want = batch.v.cpu().repeat_interleave(G, dim=1)
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("variant", [SIMT, MMA, TC])
def test_large_magnitude_scores(variant):
    sh = W.Shape("big", B=2, Hq=8, Hkv=1, D=128, max_q=1, s_max=2048)
    batch = W.make_batch(sh, [1, 1], [2048, 513], seed=4, gen_device="cuda")
    batch.q = (batch.q.float() * 30).to(torch.bfloat16)
    plan = plan_for(sh, variant=variant, **({"nsplit": 4} if variant == SIMT else {"ctas": 9}))
    out, lse = run_gpu(plan, batch)
    ref_o, ref_l = oracle_full(batch)
    compare_full(out, lse, ref_o, ref_l, covered_rows(batch))


def test_plan_choices_follow_the_split_rule():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    long_plan = plan_for(W.SHAPES["long"])
    assert long_plan.info["variant"] == MMA and long_plan.info["ctas"] == sms
    ragged_simt = plan_for(W.SHAPES["ragged"], variant=SIMT)
    assert ragged_simt.info["nsplit"] == 1          # B * Hkv = 512 blocks already fill the SMs
    assert ragged_simt.info["scratch_bytes"] <= 1024
    sq = plan_for(W.SHAPES["shortq"])
    assert sq.info["variant"] == TC and sq.info["rows_per_block"] == 128
    # static shares; one row tile per sequence: the combine kernel merges
    assert sq.info["deterministic"] == 1 and sq.info["combine"] == vg.ATTN_COMBINE_KERNEL
    assert sq.info["combine_blocks"] > 0
    # queries over several row tiles: each cut unit merged by the block
    # holding its last part, no second kernel
    pf = plan_for(W.SHAPES["prefill"])
    assert pf.info["variant"] == TC and pf.info["combine"] == vg.ATTN_COMBINE_FUSED
    assert pf.info["combine_blocks"] == 0
    tiny = plan_for(W.SHAPES["tiny"])                 # units of <= 2 tiles: one block each, none cut
    assert tiny.info["variant"] == MMA and tiny.info["ctas"] == 2
    assert tiny.info["combine"] == 0 and tiny.info["combine_blocks"] == 0      # written directly, no merge
    small = plan_for(W.Shape("small", B=300, Hq=8, Hkv=1, D=128, max_q=1, s_max=128))
    assert small.info["combine"] == vg.ATTN_COMBINE_KERNEL                    # 300 units > one wave: shares


# ------------------------------------------------------------ errors

@pytest.mark.parametrize("variant", [0, TC])
def test_device_side_errors_are_flagged_and_rows_untouched(variant):
    sh = W.Shape("err", B=3, Hq=8, Hkv=2, D=128, max_q=1, s_max=64)
    plan = plan_for(sh, variant=variant)
    g = W.make_generator(1, "cuda")
    T = 200
    q = W.bf16_normal((T, sh.Hq, sh.D), g, "cuda")
    k = W.bf16_normal((T, sh.Hkv, sh.D), g, "cuda")
    v = W.bf16_normal((T, sh.Hkv, sh.D), g, "cuda")
    cases = [
        ([0, 1, 2, 3], [0, 10, 75, 80], vg.ATTN_DEV_ERR_K_TOO_LONG, {1}),     # Lk = 65 > s_max
        ([0, 1, 3, 4], [0, 10, 20, 30], vg.ATTN_DEV_ERR_Q_TOO_LONG, {1}),     # Lq = 2 > max_q
        ([0, 1, 2, 3], [0, 10, 5, 30], vg.ATTN_DEV_ERR_OFFSETS, {1}),         # decreasing cu_k
    ]
    for cq, ck, bit, bad in cases:
        out = sentinel_out(T, sh.Hq, sh.D)
        lse = sentinel_lse(T, sh.Hq)
        cu_q = torch.tensor(cq, dtype=torch.int32, device="cuda")
        cu_k = torch.tensor(ck, dtype=torch.int32, device="cuda")
        plan.run(q, k, v, cu_q, cu_k, out, lse)
        flags = plan.check_error()
        assert flags & bit, (flags, bit)
        assert plan.check_error() == 0                       # read-and-clear
        raw = out.view(torch.int16).cpu()
        for b in range(3):
            rows = range(cq[b], cq[b + 1])
            for r in rows:
                written = not bool(torch.all(raw[r] == np.int16(0x7FC0)))
                assert written == (b not in bad), (cq, ck, b)


@pytest.mark.parametrize("variant,combine", [(MMA, 0), (TC, vg.ATTN_COMBINE_KERNEL), (TC, vg.ATTN_COMBINE_FUSED)])
def test_bounded_wait_runs_out_and_plan_recovers(variant, combine):
    """A merge wait that can never be satisfied (the plan's test hook adds a
    part nobody writes; the wait is the combine kernel's, or the merging
    block's in the fused mode) gives up after the plan's wait limit: the call ends,
    ATTN_DEV_ERR_TIMEOUT is reported, the rows of every cut unit keep their
    NaN sentinels while whole units are written and exact, and after
    attn_check_error the same plan gives the oracle's result."""
    sh = W.Shape("stall", B=3, Hq=32, Hkv=4, D=128, max_q=1, s_max=4096)
    # 4096 keys (64 tiles) per KV head of sequence 0 across 16 blocks of about
    # 18 tiles each: those units are always cut; sequence 2 (one tile) never
    batch = W.make_batch(sh, [1, 1, 1], [4096, 300, 17], seed=41, gen_device="cuda")
    ref_o, ref_l = oracle_full(batch)
    plan = plan_for(sh, variant=variant, ctas=16, wait_limit_us=2000, test_stall=1, combine=combine)
    q, k, v, cu_q, cu_k = to_device(batch)
    out = sentinel_out(q.shape[0], sh.Hq, sh.D)
    lse = sentinel_lse(q.shape[0], sh.Hq)
    plan.run(q, k, v, cu_q, cu_k, out, lse)
    flags = plan.check_error()                    # synchronises: the call has ended
    assert flags & vg.ATTN_DEV_ERR_TIMEOUT, flags
    raw = out.view(torch.int16).cpu().numpy()
    o = out.float().cpu().numpy()
    l_ = lse.cpu().numpy()
    untouched = np.all(raw == np.int16(BF16_NAN_BITS), axis=2)       # [T, Hq]
    assert untouched[0].all() and np.isnan(l_[0]).all(), "a cut unit's rows were written"
    written = ~untouched
    # 8 short units (about 2.4 blocks' shares) meet at most 3 share boundaries:
    # most of them are whole, written by the split kernel alone
    assert written[1:].sum() >= 5 * sh.Hq // sh.Hkv, "whole units were not written"
    if variant == MMA:
        assert written[2].all()          # one-tile units, and no fixed cost per unit here: never cut
    check_values(o[written], l_[written], ref_o[written], ref_l[written])
    # the same plan, next call: counters reset, hook cleared
    out2, lse2 = run_gpu(plan, batch)
    compare_full(out2, lse2, ref_o, ref_l, covered_rows(batch))


def test_host_side_errors_launch_nothing():
    import ctypes
    L = vg.lib()
    sh = W.Shape("h", B=1, Hq=4, Hkv=1, D=64, max_q=1, s_max=64)
    plan = plan_for(sh)
    q = torch.zeros(4, 4, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(4, 1, 64, dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    lse = torch.zeros(4, 4, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    h = plan.handle
    assert L.attn_run(h, q.data_ptr() + 2, k.data_ptr(), k.data_ptr(), cu.data_ptr(), cu.data_ptr(),
                      out.data_ptr(), lse.data_ptr(), s) == -4
    assert L.attn_run(h, None, k.data_ptr(), k.data_ptr(), cu.data_ptr(), cu.data_ptr(),
                      out.data_ptr(), lse.data_ptr(), s) == -3
    with pytest.raises(vg.AttnError):
        vg.Plan(1, 64, 4, 1, 96, 1)                         # unsupported head dim
    with pytest.raises(vg.AttnError):
        vg.Plan(1, 64, 64, 8, 128, 4, variant=MMA)         # 32 rows > warp-MMA path limit
    with pytest.raises(vg.AttnError):
        vg.Plan(1, 64, 256, 1, 64, 1, variant=TC)          # G = 256 heads of one token exceed a 128-row tile
    with pytest.raises(vg.AttnError):
        vg.Plan(1, 64, 8, 1, 128, 1, variant=MMA, nsplit=2)  # split count belongs to the SIMT grid
    with pytest.raises(vg.AttnError):                       # the fused merge needs static shares
        vg.Plan(1, 64, 64, 8, 128, 8, variant=TC, deterministic=-1, combine=vg.ATTN_COMBINE_FUSED)
    handle = plan.handle
    plan.close()
    assert L.attn_run(handle, q.data_ptr(), k.data_ptr(), k.data_ptr(), cu.data_ptr(), cu.data_ptr(),
                      out.data_ptr(), lse.data_ptr(), s) == -5
    torch.cuda.synchronize()
    assert torch.all(out == 0)


# ------------------------------------------------------------ long queries (row tiles on tcgen05)

@pytest.mark.parametrize("Hq,Hkv,D,max_q", [(16, 2, 128, 100), (40, 8, 128, 60), (8, 8, 64, 300),
                                            (32, 2, 128, 33), (16, 1, 64, 40)])
def test_tc_row_tiles_long_queries(Hq, Hkv, D, max_q):
    """Queries longer than one 128-row tile: each sequence's queries are cut
    into row tiles of 128 / G tokens from its end, each its own unit with the
    keys its last token sees under the tail-aligned causal mask.  Includes
    Lq > Lk (leading queries that see no key), Lq = 1, an empty sequence and
    a partial first row tile."""
    G = Hq // Hkv
    lq = [max_q, min(37, max_q), 1, max_q // 2 + 1, 0, 7]
    lk = [1000, 37, 5, 20, 9, 0]
    sh = W.Shape("rowtiles", B=len(lq), Hq=Hq, Hkv=Hkv, D=D, max_q=max_q, s_max=1000)
    batch = W.make_batch(sh, lq, lk, seed=29, gen_device="cuda")
    ref_o, ref_l = oracle_full(batch)
    cov = covered_rows(batch)
    for kw in ({}, {"ctas": 5}, {"ctas": 5, "deterministic": 1}, {"ctas": 5, "deterministic": -1},
               {"ctas": 5, "combine": vg.ATTN_COMBINE_KERNEL}, {"ctas": 5, "deterministic": 1,
                                                                "combine": vg.ATTN_COMBINE_FUSED},
               {"ctas": 5, "deterministic": -1, "combine": vg.ATTN_COMBINE_KERNEL}):
        plan = plan_for(sh, **kw)
        assert plan.info["variant"] == TC, plan.info
        out, lse = run_gpu(plan, batch, extra_q_rows=2)
        compare_full(out, lse, ref_o, ref_l, cov)


@pytest.mark.parametrize("variant", [0, SIMT])
def test_prefill_workload_sampled(variant):
    """Causal prefill (q_len = kv_len up to 2048, G = 8: 128 row tiles of 16
    tokens per sequence and KV head) against the oracle on sampled rows, and
    the sentinel rows past cu_q untouched."""
    batch = W.workload("prefill", gen_device="cuda")
    sh = batch.shape
    plan = plan_for(sh, variant=variant)
    assert plan.info["variant"] == (variant or TC)
    out, lse = run_gpu(plan, batch, extra_q_rows=3)
    rng = np.random.default_rng(4)
    rows = sample_rows(batch, 300, rng)
    compare_rows(out, lse, batch, rows)
    raw = out.view(torch.int16).numpy()
    assert np.all(raw[int(batch.cu_q[-1]):] == np.int16(0x7FC0))
