"""attn_run_noalloc, the entry point for callers that cannot allocate device
memory (for example code inside a framework whose pool allocator owns the
whole device budget, or a latency-critical path where cudaMalloc could
synchronise the device).  It keeps its scratch in a fixed array inside the
library instead of allocating.

Checked through the C ABI on two calls in a row (the second call finds the
first call's leftovers in the shared array): each call against the fp64
oracle with the suite's tolerances and sentinel rows, and against the regular
entry point (attn_run through a plan) on the same inputs.  Further calls must
not change the device's free memory.  This file is collected last so that a
failure here cannot hide another test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
import varlen_gqa_split_b200 as vg
from gpu_helpers import (ATOL_LSE, ATOL_OUT, compare_full, covered_rows, oracle_full, sentinel_lse,
                         sentinel_out, to_device)

pytestmark = pytest.mark.gpu


def _lib():
    L = vg.lib()
    L.attn_run_noalloc.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p] * 8
    L.attn_run_noalloc.restype = ctypes.c_int
    return L


def _noalloc(L, sh, q, k, v, cu_q, cu_k, out, lse):
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.attn_run_noalloc(sh.B, sh.s_max, sh.Hq, sh.Hkv, sh.D, sh.max_q, q.data_ptr(), k.data_ptr(),
                              v.data_ptr(), cu_q.data_ptr(), cu_k.data_ptr(), out.data_ptr(),
                              lse.data_ptr(), s)


CASES = [
    # split across many chunks: partials and merge tickets live in the array
    (W.Shape("na_long", B=2, Hq=64, Hkv=8, D=128, max_q=1, s_max=8192), [1, 1], [8192, 3001]),
    # short queries with the causal tail, several row tiles, a zero-length sequence
    (W.Shape("na_shortq", B=4, Hq=32, Hkv=4, D=128, max_q=4, s_max=2048), [4, 1, 3, 2], [2048, 700, 0, 5]),
    (W.Shape("na_tiny", B=2, Hq=4, Hkv=1, D=64, max_q=1, s_max=128), [1, 1], [37, 100]),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_matches_oracle_and_attn_run_twice(case):
    sh, lq, lk = CASES[case]
    L = _lib()
    batch = W.make_batch(sh, lq, lk, seed=21 + case, gen_device="cuda")
    q, k, v, cu_q, cu_k = to_device(batch)
    ref_o, ref_l = oracle_full(batch)
    cov = covered_rows(batch)
    plan = vg.Plan(sh.B, sh.s_max, sh.Hq, sh.Hkv, sh.D, sh.max_q)
    run_o, run_l = plan.run(q, k, v, cu_q, cu_k)
    torch.cuda.synchronize()
    assert plan.check_error() == 0
    run_o = run_o.float().cpu().numpy()
    run_l = run_l.cpu().numpy()
    fin = np.isfinite(run_l)
    for call in range(2):
        out = sentinel_out(q.shape[0], sh.Hq, sh.D)
        lse = sentinel_lse(q.shape[0], sh.Hq)
        rc = _noalloc(L, sh, q, k, v, cu_q, cu_k, out, lse)
        assert rc == 0, vg.strerror(rc)
        torch.cuda.synchronize()
        compare_full(out.cpu(), lse.cpu(), ref_o, ref_l, cov)
        o = out.float().cpu().numpy()
        l_ = lse.cpu().numpy()
        assert np.abs(o - run_o).max() <= ATOL_OUT, f"call {call}"
        assert np.array_equal(np.isfinite(l_), fin), f"call {call}: -inf pattern"
        assert np.abs(l_[fin] - run_l[fin]).max() <= ATOL_LSE, f"call {call}"
    plan.close()


def test_noalloc_calls_leave_free_memory_unchanged():
    """After a first call (which looks up the array and, under lazy module
    loading, commits it), further calls allocate nothing: the device's free
    memory is the same before and after them."""
    sh, lq, lk = CASES[0]
    L = _lib()
    batch = W.make_batch(sh, lq, lk, seed=31, gen_device="cuda")
    q, k, v, cu_q, cu_k = to_device(batch)
    out = sentinel_out(q.shape[0], sh.Hq, sh.D)
    lse = sentinel_lse(q.shape[0], sh.Hq)
    assert _noalloc(L, sh, q, k, v, cu_q, cu_k, out, lse) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(10):
        assert _noalloc(L, sh, q, k, v, cu_q, cu_k, out, lse) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    ref_o, ref_l = oracle_full(batch)
    compare_full(out.cpu(), lse.cpu(), ref_o, ref_l, covered_rows(batch))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    L = _lib()
    # one sequence of 16 query tokens over 256 query heads: 256 row tiles get
    # 2 splits each, whose fp32 partials (4.26 MB) do not fit the fixed array;
    # the call must refuse and launch nothing
    sh = W.Shape("na_big", B=1, Hq=256, Hkv=1, D=128, max_q=16, s_max=4096)
    q = torch.zeros(16, sh.Hq, sh.D, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(16, sh.Hkv, sh.D, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(sh.B + 1, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    lse = torch.zeros(16, sh.Hq, device="cuda")
    rc = _noalloc(L, sh, q, k, k, cu, cu, out, lse)
    assert rc == -10
    assert "scratch" in vg.strerror(rc)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
