"""The seeded input recipes (workloads.py) against the workload descriptions
they follow, and bench.py's byte accounting (CPU only).

The descriptions fix: tiny decode with kv lengths {37, 100}, Hq = 4, Hkv = 1,
D = 64; one 32768-key sequence with Hq = 64, Hkv = 8, D = 128; a ragged
batch of 64 lengths uniform on the integers [0, 8192] (zeros allowed); 100
continuous-batching steps of 256 lengths lognormal with mean 2048 and
sigma 1, clamped to [1, 16384]; short queries of U{1..16} tokens over
U{q_len..4096} keys; Q/K/V iid N(0, 1) in bf16."""
import json
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402


def test_shapes_match_the_descriptions():
    S = W.SHAPES
    assert (S["tiny"].B, S["tiny"].Hq, S["tiny"].Hkv, S["tiny"].D, S["tiny"].max_q) == (2, 4, 1, 64, 1)
    assert (S["long"].B, S["long"].Hq, S["long"].Hkv, S["long"].D, S["long"].s_max) == (1, 64, 8, 128, 32768)
    assert (S["ragged"].B, S["ragged"].Hq, S["ragged"].Hkv, S["ragged"].s_max) == (64, 32, 8, 8192)
    assert (S["continuous"].B, S["continuous"].Hq, S["continuous"].Hkv, S["continuous"].s_max) == (256, 64, 8, 16384)
    assert (S["shortq"].B, S["shortq"].Hq, S["shortq"].Hkv, S["shortq"].max_q, S["shortq"].s_max) == (32, 32, 4, 16, 4096)
    for sh in S.values():
        assert sh.Hq % sh.Hkv == 0 and sh.G == sh.Hq // sh.Hkv


def test_fixed_lengths():
    (lq, lk), = W.lengths("tiny")
    assert lq.tolist() == [1, 1] and lk.tolist() == [37, 100]
    (lq, lk), = W.lengths("long")
    assert lq.tolist() == [1] and lk.tolist() == [32768]


def test_ragged_lengths_are_integers_on_the_closed_range():
    (lq, lk), = W.lengths("ragged", seed=0)
    assert lk.dtype == np.int64 and len(lk) == 64 and (lq == 1).all()
    assert lk.min() >= 0 and lk.max() <= 8192
    # over many seeds both ends of the closed range are reached
    allk = np.concatenate([W.lengths("ragged", seed=s)[0][1] for s in range(400)])
    assert allk.min() == 0 and allk.max() == 8192
    assert abs(allk.mean() - 4096) < 60                      # uniform mean, 25600 draws


def test_continuous_lengths_lognormal_mean_2048_clamped():
    steps = W.lengths("continuous", seed=0)
    assert len(steps) == 100
    lk = np.stack([s[1] for s in steps])
    assert lk.shape == (100, 256) and lk.min() >= 1 and lk.max() <= 16384
    assert all((s[0] == 1).all() for s in steps)
    # arithmetic mean 2048 before clamping; the clamp at 16384 removes about
    # 1% of the mass (sigma = 1), so the sample mean sits a little below
    assert 1900 < lk.mean() < 2100
    # sigma 1 in log space: the median is 2048 / e^(1/2)
    assert abs(np.median(lk) / (2048 / np.exp(0.5)) - 1) < 0.05
    # steps differ (lengths re-drawn every step)
    assert not np.array_equal(lk[0], lk[1])


def test_shortq_lengths():
    for seed in range(20):
        (lq, lk), = W.lengths("shortq", seed=seed)
        assert len(lq) == 32 and lq.min() >= 1 and lq.max() <= 16
        assert (lk >= lq).all() and lk.max() <= 4096


def test_cu_from_lengths_pads_and_checks():
    cu = W.cu_from_lengths([3, 0, 5], entries=6)
    assert cu.dtype == np.int32 and cu.tolist() == [0, 3, 3, 8, 8, 8]
    with pytest.raises(ValueError):
        W.cu_from_lengths([1, 2], entries=2)
    with pytest.raises(ValueError):
        W.cu_from_lengths([2 ** 31])


def test_batches_are_seeded_bf16_normal():
    b1 = W.workload("tiny", seed=0)
    b2 = W.workload("tiny", seed=0)
    b3 = W.workload("tiny", seed=1)
    assert b1.q.dtype == torch.bfloat16 and tuple(b1.q.shape) == (2, 4, 64)
    assert tuple(b1.k.shape) == (137, 1, 64) and tuple(b1.v.shape) == (137, 1, 64)
    assert torch.equal(b1.k, b2.k) and not torch.equal(b1.k, b3.k)
    assert b1.cu_k.tolist() == [0, 37, 137] and b1.cu_q.tolist() == [0, 1, 2]
    x = W.bf16_normal((200000,), W.make_generator(5, "cpu"), "cpu").float()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1) < 0.01


def test_bf16_bit_round_trip():
    a = np.array([0.0, -0.0, 1.0, -2.5, 3.140625, 1e-30, 65504.0], np.float64)
    bits = W.f64_to_bf16_bits(a)
    back = W.bf16_bits_to_f64(bits)
    assert np.array_equal(back, torch.tensor(a).to(torch.bfloat16).double().numpy())


def test_paginated_cache_gathers_back_to_the_packed_keys():
    sh = W.Shape("pg", B=3, Hq=4, Hkv=2, D=64, max_q=1, s_max=100)
    batch = W.make_batch(sh, [1, 1, 1], [100, 0, 37], seed=4)
    for page in (8, 16, 64):
        pc = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, page, sh.s_max, seed=page, fill=float("nan"))
        bt = pc.block_table.cpu().numpy()
        for b in range(sh.B):
            k0, k1 = int(batch.cu_k[b]), int(batch.cu_k[b + 1])
            for j in range(k1 - k0):
                pg, slot = bt[b, j // page], j % page
                assert torch.equal(pc.k_cache[pg, slot], batch.k[k0 + j])
                assert torch.equal(pc.v_cache[pg, slot], batch.v[k0 + j])


def test_algorithmic_bytes_of_the_workloads():
    import bench
    # K and V: sum(Lk) * Hkv * D * 2 bytes each; Q and O: T_q * Hq * D * 2 each
    assert bench.algorithmic_bytes(W.workload("tiny"))["total"] == 137 * 1 * 64 * 4 + 2 * 4 * 64 * 4 == 37120
    long = W.Batch(W.SHAPES["long"], None, None, None, np.array([0, 1], np.int32), np.array([0, 32768], np.int32),
                   np.array([1]), np.array([32768]))
    assert bench.algorithmic_bytes(long)["total"] == 32768 * 8 * 128 * 4 + 64 * 128 * 4 == 134250496


def test_recorded_traffic_follows_the_source_hash():
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    for wl, e in rec.items():
        got, note = bench.recorded_traffic(wl, e["kernel"])
        if e["source_hash"] == bench.kernel_source_hash():
            assert got == e["dram_bytes_per_launch"]
        else:
            assert got is None and "changed" in note
    assert bench.recorded_traffic("long", "another_kernel")[0] is None
    assert bench.recorded_traffic("no_such_workload", "split_mma_kernel")[0] is None


def test_comment_edits_keep_the_source_hash():
    import bench
    a = 'int f(int x) {\n    return x + 1;   // one more\n}\n'
    b = '/* f: the successor */\nint f(int x) {\n\n    return x + 1;\n}\n'
    c = 'int f(int x) {\n    return x + 2;\n}\n'
    assert bench.strip_c_comments(a) == bench.strip_c_comments(b) != bench.strip_c_comments(c)
    s = 'const char *p = "a // b /* c */"; char q = \'"\';  // tail'
    assert bench.strip_c_comments(s) == 'const char *p = "a // b /* c */"; char q = \'"\';'
