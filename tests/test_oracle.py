"""Pins for the fp64 oracle (CPU only).

Each check ties the oracle to something other than itself: a closed form, an
invariant of softmax attention, a second formulation built from library
routines (scipy's softmax / logsumexp over a dense masked score matrix), or
the case counts the TransformerEngine PR prints for its exhaustive
enumeration.  Together they are chosen so that a dropped term, a wrong sign,
a wrong head or token index, or a transposed operand fails at least one.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_bits(rng, shape, scale=1.0):
    return W.f64_to_bf16_bits(rng.standard_normal(shape) * scale)


def f64(bits):
    return W.bf16_bits_to_f64(bits)


def run(q, k, v, lens_q, lens_k, Hq, Hkv, D, causal=True, B_max=None):
    B = len(lens_q)
    B_max = B if B_max is None else B_max
    cu_q = W.cu_from_lengths(lens_q, B_max + 1)
    cu_k = W.cu_from_lengths(lens_k, B_max + 1)
    return oracle.attention(q, k, v, cu_q, cu_k, B=B_max, Hq=Hq, Hkv=Hkv, D=D,
                            causal=causal)


# ---------------------------------------------------------------- closed forms

def test_single_key_returns_v_and_its_score():
    # one key: the softmax weight is 1, out = v0 exactly, lse = the score.
    # q and k are one-hot so the score is known without a dot product.
    D, Hq, Hkv = 64, 4, 1
    rng = np.random.default_rng(1)
    q = np.zeros((1, Hq, D))
    k = np.zeros((1, Hkv, D))
    for h in range(Hq):
        q[0, h, 3] = 1.5 + h          # exact in bf16
    k[0, 0, 3] = -2.0
    v = rand_bits(rng, (1, Hkv, D))
    out, lse = run(W.f64_to_bf16_bits(q), W.f64_to_bf16_bits(k), v, [1], [1], Hq, Hkv, D)
    for h in range(Hq):
        assert np.array_equal(out[0, h], f64(v[0, 0]))
        assert lse[0, h] == pytest.approx((1.5 + h) * -2.0 / math.sqrt(D), abs=1e-15)


def test_identical_keys_give_mean_of_v():
    # n identical keys: uniform weights -> out = mean(V), lse = s + ln n
    D, Hq, Hkv, n = 128, 8, 2, 37
    rng = np.random.default_rng(2)
    q = np.zeros((1, Hq, D))
    q[0, :, 10] = 0.75
    k = np.zeros((n, Hkv, D))
    k[:, :, 10] = 3.0
    v = rand_bits(rng, (n, Hkv, D))
    out, lse = run(W.f64_to_bf16_bits(q), W.f64_to_bf16_bits(k), v, [1], [n], Hq, Hkv, D)
    G = Hq // Hkv
    for h in range(Hq):
        np.testing.assert_allclose(out[0, h], f64(v)[:, h // G].mean(axis=0), rtol=0, atol=1e-14)
        assert lse[0, h] == pytest.approx(0.75 * 3.0 / math.sqrt(D) + math.log(n), abs=1e-13)


def test_zero_query_uniform_over_visible_keys():
    # q = 0: every visible key has score 0 -> out = mean of the visible V rows,
    # lse = ln(visible count); covers the tail-aligned causal counts too
    D, Hq, Hkv = 64, 4, 2
    rng = np.random.default_rng(3)
    lens_q = [3, 1, 5, 2]
    lens_k = [7, 4, 5, 9]
    Tq, Tk = sum(lens_q), sum(lens_k)
    q = np.zeros((Tq, Hq, D), np.uint16)
    k = rand_bits(rng, (Tk, Hkv, D))
    v = rand_bits(rng, (Tk, Hkv, D))
    out, lse = run(q, k, v, lens_q, lens_k, Hq, Hkv, D)
    cq, ck = np.cumsum([0] + lens_q), np.cumsum([0] + lens_k)
    G = Hq // Hkv
    vf = f64(v)
    for b in range(len(lens_q)):
        for qi in range(lens_q[b]):
            n = min(max(lens_k[b] - lens_q[b] + qi + 1, 0), lens_k[b])
            for h in range(Hq):
                row = out[cq[b] + qi, h]
                want = vf[ck[b]:ck[b] + n, h // G].mean(axis=0)
                np.testing.assert_allclose(row, want, rtol=0, atol=1e-14)
                assert lse[cq[b] + qi, h] == pytest.approx(math.log(n), abs=1e-14)


def test_constant_v_gives_constant_out():
    D, Hq, Hkv, n = 128, 8, 1, 200
    rng = np.random.default_rng(4)
    q = rand_bits(rng, (1, Hq, D))
    k = rand_bits(rng, (n, Hkv, D))
    c = rand_bits(rng, (D,))
    v = np.broadcast_to(c, (n, Hkv, D)).copy()
    out, _ = run(q, k, v, [1], [n], Hq, Hkv, D)
    for h in range(Hq):
        np.testing.assert_allclose(out[0, h], f64(c), rtol=1e-14, atol=1e-14)


def test_causal_first_query_sees_only_first_key():
    # Lq = Lk: query 0 sits at absolute position 0 and sees key 0 only
    D, Hq, Hkv, L = 64, 4, 2, 6
    rng = np.random.default_rng(5)
    q = rand_bits(rng, (L, Hq, D))
    k = rand_bits(rng, (L, Hkv, D))
    v = rand_bits(rng, (L, Hkv, D))
    out, _ = run(q, k, v, [L], [L], Hq, Hkv, D)
    G = Hq // Hkv
    for h in range(Hq):
        assert np.array_equal(out[0, h], f64(v[0, h // G]))
    # and the last query sees every key: same as a one-query sequence
    out1, lse1 = run(q[L - 1:L], k, v, [1], [L], Hq, Hkv, D)
    np.testing.assert_allclose(out[L - 1], out1[0], rtol=0, atol=1e-15)


def test_two_keys_logistic_weights_and_scale():
    # two keys with scores s0, s1 known by construction: the weight of key 0
    # is the logistic 1 / (1 + exp(s1 - s0)); pins the 1/sqrt(D) scale and the
    # sign of the max subtraction
    for D in (64, 128):
        Hq = Hkv = 1
        q = np.zeros((1, 1, D)); q[0, 0, 0] = 2.0
        k = np.zeros((2, 1, D)); k[0, 0, 0] = 1.25; k[1, 0, 0] = -0.5
        v = np.zeros((2, 1, D)); v[0, 0, :] = 1.0; v[1, 0, :] = -1.0
        out, lse = run(W.f64_to_bf16_bits(q), W.f64_to_bf16_bits(k), W.f64_to_bf16_bits(v),
                       [1], [2], Hq, Hkv, D)
        s0, s1 = 2.0 * 1.25 / math.sqrt(D), 2.0 * -0.5 / math.sqrt(D)
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))
        np.testing.assert_allclose(out[0, 0], np.full(D, w0 - (1 - w0)), rtol=1e-14)
        assert lse[0, 0] == pytest.approx(math.log(math.exp(s0) + math.exp(s1)), abs=1e-14)


def test_scores_beyond_exp_range_pick_the_top_key():
    # scores 2000, 0, -2000 (one-hot q and k, known without a dot product):
    # exp of their spread overflows fp64, so only a max-subtracted softmax
    # returns the closed form out = v of the top key, lse = 2000
    D = 64
    q = np.zeros((1, 1, D)); q[0, 0, 5] = 256.0
    k = np.zeros((3, 1, D)); k[0, 0, 5] = 0.0; k[1, 0, 5] = 62.5; k[2, 0, 5] = -62.5
    rng = np.random.default_rng(15)
    v = rand_bits(rng, (3, 1, D))
    out, lse = run(W.f64_to_bf16_bits(q), W.f64_to_bf16_bits(k), v, [1], [3], 1, 1, D)
    assert np.array_equal(out[0, 0], f64(v[1, 0]))
    assert lse[0, 0] == 2000.0


def test_gqa_head_mapping_contiguous_groups():
    # V of KV head hk is the constant hk+1: query head h must read KV head h // G
    D, Hq, Hkv, n = 64, 8, 4, 9
    rng = np.random.default_rng(6)
    q = rand_bits(rng, (1, Hq, D))
    k = rand_bits(rng, (n, Hkv, D))
    v = np.zeros((n, Hkv, D))
    for hk in range(Hkv):
        v[:, hk, :] = hk + 1
    out, _ = run(q, k, W.f64_to_bf16_bits(v), [1], [n], Hq, Hkv, D)
    for h in range(Hq):
        np.testing.assert_allclose(out[0, h], h // (Hq // Hkv) + 1, rtol=1e-14)


def test_token_offsets_and_visible_counts():
    # q = 0 and V[t] = t: out = mean of the visible token indices, i.e.
    # cu_k[b] + (n - 1) / 2 -> pins the per-sequence offsets and the counts
    D, Hq, Hkv = 64, 2, 1
    lens_q = [2, 0, 1, 3, 1]
    lens_k = [5, 3, 0, 3, 8]
    Tq, Tk = sum(lens_q), sum(lens_k)
    q = np.zeros((Tq, Hq, D), np.uint16)
    k = rand_bits(np.random.default_rng(7), (Tk, Hkv, D))
    v = W.f64_to_bf16_bits(np.broadcast_to(np.arange(Tk, dtype=np.float64)[:, None, None],
                                           (Tk, Hkv, D)))
    out, lse = run(q, k, v, lens_q, lens_k, Hq, Hkv, D)
    cq, ck = np.cumsum([0] + lens_q), np.cumsum([0] + lens_k)
    for b in range(len(lens_q)):
        for qi in range(lens_q[b]):
            n = min(max(lens_k[b] - lens_q[b] + qi + 1, 0), lens_k[b])
            row = out[cq[b] + qi]
            if n == 0:
                assert np.all(row == 0.0) and np.all(np.isneginf(lse[cq[b] + qi]))
            else:
                np.testing.assert_allclose(row, ck[b] + (n - 1) / 2.0, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- invariants

def test_weights_sum_to_one_and_reproduce_out():
    D, Hq, Hkv = 128, 8, 2
    rng = np.random.default_rng(8)
    lens_q, lens_k = [4, 1], [50, 300]
    Tq, Tk = sum(lens_q), sum(lens_k)
    q, k, v = rand_bits(rng, (Tq, Hq, D)), rand_bits(rng, (Tk, Hkv, D)), rand_bits(rng, (Tk, Hkv, D))
    cu_q, cu_k = W.cu_from_lengths(lens_q), W.cu_from_lengths(lens_k)
    for b, qi, h in [(0, 0, 0), (0, 3, 5), (1, 0, 7)]:
        p, o, lse = oracle.row_weights(q, k, v, cu_q, cu_k, b, qi, h, B=2, Hq=Hq, Hkv=Hkv, D=D)
        assert np.all(p >= 0.0)
        assert abs(p.sum() - 1.0) < 1e-12
        n = p.size
        vf = f64(v)[cu_k[b]:cu_k[b] + n, h // (Hq // Hkv)]
        np.testing.assert_allclose(p @ vf, o, rtol=0, atol=1e-13)


def test_key_permutation_invariance():
    # with every key visible, reordering K and V rows together changes nothing;
    # reordering V alone does (so K and V must be indexed by the same token)
    D, Hq, Hkv, n = 64, 4, 2, 41
    rng = np.random.default_rng(9)
    q, k, v = rand_bits(rng, (1, Hq, D)), rand_bits(rng, (n, Hkv, D)), rand_bits(rng, (n, Hkv, D))
    perm = rng.permutation(n)
    o1, l1 = run(q, k, v, [1], [n], Hq, Hkv, D)
    o2, l2 = run(q, k[perm], v[perm], [1], [n], Hq, Hkv, D)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
    o3, _ = run(q, k, v[perm], [1], [n], Hq, Hkv, D)
    assert np.max(np.abs(o3 - o1)) > 1e-3


def test_lse_merge_identity():
    # oracle partials over [0, a) and [a, n) merged by the log-sum-exp rule
    # equal the oracle over [0, n); includes empty and one-key pieces
    D = 128
    rng = np.random.default_rng(10)
    n = 257
    qrow = rand_bits(rng, (D,), 2.0)
    kr, vr = rand_bits(rng, (n, D)), rand_bits(rng, (n, D))
    scale = 1.0 / math.sqrt(D)
    o_full, m_full, l_full = oracle.partial(qrow, kr, vr, 0, n, scale=scale)
    ref_out = o_full / l_full
    ref_lse = m_full + math.log(l_full)
    for cuts in ([0, n], [0, 100, n], [0, 0, 5, 5, 200, n], [0, 1, 2, 256, n],
                 sorted(set([0, n] + list(rng.integers(0, n, 9))))):
        parts = [oracle.partial(qrow, kr, vr, a, b, scale=scale) for a, b in zip(cuts, cuts[1:])]
        o = np.stack([p[0] for p in parts]); m = np.array([p[1] for p in parts])
        l = np.array([p[2] for p in parts])
        out, lse = oracle.merge(o, m, l)
        np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-13)
        assert lse == pytest.approx(ref_lse, abs=1e-12)
    # the partial of the whole range agrees with the batch oracle
    q3 = qrow.reshape(1, 1, D); k3 = kr.reshape(n, 1, D); v3 = vr.reshape(n, 1, D)
    out, lse = run(q3, k3, v3, [1], [n], 1, 1, D)
    np.testing.assert_allclose(out[0, 0], ref_out, rtol=0, atol=1e-13)
    assert lse[0, 0] == pytest.approx(ref_lse, abs=1e-12)


def test_merge_of_nothing_is_zero_and_neg_inf():
    out, lse = oracle.merge(np.zeros((3, 8)), np.full(3, -np.inf), np.zeros(3))
    assert np.all(out == 0.0) and lse == -np.inf


def test_zero_lengths():
    D, Hq, Hkv = 64, 4, 1
    rng = np.random.default_rng(11)
    lens_q, lens_k = [1, 0, 2, 1], [0, 5, 1, 3]
    Tq, Tk = sum(lens_q), sum(lens_k)
    q, k, v = rand_bits(rng, (Tq, Hq, D)), rand_bits(rng, (Tk, Hkv, D)), rand_bits(rng, (Tk, Hkv, D))
    out, lse = run(q, k, v, lens_q, lens_k, Hq, Hkv, D)
    # b=0: no keys at all -> zero output, lse = -inf
    assert np.all(out[0] == 0.0) and np.all(np.isneginf(lse[0]))
    # b=2: Lq=2 > Lk=1, tail-aligned: query 0 sees nothing, query 1 sees key 0
    assert np.all(out[1] == 0.0) and np.all(np.isneginf(lse[1]))
    assert np.array_equal(out[2, 0], f64(v[5, 0]))
    assert np.all(np.isfinite(out)) and not np.any(np.isnan(lse))


def test_rows_outside_cu_untouched_and_extra_entries_ignored():
    D, Hq, Hkv = 64, 2, 1
    rng = np.random.default_rng(12)
    q, k, v = rand_bits(rng, (6, Hq, D)), rand_bits(rng, (9, Hkv, D)), rand_bits(rng, (9, Hkv, D))
    cu_q = np.array([0, 2, 3], np.int32)
    cu_k = np.array([0, 4, 9], np.int32)
    o1, l1 = oracle.attention(q, k, v, cu_q, cu_k, B=2, Hq=Hq, Hkv=Hkv, D=D)
    assert np.all(np.isnan(o1[3:])) and np.all(np.isnan(l1[3:]))
    # cu buffers longer than B+1 (allocated for a larger batch): the extra
    # entries are never read, even when they hold garbage
    cu_q2 = np.array([0, 2, 3, -7, 1 << 30], np.int32)
    cu_k2 = np.array([0, 4, 9, 2, -1], np.int32)
    o2, l2 = oracle.attention(q, k, v, cu_q2, cu_k2, B=2, Hq=Hq, Hkv=Hkv, D=D)
    np.testing.assert_array_equal(np.nan_to_num(o1, nan=7.0), np.nan_to_num(o2, nan=7.0))
    np.testing.assert_array_equal(np.nan_to_num(l1, nan=7.0), np.nan_to_num(l2, nan=7.0))


def test_rejects_decreasing_offsets():
    D = 64
    z = np.zeros((4, 1, D), np.uint16)
    with pytest.raises(ValueError):
        oracle.attention(z, z, z, np.array([0, 3, 2], np.int32), np.array([0, 1, 2], np.int32),
                         B=2, Hq=1, Hkv=1, D=D)


def test_rows_api_matches_batch():
    D, Hq, Hkv = 128, 8, 2
    rng = np.random.default_rng(13)
    lens_q, lens_k = [3, 1, 2], [20, 70, 2]
    Tq, Tk = sum(lens_q), sum(lens_k)
    q, k, v = rand_bits(rng, (Tq, Hq, D)), rand_bits(rng, (Tk, Hkv, D)), rand_bits(rng, (Tk, Hkv, D))
    out, lse = run(q, k, v, lens_q, lens_k, Hq, Hkv, D)
    cu_q, cu_k = W.cu_from_lengths(lens_q), W.cu_from_lengths(lens_k)
    rows = [(b, qi, h) for b in range(3) for qi in range(lens_q[b]) for h in range(Hq)]
    o2, l2 = oracle.attention_rows(q, k, v, cu_q, cu_k, rows, B=3, Hq=Hq, Hkv=Hkv, D=D)
    for i, (b, qi, h) in enumerate(rows):
        assert np.array_equal(o2[i], out[cu_q[b] + qi, h])
        assert np.array_equal(l2[i], lse[cu_q[b] + qi, h])


# ---------------------------------------------- second formulation (library)

def dense_reference(q, k, v, lens_q, lens_k, Hq, Hkv, D, causal=True):
    """Padded [B, Hq, max_q, max_k] score matrix, boolean padding mask built as
    positions >= seqlens (the construction of TransformerEngine PR #24,
    section Description) plus the tail-aligned causal term, then scipy's
    softmax and logsumexp."""
    B = len(lens_q)
    mq, mk = max(max(lens_q), 1), max(max(lens_k), 1)
    G = Hq // Hkv
    cq, ck = np.cumsum([0] + list(lens_q)), np.cumsum([0] + list(lens_k))
    Q = np.zeros((B, mq, Hq, D)); K = np.zeros((B, mk, Hkv, D)); V = np.zeros((B, mk, Hkv, D))
    for b in range(B):
        Q[b, :lens_q[b]] = f64(q[cq[b]:cq[b + 1]])
        K[b, :lens_k[b]] = f64(k[ck[b]:ck[b + 1]])
        V[b, :lens_k[b]] = f64(v[ck[b]:ck[b + 1]])
    Kh = np.repeat(K, G, axis=2)      # [B, mk, Hq, D]
    Vh = np.repeat(V, G, axis=2)
    S = np.einsum("bqhd,bkhd->bhqk", Q, Kh) / math.sqrt(D)
    seqlens_k = np.asarray(lens_k)
    positions = np.arange(mk)
    masked = positions[None, :] >= seqlens_k[:, None]              # [B, mk]
    masked = np.broadcast_to(masked[:, None, None, :], S.shape).copy()
    if causal:
        qpos = np.arange(mq)[None, :] + (np.asarray(lens_k) - np.asarray(lens_q))[:, None]
        masked |= positions[None, None, None, :] > qpos[:, None, :, None]
    S = np.where(masked, -np.inf, S)
    lse = scipy.special.logsumexp(S, axis=-1)                         # [B, Hq, mq]
    with np.errstate(invalid="ignore"):
        P = np.exp(S - lse[..., None])
    P = np.nan_to_num(P, nan=0.0)
    O = np.einsum("bhqk,bkhd->bqhd", P, Vh)
    return O, np.transpose(lse, (0, 2, 1))                            # [B, mq, Hq, D], [B, mq, Hq]


@pytest.mark.parametrize("seed", range(6))
def test_dense_masked_softmax_agrees(seed):
    rng = np.random.default_rng(100 + seed)
    Hkv = int(rng.choice([1, 2]))
    Hq = Hkv * int(rng.choice([1, 4, 8]))
    D = int(rng.choice([64, 128]))
    B = int(rng.integers(1, 5))
    lens_q = [int(x) for x in rng.integers(0, 5, B)]
    lens_k = [int(x) for x in rng.integers(0, 40, B)]
    Tq, Tk = sum(lens_q), sum(lens_k)
    mag = float(rng.choice([1.0, 30.0]))   # large scores: max subtraction must hold
    q = rand_bits(rng, (Tq, Hq, D), mag)
    k, v = rand_bits(rng, (Tk, Hkv, D)), rand_bits(rng, (Tk, Hkv, D))
    out, lse = run(q, k, v, lens_q, lens_k, Hq, Hkv, D)
    O, L = dense_reference(q, k, v, lens_q, lens_k, Hq, Hkv, D)
    cq = np.cumsum([0] + lens_q)
    for b in range(B):
        for qi in range(lens_q[b]):
            np.testing.assert_allclose(out[cq[b] + qi], O[b, qi], rtol=1e-10, atol=1e-12)
            want = L[b, qi]
            got = lse[cq[b] + qi]
            assert np.array_equal(np.isneginf(got), np.isneginf(want))
            fin = np.isfinite(want)
            np.testing.assert_allclose(got[fin], want[fin], rtol=1e-12, atol=1e-11)


# ------------------------------------- exhaustive enumeration (TE PR #24 method)

def read_golden_counts():
    counts = {}
    with open(os.path.join(GOLDEN, "te_pr24_exhaustive_counts.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fields = line.split()
            counts[fields[0]] = int(fields[-1].split("=")[1])
    return counts


def self_attention_cases():
    for s in range(1, 9):
        for B in range(1, 5):
            for lens in itertools.product(range(s + 1), repeat=B):
                for longer in (False, True):
                    yield s, B, lens, longer


def cross_attention_cases():
    for sq in range(1, 6):
        for sk in range(1, 6):
            for B in range(1, 4):
                for lq in itertools.product(range(sq + 1), repeat=B):
                    for lk in itertools.product(range(sk + 1), repeat=B):
                        yield sq, sk, B, lq, lk


def test_enumeration_reproduces_page_case_counts():
    golden = read_golden_counts()
    assert sum(1 for _ in self_attention_cases()) == golden["self_attention"]
    assert sum(1 for _ in cross_attention_cases()) == golden["cross_attention"]


def _check_packed_group(lq_cases, lk_cases, Hq=2, Hkv=1, D=8, seed=0):
    """Pack many small cases into one batch, run the oracle with q = 0, and
    check every row against the padding mask built as positions >= seqlens
    (plus the tail-aligned causal term): uniform weights over exactly the
    keys the mask leaves visible.

    lq_cases / lk_cases: int arrays [n_cases, B] of query / key lengths."""
    rng = np.random.default_rng(seed)
    LQ = np.asarray(lq_cases, np.int64)
    LK = np.asarray(lk_cases, np.int64)
    nc, Bc = LQ.shape
    lens_q, lens_k = LQ.reshape(-1), LK.reshape(-1)
    Tq, Tk = int(lens_q.sum()), int(lens_k.sum())
    q = np.zeros((max(Tq, 1), Hq, D), np.uint16)
    k = rand_bits(rng, (max(Tk, 1), Hkv, D))
    v = rand_bits(rng, (max(Tk, 1), Hkv, D))
    out, lse = run(q, k, v, list(lens_q), list(lens_k), Hq, Hkv, D)

    # the mask, per case, exactly as the page builds it (vectorised over cases)
    mq, mk = max(int(LQ.max()), 1), max(int(LK.max()), 1)
    positions = np.arange(mk)
    pad = positions[None, None, :] >= LK[:, :, None]                      # [nc, Bc, mk]
    qpos = np.arange(mq)[None, None, :] + (LK - LQ)[:, :, None]          # [nc, Bc, mq]
    vis = ~(pad[:, :, None, :] | (positions[None, None, None, :] > qpos[..., None]))
    # visible sets are prefixes of the sequence's keys, so a count and the
    # sequence offset identify each set
    assert np.all(np.diff(vis.astype(np.int8), axis=-1) <= 0)
    n = vis.sum(axis=-1).reshape(nc * Bc, mq)                            # [seqs, mq]

    cq = np.concatenate([[0], np.cumsum(lens_q)])
    ck = np.concatenate([[0], np.cumsum(lens_k)])
    seq = np.repeat(np.arange(nc * Bc), lens_q)                          # per query row
    qi = np.arange(Tq) - cq[seq]
    nrow = n[seq, qi]
    G = Hq // Hkv
    vf = f64(v)                                                          # [Tk, Hkv, D]
    cum = np.concatenate([np.zeros((1, Hkv, D)), np.cumsum(vf, axis=0)])
    start = ck[seq]
    with np.errstate(invalid="ignore", divide="ignore"):
        want = (cum[start + nrow] - cum[start]) / nrow[:, None, None]
    want = np.repeat(want, G, axis=1)                                    # [Tq, Hq, D]
    live = nrow > 0
    np.testing.assert_allclose(out[:Tq][live], want[live], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[:Tq][live], np.log(nrow[live])[:, None].repeat(Hq, 1),
                               rtol=0, atol=1e-14)
    assert np.all(out[:Tq][~live] == 0.0)
    assert np.all(np.isneginf(lse[:Tq][~live]))


def test_exhaustive_self_attention_placement():
    # every length tuple in [0, s]^B, s <= 8, B <= 4, q length = kv length
    groups = {}
    for s, B, lens, longer in self_attention_cases():
        if longer:
            continue      # the longer-buffer variant is checked separately below
        groups.setdefault((s, B), []).append(lens)
    for i, cases in enumerate(groups.values()):
        _check_packed_group(cases, cases, seed=i)


def test_exhaustive_cross_attention_placement():
    groups = {}
    for sq, sk, B, lq, lk in cross_attention_cases():
        g = groups.setdefault((sq, sk, B), ([], []))
        g[0].append(lq)
        g[1].append(lk)
    for i, (lq, lk) in enumerate(groups.values()):
        _check_packed_group(lq, lk, Hq=1, Hkv=1, D=4, seed=1000 + i)


def test_longer_cu_buffer_is_zero_length_padding():
    # the plan-sized form of a longer buffer: B_max + 1 entries, the unused
    # trailing sequences repeat the last offset (zero length) and write nothing
    D, Hq, Hkv = 64, 4, 2
    rng = np.random.default_rng(14)
    for lens in itertools.product(range(4), repeat=2):
        lens = list(lens)
        T = max(sum(lens), 1)
        q, k, v = rand_bits(rng, (T, Hq, D)), rand_bits(rng, (T, Hkv, D)), rand_bits(rng, (T, Hkv, D))
        o1, l1 = run(q, k, v, lens, lens, Hq, Hkv, D)
        o2, l2 = run(q, k, v, lens, lens, Hq, Hkv, D, B_max=5)
        np.testing.assert_array_equal(np.nan_to_num(o1, nan=3.0), np.nan_to_num(o2, nan=3.0))
        np.testing.assert_array_equal(np.nan_to_num(l1, nan=3.0), np.nan_to_num(l2, nan=3.0))


# ------------------------------------------------------------ paged K/V

def _paged_case(page_size, seed, fused=False):
    sh = W.Shape("paged", B=5, Hq=8, Hkv=2, D=64, max_q=3, s_max=70)
    batch = W.make_batch(sh, [1, 3, 2, 1, 2], [0, 70, 9, 16, 33], seed=seed)
    pc = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, page_size, sh.s_max, seed=seed, fused=fused)
    return sh, batch, pc


@pytest.mark.parametrize("page_size", [8, 16, 64])
def test_gather_pages_follows_the_block_table_by_loops(page_size):
    """Element by element: key j of sequence b is slot j % page_size of page
    block_table[b][j // page_size]; the packed offsets are the running sums of
    the lengths."""
    sh, batch, pc = _paged_case(page_size, seed=4)
    kc = W.bits(pc.k_cache)
    bt = pc.block_table.numpy()
    packed, cu = oracle.gather_pages(kc, bt, page_size, batch.cu_k, B=sh.B)
    lens = np.diff(batch.cu_k)
    assert cu.tolist() == [0] + list(np.cumsum(lens))
    for b in range(sh.B):
        for j in range(int(lens[b])):
            page, slot = int(bt[b][j // page_size]), j % page_size
            for hk in range(sh.Hkv):
                for d in range(0, sh.D, 7):
                    assert packed[cu[b] + j, hk, d] == kc[page, slot, hk, d]


@pytest.mark.parametrize("page_size,fused", [(8, False), (16, True), (64, False)])
def test_paged_attention_equals_packed(page_size, fused):
    """The same keys reached through a shuffled page table, with every slot no
    key uses holding NaN, give bit-identical results to the packed layout."""
    sh, batch, pc = _paged_case(page_size, seed=5, fused=fused)
    ref_o, ref_l = oracle.attention(W.bits(batch.q), W.bits(batch.k), W.bits(batch.v), batch.cu_q, batch.cu_k,
                                    B=sh.B, Hq=sh.Hq, Hkv=sh.Hkv, D=sh.D)
    o, l = oracle.attention_paged(W.bits(batch.q), W.bits(pc.k_cache), W.bits(pc.v_cache),
                                  pc.block_table.numpy(), page_size, batch.cu_q, batch.cu_k, B=sh.B, Hq=sh.Hq,
                                  Hkv=sh.Hkv, D=sh.D)
    assert np.array_equal(o, ref_o, equal_nan=True)
    assert np.array_equal(l, ref_l, equal_nan=True)
    assert np.all(np.isfinite(o[: int(batch.cu_q[-1])]))


def test_paged_attention_ignores_physical_placement():
    sh, batch, pc1 = _paged_case(16, seed=6)
    pc2 = W.paginate(batch.k, batch.v, batch.cu_k, sh.B, 16, sh.s_max, seed=99, spare_pages=11)
    assert not np.array_equal(pc1.block_table.numpy(), pc2.block_table.numpy())
    res = [oracle.attention_paged(W.bits(batch.q), W.bits(pc.k_cache), W.bits(pc.v_cache),
                                  pc.block_table.numpy(), 16, batch.cu_q, batch.cu_k, B=sh.B, Hq=sh.Hq,
                                  Hkv=sh.Hkv, D=sh.D) for pc in (pc1, pc2)]
    assert np.array_equal(res[0][0], res[1][0], equal_nan=True)
    assert np.array_equal(res[0][1], res[1][1], equal_nan=True)


def test_gather_pages_rejects_a_page_outside_the_cache():
    sh, batch, pc = _paged_case(16, seed=7)
    bt = pc.block_table.numpy().copy()
    bt[1, 2] = pc.k_cache.shape[0]                  # sequence 1 has 70 keys: its third page is used
    with pytest.raises(ValueError):
        oracle.gather_pages(W.bits(pc.k_cache), bt, 16, batch.cu_k, B=sh.B)


# ------------------------------------------------------------ merge of normalised parts

@pytest.mark.parametrize("n_parts", [1, 2, 3, 7])
def test_merge_lse_of_key_ranges_equals_whole(n_parts):
    """Attention over disjoint key ranges of each sequence (some ranges empty,
    one sequence without keys), merged from (out, lse) pairs, equals the
    attention over all keys."""
    sh = W.Shape("cp", B=5, Hq=8, Hkv=2, D=64, max_q=1, s_max=300)
    lk = [300, 5, 0, 2, 77]
    batch = W.make_batch(sh, [1] * 5, lk, seed=11)
    q, k, v = W.bits(batch.q), W.bits(batch.k), W.bits(batch.v)
    ref_o, ref_l = oracle.attention(q, k, v, batch.cu_q, batch.cu_k, B=sh.B, Hq=sh.Hq, Hkv=sh.Hkv, D=sh.D)
    outs, lses = [], []
    for r in range(n_parts):
        sel, lens = [], []
        for b in range(sh.B):
            a = int(batch.cu_k[b]) + lk[b] * r // n_parts
            e = int(batch.cu_k[b]) + lk[b] * (r + 1) // n_parts
            sel.extend(range(a, e))
            lens.append(e - a)
        cu = W.cu_from_lengths(np.array(lens))
        o, l = oracle.attention(q, k[sel], v[sel], batch.cu_q, cu, B=sh.B, Hq=sh.Hq, Hkv=sh.Hkv, D=sh.D)
        outs.append(o)
        lses.append(l)
    o, l = oracle.merge_lse(np.stack(outs), np.stack(lses))
    assert np.abs(o - ref_o).max() < 1e-12
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isneginf(l), np.isneginf(ref_l))
    assert np.abs(l[fin] - ref_l[fin]).max() < 1e-12
    assert np.all(o[~fin] == 0.0)


def test_merge_lse_weights_by_exponentiated_lse():
    """Two parts with lse ln 1 and ln 3 (weights 1/4 and 3/4), and a part
    with no key, which is ignored."""
    outs = np.array([[[1.0, 0.0]], [[0.0, 4.0]], [[np.nan, np.nan]]])
    lses = np.array([[0.0], [np.log(3.0)], [-np.inf]])
    o, l = oracle.merge_lse(outs, lses)
    assert np.allclose(o, [[0.25, 3.0]], atol=1e-15, rtol=0)
    assert abs(l[0] - np.log(4.0)) < 1e-15
