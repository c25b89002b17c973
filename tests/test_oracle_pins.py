"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

Every check here is fixed by the mathematics or by a hand-worked example:
closed forms, invariants, special cases that reduce to a library routine
(torch SDPA, logsumexp), and brute force by rank counting on tiny inputs.
They are chosen so that a plausible slip in the oracle (a dropped token, a
wrong divisor, a wrong head-to-group map, a flipped tie rule, a window
overlap) fails at least one of them.  No expected value comes from the CUDA
library.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle.oracle import bf16_bits, bf16_value

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = {}
    extra = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(" ")
            if key in ("select", "case"):
                extra.append(rest)
            else:
                rows[key] = rest
    return rows, extra


def _shape(rows):
    return {k: int(v) for k, v in (kv.split("=") for kv in rows["shape"].split())}


def _nums(s, dtype=float):
    return np.array([dtype(x) for x in s.split()])


def rank_count_topk(s, k):
    """Brute-force top-k by rank counting: j is kept iff fewer than k entries
    beat it, where i beats j when s_i > s_j, or s_i == s_j and i < j."""
    n = len(s)
    keep = []
    for j in range(n):
        beaten_by = sum(1 for i in range(n) if s[i] > s[j] or (s[i] == s[j] and i < j))
        if beaten_by < k:
            keep.append(j)
    return np.array(keep, np.int32)


def rnd_bits(rng, shape, scale=1.0):
    return bf16_bits(rng.standard_normal(shape) * scale)


def dyadic_bits(rng, shape, step=0.25, lim=4.0):
    x = np.clip(np.round(rng.standard_normal(shape) / step) * step, -lim, lim)
    return bf16_bits(x)


# --------------------------------------------------------------------------
# hand-worked examples


def test_golden_block_topk(oracle):
    rows, selects = _read_golden("block_topk_hand.txt")
    sh = _shape(rows)
    B, Hq, Hkv, D, T, bs = sh["B"], sh["Hq"], sh["Hkv"], sh["D"], sh["T"], sh["bs"]
    L = _nums(rows["seq_lens"], int).astype(np.int32)
    q = bf16_bits(_nums(rows["q"]).reshape(B, Hq, D))
    K = bf16_bits(_nums(rows["K"]).reshape(B, Hkv, T, D))
    S = oracle.block_summaries(K, L, bs)
    assert np.array_equal(S.reshape(-1), _nums(rows["summaries"]))
    s = oracle.block_scores(q, S, L, bs)
    assert np.array_equal(s.reshape(-1), _nums(rows["scores"]))
    for sel in selects:
        k, _, want = sel.partition(":")
        k = int(k)
        idx, cnt = oracle.select_blocks(q, K, L, bs, k)
        want = _nums(want, int)
        assert cnt[0, 0] == len(want)
        assert np.array_equal(idx[0, 0, :cnt[0, 0]], want)
        assert np.all(idx[0, 0, cnt[0, 0]:] == -1)


def test_golden_attention(oracle):
    rows, _ = _read_golden("attention_hand.txt")
    sh = _shape(rows)
    B, Hq, Hkv, D, T = sh["B"], sh["Hq"], sh["Hkv"], sh["D"], sh["T"]
    L = _nums(rows["seq_lens"], int).astype(np.int32)
    q = bf16_bits(_nums(rows["q"]).reshape(B, Hq, D))
    K = bf16_bits(_nums(rows["K"]).reshape(B, Hkv, T, D))
    V = bf16_bits(_nums(rows["V"]).reshape(B, Hkv, T, D))
    idx = _nums(rows["idx"], int).astype(np.int32).reshape(1, 1, -1)
    cnt = np.array([[idx.shape[-1]]], np.int32)
    out, lse, ws = oracle.attention(q, K, V, L, idx, cnt, 1, False, float(rows["scale"]))
    np.testing.assert_allclose(out.reshape(-1), _nums(rows["out"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse.reshape(-1), _nums(rows["lse"]), rtol=0, atol=1e-15)
    assert abs(ws[0, 0] - 1.0) < 1e-15


def test_golden_unified(oracle):
    rows, cases = _read_golden("unified_hand.txt")
    sh = _shape(rows)
    B, Hq, Hkv, D, T = sh["B"], sh["Hq"], sh["Hkv"], sh["D"], sh["T"]
    L = _nums(rows["seq_lens"], int).astype(np.int32)
    K = bf16_bits(_nums(rows["K"]).reshape(B, Hkv, T, D))
    for case in cases:
        head, _, want = case.partition(":")
        parts = head.split()
        qi = parts.index("q")
        vi = parts.index("votes")
        q = bf16_bits(np.array([float(x) for x in parts[qi + 1:vi]]).reshape(B, Hq, D))
        votes_want = np.array([int(x) for x in parts[vi + 1:]])
        idx, cnt, votes = oracle.unified_select(q, K, L, sh["P"], sh["budget"], sh["R"],
                                                want_votes=True)
        assert np.array_equal(votes[0], votes_want), parts[0]
        want = _nums(want, int)
        assert cnt[0] == len(want)
        assert np.array_equal(idx[0, :cnt[0]], want), parts[0]


# --------------------------------------------------------------------------
# A1 block summaries: closed forms


@pytest.mark.parametrize("bs", [1, 2, 16, 32])
def test_summaries_constant_blocks(oracle, bs):
    """Keys constant inside each block -> the mean is that constant, exactly,
    for full blocks and for a partial tail block."""
    rng = np.random.default_rng(11)
    B, Hkv, T, D = 3, 2, 5 * bs + 3, 8
    nb = -(-T // bs)
    consts = np.round(rng.standard_normal((B, Hkv, nb, D)) * 8) / 8  # exact in bf16
    K = np.repeat(consts, bs, axis=2)[:, :, :T]
    lens = np.array([T, T - 2, max(1, bs + 1)], np.int32)
    S = oracle.block_summaries(bf16_bits(K), lens, bs)
    for b in range(B):
        nbb = -(-lens[b] // bs)
        assert np.array_equal(S[b, :, :nbb], consts[b, :, :nbb])
        assert np.all(S[b, :, nbb:] == 0)


def test_summaries_arithmetic_series(oracle):
    """K[t] = a + t*c (dyadic): the mean of tokens [s, s+n) is a + c*(s + (n-1)/2).
    Catches a wrong start, a wrong count, or a divisor of bs on the tail."""
    rng = np.random.default_rng(12)
    bs, T, D = 16, 16 * 4, 4
    a = np.round(rng.standard_normal(D) * 4) / 4
    c = np.array([0.25, -0.5, 1.0, 0.125])
    t = np.arange(T)[:, None]
    K = (a[None, :] + t * c[None, :]).reshape(1, 1, T, D)
    for L in (T, T - 1, T - 15, 17, 1):
        S = oracle.block_summaries(bf16_bits(K), np.array([L], np.int32), bs)
        for j in range(-(-L // bs)):
            s0, n = j * bs, min(bs, L - j * bs)
            want = a + c * (s0 + (n - 1) / 2.0)
            np.testing.assert_allclose(S[0, 0, j], want, rtol=0, atol=1e-12)


def test_summaries_ignore_slots_past_length(oracle):
    rng = np.random.default_rng(13)
    K = rng.standard_normal((2, 2, 50, 8))
    lens = np.array([37, 50], np.int32)
    K2 = K.copy()
    K2[0, :, 37:] = 1e6
    S1 = oracle.block_summaries(bf16_bits(K), lens, 16)
    S2 = oracle.block_summaries(bf16_bits(K2), lens, 16)
    assert np.array_equal(S1, S2)


def test_summaries_single_token_tail(oracle):
    rng = np.random.default_rng(14)
    K = rnd_bits(rng, (1, 3, 33, 16))
    S = oracle.block_summaries(K, np.array([33], np.int32), 16)
    assert np.array_equal(S[0, :, 2], bf16_value(K[0, :, 32]))


# --------------------------------------------------------------------------
# A2 block scores: special cases and invariants


def test_scores_basis_queries_pick_components(oracle):
    """q_h = e_{i_h}: the score of block j is sum over the group's heads of
    S_j[i_h].  A wrong head->group map or a wrong dimension index changes it."""
    B, Hq, Hkv, D, bs = 1, 6, 2, 8, 4
    G = Hq // Hkv
    T = 5 * bs
    consts = np.arange(5 * Hkv * D, dtype=float).reshape(1, Hkv, 5, D)  # distinct values
    K = np.repeat(consts, bs, axis=2)
    comp = [[1, 5, 6], [0, 3, 7]]  # dims picked by the heads of group 0 and group 1
    q = np.zeros((B, Hq, D))
    for g in range(Hkv):
        for i, d in enumerate(comp[g]):
            q[0, g * G + i, d] = 1.0
    L = np.array([T], np.int32)
    S = oracle.block_summaries(bf16_bits(K), L, bs)
    s = oracle.block_scores(bf16_bits(q), S, L, bs)
    for g in range(Hkv):
        for j in range(5):
            assert s[0, g, j] == sum(consts[0, g, j, d] for d in comp[g])


def test_scores_linear_in_query(oracle):
    rng = np.random.default_rng(21)
    B, Hq, Hkv, D, T, bs = 2, 4, 2, 16, 64, 16
    K = dyadic_bits(rng, (B, Hkv, T, D))
    q1 = dyadic_bits(rng, (B, Hq, D))
    q2 = dyadic_bits(rng, (B, Hq, D))
    L = np.array([64, 50], np.int32)
    S = oracle.block_summaries(K, L, bs)
    s1 = oracle.block_scores(q1, S, L, bs)
    s2 = oracle.block_scores(q2, S, L, bs)
    s12 = oracle.block_scores(bf16_bits(bf16_value(q1) + bf16_value(q2)), S, L, bs)
    s_neg = oracle.block_scores(bf16_bits(-bf16_value(q1)), S, L, bs)
    fin = np.isfinite(s1)
    np.testing.assert_allclose(s12[fin], (s1 + s2)[fin], rtol=0, atol=1e-9)
    assert np.array_equal(s_neg[fin], -s1[fin])
    # blocks past the sequence end are never candidates
    assert np.all(np.isneginf(s1[1, :, 4:]))
    assert np.all(np.isfinite(s1[1, :, :4]))


# --------------------------------------------------------------------------
# A3 top-k: brute force by rank counting, dominance, ties


def test_topk_bruteforce_with_ties(oracle):
    rng = np.random.default_rng(31)
    for n in range(1, 41):
        for trial in range(3):
            s = rng.integers(-3, 4, size=n).astype(float)  # many exact ties
            for k in range(1, n + 3):
                got = oracle.topk(s, k)
                want = rank_count_topk(s, k)
                assert np.array_equal(got, want), (n, k, s)


def test_topk_dominance_random(oracle):
    rng = np.random.default_rng(32)
    for n, k in [(100, 7), (2048, 128), (513, 512), (8192, 512)]:
        s = np.round(rng.standard_normal(n) * 4) / 4
        sel = oracle.topk(s, k)
        assert len(sel) == k and np.all(np.diff(sel) > 0)
        mask = np.zeros(n, bool)
        mask[sel] = True
        lo = s[mask].min()
        assert np.all(s[~mask] <= lo)
        # at the boundary value, every kept index is below every dropped one
        kept_eq = np.nonzero(mask & (s == lo))[0]
        drop_eq = np.nonzero(~mask & (s == lo))[0]
        if len(drop_eq):
            assert kept_eq.max() < drop_eq.min()


def test_topk_all_when_k_covers(oracle):
    s = np.array([0.5, -1.0, 2.0])
    assert np.array_equal(oracle.topk(s, 3), [0, 1, 2])
    assert np.array_equal(oracle.topk(s, 10), [0, 1, 2])


def test_select_blocks_matches_bruteforce_on_scores(oracle):
    rng = np.random.default_rng(33)
    B, Hq, Hkv, D, T, bs, k = 3, 4, 2, 8, 100, 8, 5
    q = dyadic_bits(rng, (B, Hq, D))
    K = dyadic_bits(rng, (B, Hkv, T, D))
    L = np.array([100, 33, 7], np.int32)
    idx, cnt, scores = oracle.select_blocks(q, K, L, bs, k, want_scores=True)
    for b in range(B):
        nb = -(-L[b] // bs)
        for g in range(Hkv):
            want = rank_count_topk(list(scores[b, g, :nb]), k)
            assert cnt[b, g] == len(want)
            assert np.array_equal(idx[b, g, :cnt[b, g]], want)
            assert np.all(idx[b, g, cnt[b, g]:] == -1)


# --------------------------------------------------------------------------
# A4/A5/A8 attention: reduction to torch SDPA, invariants, closed forms


def _sdpa_fp64(q, K, V, scale):
    """torch SDPA in fp64 on the CPU, GQA by repeating each kv-head G times."""
    qt = torch.from_numpy(bf16_value(q))[:, :, None, :]  # [B,Hq,1,D]
    G = q.shape[1] // K.shape[1]
    Kt = torch.from_numpy(bf16_value(K)).repeat_interleave(G, dim=1)
    Vt = torch.from_numpy(bf16_value(V)).repeat_interleave(G, dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    logits = torch.einsum("bhqd,bhtd->bhqt", qt, Kt) * scale
    return out[:, :, 0].numpy(), torch.logsumexp(logits, -1)[:, :, 0].numpy()


@pytest.mark.parametrize("G,D,L", [(1, 64, 37), (2, 64, 300), (4, 128, 129)])
def test_dense_attention_equals_sdpa(oracle, G, D, L):
    rng = np.random.default_rng(41)
    B, Hkv = 2, 2
    Hq = G * Hkv
    q = rnd_bits(rng, (B, Hq, D))
    K = rnd_bits(rng, (B, Hkv, L, D))
    V = rnd_bits(rng, (B, Hkv, L, D))
    lens = np.array([L, L], np.int32)
    scale = 1.0 / math.sqrt(D)
    out, lse, ws = oracle.attention(q, K, V, lens)  # scale 0 -> 1/sqrt(D)
    ref, ref_lse = _sdpa_fp64(q, K, V, scale)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ws, 1.0, rtol=0, atol=1e-12)


def test_block_selection_attention_equals_sdpa_on_gathered(oracle):
    """Attention over selected blocks == SDPA over the gathered tokens, with a
    partial tail block (tokens past L dropped)."""
    rng = np.random.default_rng(42)
    B, Hq, Hkv, D, T, bs = 1, 4, 2, 64, 96, 16
    q = rnd_bits(rng, (B, Hq, D))
    K = rnd_bits(rng, (B, Hkv, T, D))
    V = rnd_bits(rng, (B, Hkv, T, D))
    L = 90  # block 5 holds 10 valid tokens
    idx = np.array([[[1, 3, 5, -1], [0, 5, -1, -1]]], np.int32)
    cnt = np.array([[3, 2]], np.int32)
    out, lse, _ = oracle.attention(q, K, V, np.array([L], np.int32), idx, cnt, bs)
    for g in range(Hkv):
        toks = [t for j in idx[0, g, :cnt[0, g]] for t in range(j * bs, min(j * bs + bs, L))]
        hs = slice(g * 2, g * 2 + 2)
        ref, ref_lse = _sdpa_fp64(q[:, hs], K[:, g:g + 1, toks], V[:, g:g + 1, toks],
                                  1.0 / math.sqrt(D))
        np.testing.assert_allclose(out[:, hs], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, hs], ref_lse, rtol=0, atol=1e-12)


def test_attention_convex_hull_and_weights(oracle):
    rng = np.random.default_rng(43)
    B, Hq, Hkv, D, T = 2, 8, 2, 64, 200
    q = rnd_bits(rng, (B, Hq, D), 3.0)  # peaked softmax
    K = rnd_bits(rng, (B, Hkv, T, D))
    V = rnd_bits(rng, (B, Hkv, T, D))
    lens = np.array([200, 150], np.int32)
    out, _, ws = oracle.attention(q, K, V, lens)
    np.testing.assert_allclose(ws, 1.0, rtol=0, atol=1e-12)
    Vv = bf16_value(V)
    for b in range(B):
        for h in range(Hq):
            rowsV = Vv[b, h // 4, :lens[b]]
            assert np.all(out[b, h] <= rowsV.max(0) + 1e-12)
            assert np.all(out[b, h] >= rowsV.min(0) - 1e-12)


def test_attention_single_token_and_zero_query(oracle):
    rng = np.random.default_rng(44)
    B, Hq, Hkv, D, T = 1, 2, 1, 64, 40
    q = rnd_bits(rng, (B, Hq, D))
    K = rnd_bits(rng, (B, Hkv, T, D))
    V = rnd_bits(rng, (B, Hkv, T, D))
    L = np.array([40], np.int32)
    idx = np.array([[[17]]], np.int32)
    out, lse, _ = oracle.attention(q, K, V, L, idx, np.array([[1]], np.int32), 1)
    assert np.array_equal(out[0, 0], bf16_value(V[0, 0, 17]))
    z = (bf16_value(q[0, 0]) * bf16_value(K[0, 0, 17])).sum() / 8.0
    assert abs(lse[0, 0] - z) < 1e-12
    # q = 0: uniform weights -> plain mean of the selected values, lse = log n
    q0 = np.zeros_like(q)
    idx = np.array([[[2, 5, 39, 11]]], np.int32)
    out, lse, _ = oracle.attention(q0, K, V, L, idx, np.array([[4]], np.int32), 1)
    want = bf16_value(V[0, 0, [2, 5, 39, 11]]).mean(0)
    np.testing.assert_allclose(out[0, 0], want, rtol=0, atol=1e-14)
    assert abs(lse[0, 0] - math.log(4)) < 1e-14


def test_attention_ignores_slots_past_length_and_shared_lists(oracle):
    rng = np.random.default_rng(45)
    B, Hq, Hkv, D, T = 2, 4, 2, 64, 64
    q = rnd_bits(rng, (B, Hq, D))
    K = rng.standard_normal((B, Hkv, T, D))
    V = rng.standard_normal((B, Hkv, T, D))
    lens = np.array([50, 64], np.int32)
    K2, V2 = K.copy(), V.copy()
    K2[0, :, 50:] = 1e4
    V2[0, :, 50:] = 1e4
    idx = np.array([[0, 10, 49, 55, 63], [1, 2, 3, 4, 63]], np.int32)  # row 0 lists t >= L
    cnt = np.array([5, 5], np.int32)
    a = oracle.attention(q, bf16_bits(K), bf16_bits(V), lens, idx, cnt, 1, True)
    b = oracle.attention(q, bf16_bits(K2), bf16_bits(V2), lens, idx, cnt, 1, True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    # a shared list equals the same list given to every kv-head
    per_head = np.repeat(idx[:, None, :], Hkv, axis=1)
    c = oracle.attention(q, bf16_bits(K), bf16_bits(V), lens, per_head,
                         np.repeat(cnt[:, None], Hkv, 1), 1, False)
    assert np.array_equal(a[0], c[0])


def test_attention_empty_selection(oracle):
    rng = np.random.default_rng(46)
    q = rnd_bits(rng, (1, 2, 64))
    K = rnd_bits(rng, (1, 1, 8, 64))
    out, lse, _ = oracle.attention(q, K, K, np.array([8], np.int32),
                                   np.full((1, 1, 4), -1, np.int32), np.array([[0]], np.int32), 1)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# --------------------------------------------------------------------------
# A6 LessIsMore unified selection: brute force and closed forms


def _bruteforce_unified(q, K, L, P, budget, R):
    qv, Kv = bf16_value(q), bf16_value(K)
    B, Hq, D = qv.shape
    Hkv = Kv.shape[1]
    G = Hq // Hkv
    res = []
    for b in range(B):
        if L[b] <= budget:
            res.append(list(range(L[b])))
            continue
        votes = np.zeros(L[b], int)
        for h in range(Hq):
            s = [float(np.dot(qv[b, h], Kv[b, h // G, t])) for t in range(L[b])]
            for t in rank_count_topk(s, P):
                votes[t] += 1
        cand = list(votes[:L[b] - R].astype(float))
        voted = rank_count_topk(cand, budget - R)
        res.append(sorted(list(voted) + list(range(L[b] - R, L[b]))))
    return res


def test_unified_bruteforce_small(oracle):
    rng = np.random.default_rng(51)
    for trial in range(12):
        B, Hkv, G, D = 2, 2, int(rng.integers(1, 4)), 4
        Hq = Hkv * G
        T = int(rng.integers(8, 64))
        q = dyadic_bits(rng, (B, Hq, D), step=0.5, lim=2.0)  # coarse grid -> exact ties
        K = dyadic_bits(rng, (B, Hkv, T, D), step=0.5, lim=2.0)
        L = np.array([T, int(rng.integers(1, T + 1))], np.int32)
        budget = int(rng.integers(1, T + 1))
        R = int(rng.integers(0, budget + 1))
        P = int(rng.integers(1, T + 2))
        idx, cnt = oracle.unified_select(q, K, L, P, budget, R)
        want = _bruteforce_unified(q, K, L, P, budget, R)
        for b in range(B):
            assert cnt[b] == len(want[b])
            assert list(idx[b, :cnt[b]]) == want[b], (trial, b)
            assert np.all(idx[b, cnt[b]:] == -1)


def test_unified_closed_forms(oracle):
    rng = np.random.default_rng(52)
    B, Hq, Hkv, D, T = 1, 8, 2, 16, 300
    K = dyadic_bits(rng, (B, Hkv, T, D))
    # identical keys for both kv-heads and one query for every head:
    # votes are 0 or Hq, the voted part is that head's top (budget - R) outside the window
    K[:, 1] = K[:, 0]
    q1 = dyadic_bits(rng, (1, 1, D))
    q = np.repeat(q1, Hq, axis=1)
    L = np.array([T], np.int32)
    P, budget, R = 60, 40, 10
    idx, cnt, votes = oracle.unified_select(q, K, L, P, budget, R, want_votes=True)
    assert set(np.unique(votes[0])) <= {0, Hq}
    assert votes[0].sum() == Hq * P
    s = list((bf16_value(q1[0, 0]) * bf16_value(K[0, 0])).sum(-1))
    head_pick = set(rank_count_topk(s, P))
    voted = [t for t in idx[0, :cnt[0]] if t < T - R]
    assert set(voted) <= head_pick and len(voted) == budget - R
    assert list(idx[0, cnt[0] - R:cnt[0]]) == list(range(T - R, T))
    # P >= L: every token gets Hq votes -> voted part is the lowest tokens
    qr = dyadic_bits(rng, (B, Hq, D))
    idx, cnt, votes = oracle.unified_select(qr, K, L, T + 5, budget, R, want_votes=True)
    assert np.all(votes[0] == Hq)
    assert list(idx[0, :cnt[0]]) == list(range(budget - R)) + list(range(T - R, T))
    # R = budget: pure recency window (the local-attention special case)
    idx, cnt = oracle.unified_select(qr, K, L, P, budget, budget)
    assert list(idx[0, :cnt[0]]) == list(range(T - budget, T))
    # budget >= L: every token
    idx, cnt = oracle.unified_select(qr, K, np.array([30], np.int32), P, budget, R)
    assert list(idx[0, :cnt[0]]) == list(range(30))
    # total votes = Hq * min(P, L)
    for P2 in (1, 17, 299, 300, 400):
        _, _, votes = oracle.unified_select(qr, K, L, P2, budget, R, want_votes=True)
        assert votes[0].sum() == Hq * min(P2, T)


def test_unified_window_excluded_from_voted_part(oracle):
    """Window tokens never take a voted slot: with all votes concentrated in the
    window, the voted part still has budget - R tokens outside it."""
    B, Hq, Hkv, D, T = 1, 2, 1, 4, 50
    K = np.zeros((B, Hkv, T, D))
    K[0, 0, 40:, 0] = 1.0  # the last 10 tokens score highest for q = e0
    q = np.zeros((B, Hq, D))
    q[0, :, 0] = 1.0
    idx, cnt = oracle.unified_select(bf16_bits(q), bf16_bits(K), np.array([T], np.int32), 10,
                                     20, 10)
    assert cnt[0] == 20
    assert list(idx[0]) == list(range(10)) + list(range(40, 50))


# ---------------------------------------------------------------------------
# bf16 storage of the block summaries (the nearest bf16, ties to even)


@pytest.mark.parametrize("x,bits", [
    (1.0, 0x3F80),
    (1.0 + 2.0 ** -8, 0x3F80),              # midway between 1 and 1 + 2^-7: the even one (1)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),          # midway between 0x3F81 and 0x3F82: the even one
    (1.0 + 2.0 ** -8 + 2.0 ** -30, 0x3F81), # just past the midpoint: up
    (-2.5, 0xC020),
    (0.0, 0x0000),
    (-0.0, 0x8000),
    ((2.0 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),  # the largest bf16
    (2.0 ** 128, 0x7F80),                    # past it: infinity
    (2.0 ** -133, 0x0001),                   # the smallest subnormal bf16
    (2.0 ** -134, 0x0000),                   # half of it: ties to even (zero)
    (3 * 2.0 ** -135, 0x0001),               # three quarters of it: up
])
def test_round_bf16_format_values(oracle, x, bits):
    """Bit patterns worked out from the bf16 format (1 sign, 8 exponent, 7 mantissa bits)."""
    assert int(oracle.round_bf16(np.array([x]))[0]) == bits


def test_round_bf16_matches_torch_on_binary32(oracle):
    """For binary32 inputs the nearest-even bf16 is torch's float32 -> bfloat16 conversion."""
    rng = np.random.default_rng(31)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-40, 40, 20000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_round_bf16_is_nearest_on_doubles(oracle):
    """Brute force on doubles: no neighbouring bf16 is closer; a tie picks the even pattern."""
    rng = np.random.default_rng(32)
    x = rng.standard_normal(5000) * np.exp2(rng.integers(-20, 20, 5000).astype(np.float64))
    got = oracle.round_bf16(x)
    for xi, bi in zip(x, got):
        b = int(bi)
        mag = b & 0x7FFF
        v = float(bf16_value(np.array([b], np.uint16))[0])
        for nb in (mag - 1, mag + 1):
            if 0 <= nb < 0x7F80:
                vn = float(bf16_value(np.array([(b & 0x8000) | nb], np.uint16))[0])
                assert abs(xi - v) <= abs(xi - vn)
                if abs(xi - v) == abs(xi - vn):
                    assert mag % 2 == 0


def test_select_blocks_bf16_storage_tie(oracle):
    """Block 1's mean (1 + 2^-8 in the only non-zero column) beats block 0's mean
    (exactly 1) in fp64, but both store as bf16 1.0: the tie goes to block 0."""
    D, bs = 64, 2
    K = np.zeros((1, 1, 4, D), np.float32)
    K[0, 0, 0:2, 0] = 1.0
    K[0, 0, 2, 0] = 1.0
    K[0, 0, 3, 0] = 1.0 + 2.0 ** -7
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, 0] = 1.0
    lens = np.array([4], np.int32)
    idx64, _ = oracle.select_blocks(bf16_bits(q), bf16_bits(K), lens, bs, 1)
    idx16, _ = oracle.select_blocks(bf16_bits(q), bf16_bits(K), lens, bs, 1, summary_bf16=True)
    assert idx64[0, 0, 0] == 1 and idx16[0, 0, 0] == 0


def test_select_blocks_bf16_storage_exact_means(oracle):
    """Keys on a 1/4 grid in [-2, 2] with blocks of 4 give means on a 1/16 grid, all exact
    in bf16: the stored summaries change nothing."""
    rng = np.random.default_rng(33)
    B, Hq, Hkv, D, T, bs = 2, 4, 2, 64, 160, 4
    K = np.clip(np.round(rng.standard_normal((B, Hkv, T, D)) * 4) / 4, -2, 2).astype(np.float32)
    q = np.round(rng.standard_normal((B, Hq, D)) * 4).astype(np.float32) / 4
    lens = np.array([T, 97], np.int32)
    S = oracle.block_summaries(bf16_bits(K), lens, bs)
    assert np.array_equal(bf16_value(oracle.round_bf16(S)), S)
    a = oracle.select_blocks(bf16_bits(q), bf16_bits(K), lens, bs, 7)
    b = oracle.select_blocks(bf16_bits(q), bf16_bits(K), lens, bs, 7, summary_bf16=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---------------------------------------------------------------------------
# paged KV cache: the logical cache the pages and the block table describe


def test_gather_pages_identity_table(oracle):
    """Pages laid out in row order with the identity table are the contiguous cache."""
    rng = np.random.default_rng(41)
    B, Hkv, D, bs, mb = 2, 3, 64, 16, 5
    K = rng.integers(0, 1 << 16, size=(B, Hkv, mb * bs, D), dtype=np.uint16)
    lens = np.array([mb * bs, 37], np.int32)
    # page b*mb + j holds block j of row b, all kv-heads
    pages = K.reshape(B, Hkv, mb, bs, D).transpose(0, 2, 1, 3, 4).reshape(B * mb, Hkv, bs, D)
    tbl = np.arange(B * mb, dtype=np.int32).reshape(B, mb)
    got = oracle.gather_pages(pages, tbl, lens)
    for b in range(B):
        assert np.array_equal(got[b, :, :lens[b]], K[b, :, :lens[b]])
        assert not got[b, :, lens[b]:].any()


def test_gather_pages_scatter_roundtrip_and_bad_pages(oracle):
    """A random page placement reproduces the cache it was scattered from; a block whose
    page id is out of range reads as zeros."""
    rng = np.random.default_rng(42)
    B, Hkv, D, bs, mb, P = 3, 2, 64, 32, 4, 20
    K = rng.integers(0, 1 << 16, size=(B, Hkv, mb * bs, D), dtype=np.uint16)
    lens = np.array([mb * bs, 70, 1], np.int32)
    tbl = rng.permutation(P)[:B * mb].astype(np.int32).reshape(B, mb)
    pages = rng.integers(0, 1 << 16, size=(P, Hkv, bs, D), dtype=np.uint16)
    for b in range(B):
        for j in range(mb):
            for g in range(Hkv):
                pages[tbl[b, j], g] = K[b, g, j * bs:(j + 1) * bs]
    got = oracle.gather_pages(pages, tbl, lens)
    for b in range(B):
        assert np.array_equal(got[b, :, :lens[b]], K[b, :, :lens[b]])
    tbl2 = tbl.copy()
    tbl2[0, 1] = P          # out of range
    tbl2[0, 2] = -1         # negative
    got2 = oracle.gather_pages(pages, tbl2, lens)
    assert not got2[0, :, bs:3 * bs].any()
    assert np.array_equal(got2[0, :, :bs], K[0, :, :bs])


def test_select_window_is_topk_of_a_recency_score(oracle):
    """Local attention as a block selection equals block top-k when the scores grow with
    the block index: keys of block j are j * c * u, with u the group's query direction."""
    rng = np.random.default_rng(51)
    B, Hq, Hkv, D, bs, nbk = 3, 4, 2, 64, 16, 12
    G = Hq // Hkv
    T = nbk * bs
    lens = np.array([T, 5 * bs + 3, 2 * bs], np.int32)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    K = np.zeros((B, Hkv, T, D), np.float32)
    for b in range(B):
        for g in range(Hkv):
            u = q[b, g * G:(g + 1) * G].sum(0)
            u /= np.linalg.norm(u)
            for j in range(nbk):
                K[b, g, j * bs:(j + 1) * bs] = (j + 1) * 0.25 * u
    for k in (1, 4, 12):
        want = oracle.select_blocks(bf16_bits(q), bf16_bits(K), lens, bs, k)
        got = oracle.select_window(lens, Hkv, bs, k)
        assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])


# ---------------------------------------------------------------------------
# per-head token top-k (token-level sparse attention, one set per query head)


def test_tokens_per_head_rank_counting(oracle):
    """Brute force on small inputs: every kept token has fewer than k tokens ranked above it
    (higher score, or equal score and lower index), and min(k, L) are kept."""
    rng = np.random.default_rng(61)
    B, Hq, Hkv, D, T = 2, 4, 2, 64, 90
    G = Hq // Hkv
    q = np.round(rng.standard_normal((B, Hq, D)) * 2) / 4      # coarse grid: exact ties
    K = np.round(rng.standard_normal((B, Hkv, T, D)) * 2) / 4
    lens = np.array([T, 37], np.int32)
    for k in (1, 10, 40, 200):
        idx, cnt = oracle.select_tokens_per_head(bf16_bits(q), bf16_bits(K), lens, k)
        for b in range(B):
            L = int(lens[b])
            for h in range(Hq):
                s = K[b, h // G, :L] @ q[b, h]
                n = int(cnt[b, h])
                assert n == min(k, L)
                got = idx[b, h, :n]
                assert np.all(np.diff(got) > 0) and np.all(idx[b, h, n:] == -1)
                for t in got:
                    above = np.sum((s > s[t]) | ((s == s[t]) & (np.arange(L) < t)))
                    assert above < k


def test_tokens_per_head_equal_heads_match_unified_votes(oracle):
    """With every query head identical, each head's top-k is the set every head votes for,
    so it is the LessIsMore selection with budget k and no window."""
    rng = np.random.default_rng(62)
    B, Hq, Hkv, D, T, k = 2, 4, 1, 64, 300, 50
    q1 = rng.standard_normal((B, 1, D)).astype(np.float32)
    q = np.repeat(q1, Hq, axis=1)
    K = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    lens = np.array([T, 120], np.int32)
    idx, cnt = oracle.select_tokens_per_head(bf16_bits(q), bf16_bits(K), lens, k)
    uni, ucnt = oracle.unified_select(bf16_bits(q), bf16_bits(K), lens, k, k, 0)
    for h in range(Hq):
        assert np.array_equal(idx[:, h], uni) and np.array_equal(cnt[:, h], ucnt)


# ---------------------------------------------------------------------------
# random-head aggregation (one head's set shared by every head)


def test_one_head_set_is_that_heads_brute_force_topk(oracle):
    """Brute force on small inputs with distinct heads and exact ties: row b's set is the
    min(k, L) tokens of the chosen head ranked first by (score desc, index asc), ascending."""
    rng = np.random.default_rng(63)
    B, Hq, Hkv, D, T = 3, 8, 2, 64, 80
    G = Hq // Hkv
    q = np.round(rng.standard_normal((B, Hq, D)) * 2) / 4      # coarse grid: exact ties
    K = np.round(rng.standard_normal((B, Hkv, T, D)) * 2) / 4
    lens = np.array([T, 45, 3], np.int32)
    heads = np.array([5, 2, 7], np.int32)
    for k in (1, 9, 30, 100):
        idx, cnt = oracle.select_tokens_one_head(bf16_bits(q), bf16_bits(K), lens, heads, k)
        assert idx.shape == (B, k) and cnt.shape == (B,)
        for b in range(B):
            L, h = int(lens[b]), int(heads[b])
            s = (K[b, h // G, :L].astype(np.float64) @ q[b, h].astype(np.float64))
            order = sorted(range(L), key=lambda t: (-s[t], t))
            want = np.sort(np.array(order[:min(k, L)], np.int32))
            assert cnt[b] == len(want)
            assert np.array_equal(idx[b, :cnt[b]], want) and np.all(idx[b, cnt[b]:] == -1)


def test_one_head_set_with_equal_heads_is_the_unified_set(oracle):
    """With every query head identical, any chosen head's top-k is the set all heads vote
    for: the LessIsMore selection with budget k and no window."""
    rng = np.random.default_rng(64)
    B, Hq, Hkv, D, T, k = 2, 4, 1, 64, 300, 40
    q = np.repeat(rng.standard_normal((B, 1, D)).astype(np.float32), Hq, axis=1)
    K = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    lens = np.array([T, 90], np.int32)
    uni, ucnt = oracle.unified_select(bf16_bits(q), bf16_bits(K), lens, k, k, 0)
    for heads in ([0, 3], [2, 1]):
        idx, cnt = oracle.select_tokens_one_head(bf16_bits(q), bf16_bits(K), lens,
                                                 np.array(heads, np.int32), k)
        assert np.array_equal(idx, uni) and np.array_equal(cnt, ucnt)


def test_one_head_rejects_heads_out_of_range(oracle):
    q = np.zeros((1, 4, 64), np.uint16)
    K = np.zeros((1, 2, 16, 64), np.uint16)
    with pytest.raises(ValueError):
        oracle.select_tokens_one_head(q, K, np.array([16], np.int32), np.array([4], np.int32), 2)


# --------------------------------------------------------------------------
# attention recall (LessIsMore press summary, sections 3 and 4)


def test_golden_recall(oracle):
    rows, cases = _read_golden("recall_hand.txt")
    sh = _shape(rows)
    B, Hq, Hkv, D, T = sh["B"], sh["Hq"], sh["Hkv"], sh["D"], sh["T"]
    L = _nums(rows["seq_lens"], int).astype(np.int32)
    q = bf16_bits(_nums(rows["q"]).reshape(B, Hq, D))
    K = bf16_bits(_nums(rows["K"]).reshape(B, Hkv, T, D))
    for case in cases:
        sel, _, want = case.partition(":")
        idx = _nums(sel, int).astype(np.int32).reshape(1, -1)
        cnt = np.array([idx.shape[-1]], np.int32)
        r = oracle.attention_recall(q, K, L, idx, cnt, 1, 1, float(rows["scale"]))
        np.testing.assert_allclose(r.reshape(-1), _nums(want), rtol=0, atol=1e-15)


def test_recall_of_every_token_is_one_and_of_none_is_zero(oracle):
    rng = np.random.default_rng(71)
    B, Hq, Hkv, D, T, bs = 2, 6, 3, 32, 90, 16
    q, K = rnd_bits(rng, (B, Hq, D), 2.0), rnd_bits(rng, (B, Hkv, T, D))
    L = np.array([90, 37], np.int32)
    nb = -(-T // bs)
    idx = np.tile(np.arange(nb, dtype=np.int32), (B, Hkv, 1))
    cnt = np.tile(-(-L // bs)[:, None], (1, Hkv)).astype(np.int32)
    np.testing.assert_allclose(oracle.attention_recall(q, K, L, idx, cnt, bs), 1.0, atol=1e-13)
    none = np.zeros((B, Hkv), np.int32)
    assert np.all(oracle.attention_recall(q, K, L, idx, none, bs) == 0.0)
    # slots past L_b (block 2 holds tokens 32..47 of the 37-token row) count once, if at all
    np.testing.assert_allclose(oracle.attention_recall(q, K, L, idx, cnt * 0 + nb, bs), 1.0,
                               atol=1e-13)


def test_recall_is_the_lse_difference(oracle):
    """Mass on a set = exp(lse(set) - lse(all)): the log-sum-exps come from the attention
    routine (itself pinned against torch SDPA), a separate computation."""
    rng = np.random.default_rng(72)
    B, Hq, Hkv, D, T = 2, 8, 2, 64, 200
    q, K, V = (rnd_bits(rng, s) for s in [(B, Hq, D), (B, Hkv, T, D), (B, Hkv, T, D)])
    L = np.array([200, 131], np.int32)
    k = 17
    idx = np.full((B, Hkv, k), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        for g in range(Hkv):
            m = 9 + 4 * g + b
            idx[b, g, :m] = np.sort(rng.choice(int(L[b]), size=m, replace=False))
            cnt[b, g] = m
    r = oracle.attention_recall(q, K, L, idx, cnt, 1, 0)
    _, lse_all, _ = oracle.attention(q, K, V, L)
    _, lse_sel, _ = oracle.attention(q, K, V, L, idx, cnt, 1)
    np.testing.assert_allclose(r, np.exp(lse_sel - lse_all), rtol=1e-12, atol=0)
    # the same selections as one list per query head (each head of a group repeats its
    # kv-head's list), and as one shared list when every kv-head has the same list
    G = Hq // Hkv
    per_q = np.repeat(idx, G, axis=1)
    per_q_cnt = np.repeat(cnt, G, axis=1)
    np.testing.assert_allclose(oracle.attention_recall(q, K, L, per_q, per_q_cnt, 1, 2), r,
                               rtol=0, atol=0)
    shared = oracle.attention_recall(q, K, L, idx[:, 0], cnt[:, 0], 1, 1)
    same = oracle.attention_recall(q, K, L, np.repeat(idx[:, :1], Hkv, 1),
                                   np.repeat(cnt[:, :1], Hkv, 1), 1, 0)
    np.testing.assert_allclose(shared, same, rtol=0, atol=0)


def test_recall_with_huge_logits(oracle):
    """Logits near 1000: the dense weights must still be formed stably (e^1024 overflows
    fp64).  Weights are proportional to (1, e^-64, e^-128)."""
    q = bf16_bits(np.array([[[64.0, 0.0]]]))
    K = bf16_bits(np.array([[[[16.0, 0.0], [15.0, 0.0], [14.0, 0.0]]]]))
    L = np.array([3], np.int32)
    one = np.array([[[0]]], np.int32), np.array([[1]], np.int32)
    mid = np.array([[[1]]], np.int32), np.array([[1]], np.int32)
    r0 = oracle.attention_recall(q, K, L, *one, 1, 0, 1.0)
    r1 = oracle.attention_recall(q, K, L, *mid, 1, 0, 1.0)
    assert np.isfinite(r0).all() and np.isfinite(r1).all()
    assert r0[0, 0] == pytest.approx(1.0, abs=1e-15)
    assert r1[0, 0] == pytest.approx(math.exp(-64) / (1 + math.exp(-64) + math.exp(-128)),
                                     rel=1e-12)



# --------------------------------------------------------------------------
# fp8 (e4m3) block summaries: the stored form of a block mean (reading R13)


def _e4m3_grid():
    """Every finite non-negative e4m3 value, from the format's definition: normal
    (1 + m/8) 2^(E-7) for E = 1..15 (not E = 15, m = 7), subnormal (m/8) 2^-6."""
    vals = [(m / 8) * 2.0 ** -6 for m in range(8)]
    vals += [(1 + m / 8) * 2.0 ** (E - 7) for E in range(1, 16) for m in range(8)
             if not (E == 15 and m == 7)]
    return np.array(vals)


@pytest.mark.parametrize("x,want", [
    (1.0, 1.0), (448.0, 448.0), (500.0, 448.0), (-1e9, -448.0),
    (2.0 ** -9, 2.0 ** -9),              # the smallest subnormal
    (2.0 ** -10, 0.0),                   # halfway to 0: even (0)
    (3 * 2.0 ** -10, 2 * 2.0 ** -9),     # halfway between 1 and 2 units: even (2)
    (1.0625, 1.0),                       # 1 + 1/16: halfway, even mantissa 0
    (1.1875, 1.25),                      # 1 + 3/16: halfway, even mantissa 2
    (-7.5, -7.5), (0.0703125, 0.0703125), (240.0, 240.0), (232.0, 224.0),
])
def test_round_e4m3_format_values(oracle, x, want):
    assert oracle.round_e4m3(x) == want


def test_round_e4m3_is_the_nearest_grid_value(oracle):
    """Brute force over the grid: the nearest value, ties to the even mantissa (the even
    index in the ordered grid)."""
    grid = _e4m3_grid()
    rng = np.random.default_rng(81)
    xs = np.concatenate([rng.uniform(0, 448, 3000), np.exp2(rng.uniform(-11, 8.8, 3000)),
                         (grid[:-1] + grid[1:]) / 2])  # every midpoint
    for x in xs:
        d = np.abs(grid - x)
        best = np.flatnonzero(d == d.min())
        want = grid[best[0]] if len(best) == 1 else grid[[i for i in best if i % 2 == 0][0]]
        assert oracle.round_e4m3(x) == want, x
        assert oracle.round_e4m3(-x) == -want


def test_round_e4m3_matches_torch(oracle):
    """torch's float8_e4m3fn cast rounds to nearest even as well (values within +-448)."""
    rng = np.random.default_rng(82)
    x = np.clip(rng.standard_normal(20000) * np.exp2(rng.integers(-12, 9, 20000)), -448, 448)
    t = torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_e4m3(x), t)


def test_e4m3_scale_exponent(oracle):
    """e is the smallest exponent with amax <= 448 2^e."""
    for e in range(-20, 10):
        assert oracle.e4m3_scale_exp(448.0 * 2.0 ** e) == e
        assert oracle.e4m3_scale_exp(np.nextafter(448.0 * 2.0 ** e, np.inf)) == e + 1
    rng = np.random.default_rng(83)
    for amax in np.exp2(rng.uniform(-30, 20, 500)):
        e = oracle.e4m3_scale_exp(amax)
        assert 448.0 * 2.0 ** (e - 1) < amax <= 448.0 * 2.0 ** e
    assert oracle.e4m3_scale_exp(0.0) == 0


def test_store_fp8_blocks(oracle):
    """Each block is scaled by its own power of two: the largest |mean| lands in
    (224, 448], every stored value is an e4m3 value times 2^e, and blocks whose means are
    already such values are stored exactly."""
    rng = np.random.default_rng(84)
    S = rng.standard_normal((5, 3, 128)) * np.exp2(rng.integers(-6, 6, (5, 3, 1)))
    T = oracle.store_fp8(S)
    grid = np.concatenate([-_e4m3_grid()[::-1], _e4m3_grid()])
    for blk, out in zip(S.reshape(-1, 128), T.reshape(-1, 128)):
        e = oracle.e4m3_scale_exp(np.abs(blk).max())
        assert 224.0 < np.abs(blk).max() / 2.0 ** e <= 448.0
        assert np.all(np.isin(out / 2.0 ** e, grid))
        assert np.max(np.abs(out - blk) / 2.0 ** e) <= 16.0  # half a spacing at 448 * 2^e
    exact = np.array([[1.0, -0.5, 0.375, 448.0 / 64]])  # e4m3 values times 2^-6
    np.testing.assert_array_equal(oracle.store_fp8(exact), exact)


def test_select_blocks_fp8_storage(oracle):
    """Stored as fp8, block means change the ranking where the rounding moves a score past
    another, and not where every mean is stored exactly."""
    D, bs = 4, 2
    q = bf16_bits(np.array([[[1.0, 0, 0, 0]]]))
    # every block's largest mean is 8: scale 2^-5 (8 <= 448 2^-5 = 14 < 2 * 8), so the first
    # mean x is stored as round_e4m3(32 x) / 32, on a grid of 4 / 32 = 1/8 in [1, 2):
    #   1.0625 -> 34, halfway between 32 and 36: the even mantissa, 32 -> 1.0
    #   1.09375 -> 35 -> 36 -> 1.125;  1.125 -> 36 -> 1.125 (exact)
    K = np.zeros((1, 1, 6, D))
    K[0, 0, 0:2] = [1.0625, 8, 0, 0]
    K[0, 0, 2:4] = [1.09375, 8, 0, 0]
    K[0, 0, 4:6] = [1.125, 8, 0, 0]
    K = bf16_bits(K)
    L = np.array([6], np.int32)
    idx, _, s_exact = oracle.select_blocks(q, K, L, bs, 1, want_scores=True)
    idx8, _, s8 = oracle.select_blocks(q, K, L, bs, 1, want_scores=True, summary_fp8=True)
    assert list(idx[0, 0]) == [2]                 # 1.125 is the best exact mean
    assert s8[0, 0, 1] == s8[0, 0, 2] == 1.125    # 1.09375 is stored as 1.125: a tie ...
    assert list(idx8[0, 0]) == [1]                # ... that the lower block wins
    # means that are e4m3 values times 2^e are stored exactly: the exact path's result
    K2 = bf16_bits(np.array([[[[0.5, 4, 0, 0], [0.5, 4, 0, 0], [0.25, 2, 0, 0], [0.25, 2, 0, 0]]]]))
    i_a, _ = oracle.select_blocks(q, K2, np.array([4], np.int32), bs, 1)
    i_b, _ = oracle.select_blocks(q, K2, np.array([4], np.int32), bs, 1, summary_fp8=True)
    assert np.array_equal(i_a, i_b)
