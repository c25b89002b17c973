"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Selected indices must match bit-exactly (inputs carry a planted score gap, or
are dyadic so that every score is exact in fp32); attention outputs must meet
max|d| <= 2e-3 and max|d| / max|ref| <= 1e-2, lse within 1e-4.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from block_top_sparse_ksa_b200 import synth
from oracle.oracle import bf16_bits, bf16_value
from tests.helpers import (DELTA, LSE_TOL, assert_out_close, gap_fix_row, min_boundary_gap,
                           sample_rows)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ksa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_top_sparse_ksa_b200 as k
    k.lib()
    return k


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return synth.bits(t)


def rand_bits(rng, shape, scale=1.0):
    return bf16_bits(rng.standard_normal(shape) * scale)


def dyadic_bits(rng, shape, step=0.25, lim=4.0):
    return bf16_bits(np.clip(np.round(rng.standard_normal(shape) / step) * step, -lim, lim))


def status_tensor():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


# ---------------------------------------------------------------------------
# A1 summaries


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [16, 32, 64])
def test_summaries_all_and_last_block(ksa, oracle, D, bs):
    rng = np.random.default_rng(100 + D + bs)
    B, Hkv, T = 4, 3, 7 * bs + 5
    K = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([T, 1, bs + 3, 5 * bs], np.int32)
    Kd, Ld = to_dev_bf16(K), torch.from_numpy(lens).to(DEV)
    S = ksa.ksa_build_block_summaries(Kd, Ld, bs).cpu().numpy()
    ref = oracle.block_summaries(K, lens, bs)
    for b in range(B):
        nb = -(-lens[b] // bs)
        np.testing.assert_allclose(S[b, :, :nb], ref[b, :, :nb], rtol=1e-6, atol=1e-6)
    # LAST_BLOCK rewrites only block NB_b - 1
    S2 = torch.full_like(torch.from_numpy(S), float("nan")).to(DEV)
    ksa.ksa_build_block_summaries(Kd, Ld, bs, ksa.SUMMARY_LAST_BLOCK, summaries=S2)
    S2 = S2.cpu().numpy()
    for b in range(B):
        nb = -(-lens[b] // bs)
        np.testing.assert_allclose(S2[b, :, nb - 1], ref[b, :, nb - 1], rtol=1e-6, atol=1e-6)
        assert np.all(np.isnan(S2[b, :, :nb - 1])) and np.all(np.isnan(S2[b, :, nb:]))


# ---------------------------------------------------------------------------
# A2 + A3 selection


def _select_case(ksa, oracle, rng, B, Hq, Hkv, D, T, bs, k, lens, dyadic=False, plant=True):
    q = dyadic_bits(rng, (B, Hq, D)) if dyadic else rand_bits(rng, (B, Hq, D))
    K = dyadic_bits(rng, (B, Hkv, T, D)) if dyadic else rand_bits(rng, (B, Hkv, T, D))
    if plant:
        for b in range(B):
            K[b], _ = gap_fix_row(oracle, q[b], K[b], int(lens[b]), bs, k)
            assert min_boundary_gap(oracle, q[b], K[b], int(lens[b]), bs, k) >= DELTA
    qd, Kd, Ld = to_dev_bf16(q), to_dev_bf16(K), torch.from_numpy(lens).to(DEV)
    st = status_tensor()
    S = ksa.ksa_build_block_summaries(Kd, Ld, bs, dev_status=st)
    idx, cnt = ksa.ksa_select_blocks(qd, S, Ld, bs, T, k, dev_status=st)
    ref_idx, ref_cnt = oracle.select_blocks(q, K, lens, bs, k)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert st.item() == 0
    return q, K, idx, cnt


@pytest.mark.parametrize("D,bs,k", [(128, 16, 8), (64, 32, 5), (128, 64, 3), (128, 16, 64)])
def test_select_blocks_planted_gap(ksa, oracle, D, bs, k):
    rng = np.random.default_rng(200 + k)
    B, Hq, Hkv, T = 3, 8, 2, 40 * bs + 7
    lens = np.array([T, 13 * bs + 1, 3 * bs], np.int32)  # ragged, a 1-token tail, a short row
    _select_case(ksa, oracle, rng, B, Hq, Hkv, D, T, bs, k, lens)


@pytest.mark.parametrize("nblk", [256, 700, 1100, 3000, 7000, 16384])
def test_select_blocks_exact_ties(ksa, oracle, nblk):
    """Dyadic inputs, full blocks: every score is exact in fp32, many tie
    exactly, and both sides must break ties toward the lower block.  Rows of
    up to 1024 blocks are ranked one warp per row (256 and 700 here); longer
    rows one CTA per row with 8, 16, 32 or 64 keys per thread (1100, 3000,
    7000, and 16384 blocks, the largest row the API accepts).  k runs up to
    512, the largest budget of the sweep (8192 tokens in blocks of 16)."""
    rng = np.random.default_rng(210 + nblk)
    B, Hq, Hkv, D, bs = 2, 4, 2, 128, 16
    T = nblk * bs
    lens = np.array([T, 100 * bs], np.int32)
    q = bf16_bits(np.round(rng.standard_normal((B, Hq, D))) * 0.25)
    K = bf16_bits(np.clip(np.round(rng.standard_normal((B, Hkv, T, D)) * 0.5), -2, 2) * 0.25)
    qd, Kd, Ld = to_dev_bf16(q), to_dev_bf16(K), torch.from_numpy(lens).to(DEV)
    S = ksa.ksa_build_block_summaries(Kd, Ld, bs)
    for k in (1, 7, 50, 99, 100, 255, 256, 512):
        idx, cnt = ksa.ksa_select_blocks(qd, S, Ld, bs, T, k)
        ref_idx, ref_cnt, scores = oracle.select_blocks(q, K, lens, bs, k, want_scores=True)
        assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
        assert np.array_equal(idx.cpu().numpy(), ref_idx), k
    nb = lens[0] // bs
    assert len(np.unique(scores[0, 0, :nb])) < nb  # ties really occur


def test_select_all_blocks_when_k_covers(ksa, oracle):
    rng = np.random.default_rng(220)
    B, Hq, Hkv, D, T, bs = 2, 4, 4, 64, 300, 32
    lens = np.array([300, 31], np.int32)
    _select_case(ksa, oracle, rng, B, Hq, Hkv, D, T, bs, 10, lens, plant=False)


# ---------------------------------------------------------------------------
# A4 + A5 attention


def _attn_check(ksa, oracle, q, K, V, lens, idx=None, cnt=None, tpi=1, shared=False,
                out_dtype=0):
    qd, Kd, Vd = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V)
    Ld = torch.from_numpy(lens).to(DEV)
    idx_d = None if idx is None else torch.from_numpy(np.ascontiguousarray(idx)).to(DEV)
    cnt_d = None if cnt is None else torch.from_numpy(np.ascontiguousarray(cnt)).to(DEV)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=DEV)
    st = status_tensor()
    out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, Ld, idx_d, cnt_d, tokens_per_idx=tpi,
                                        idx_shared=shared, out_dtype=out_dtype, lse=lse,
                                        dev_status=st)
    ref, ref_lse, _ = oracle.attention(q, K, V, lens, idx, cnt, tpi, shared)
    assert_out_close(out.float().cpu().numpy(), ref, bf16_output=(out_dtype == 1))
    got_lse = lse.cpu().numpy()
    fin = np.isfinite(ref_lse)
    np.testing.assert_allclose(got_lse[fin], ref_lse[fin], rtol=0, atol=LSE_TOL)
    assert np.all(np.isneginf(got_lse[~fin]))
    return st.item()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_dense_attention(ksa, oracle, D, G):
    rng = np.random.default_rng(300 + D + G)
    B, Hkv, T = 3, 2, 700
    q = rand_bits(rng, (B, G * Hkv, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([700, 33, 1], np.int32)
    assert _attn_check(ksa, oracle, q, K, V, lens) == 0


@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("out_dtype", [0, 1])
def test_block_list_attention(ksa, oracle, bs, out_dtype):
    rng = np.random.default_rng(400 + bs)
    B, Hq, Hkv, D = 3, 8, 2, 128
    T = 50 * bs + 9
    q = rand_bits(rng, (B, Hq, D), 2.0)  # peaked softmax
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([T, 20 * bs + 3, 5], np.int32)
    cap = 24
    idx = np.full((B, Hkv, cap), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        nb = -(-lens[b] // bs)
        for g in range(Hkv):
            n = min(cap - g, nb)
            sel = np.sort(rng.choice(nb, size=n, replace=False))
            if b == 1:  # always include the partial tail block
                sel = np.unique(np.append(sel[:-1], nb - 1))
                n = len(sel)
            idx[b, g, :n] = sel
            cnt[b, g] = n
    assert _attn_check(ksa, oracle, q, K, V, lens, idx, cnt, bs, out_dtype=out_dtype) == 0


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("tpi", [1, 4, 16])
def test_token_list_attention_shared(ksa, oracle, D, tpi):
    rng = np.random.default_rng(500 + D + tpi)
    B, Hq, Hkv = 2, 16, 4
    T = 3000
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([3000, 1999], np.int32)
    cap = 700 // tpi
    idx = np.full((B, cap), -1, np.int32)
    cnt = np.zeros((B,), np.int32)
    for b in range(B):
        n_units = -(-lens[b] // tpi)
        n = cap - 3 * b
        idx[b, :n] = np.sort(rng.choice(n_units, size=n, replace=False))
        cnt[b] = n
    assert _attn_check(ksa, oracle, q, K, V, lens, idx, cnt, tpi, shared=True) == 0


# Row counts, in SMs, that reach each way the attention launch splits its work (for one
# query-head group of 4 at head_dim 128, three CTAs per SM, two in the deep form): rows cut
# into equal parts, one deep CTA per row, one CTA per row, two whole rows per deep CTA, and
# the stream-K split (an odd count, and more rows than two deep grids hold).
PARTITION_ROWS = [(0.5, 0), (2.0, -8), (3.0, -4), (4.0, -16), (4.0, -15), (5.0, 0)]


@pytest.mark.parametrize("D,Hq", [(128, 4), (64, 8)])
@pytest.mark.parametrize("tpi", [16, 1])
@pytest.mark.parametrize("per_sm,extra", PARTITION_ROWS)
def test_attention_partition_forms(ksa, oracle, D, Hq, tpi, per_sm, extra):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B = max(1, int(per_sm * sms) + extra)
    rng = np.random.default_rng(900 + B + tpi + D)
    Hkv, T = 1, 320
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = rng.integers(T // 2, T + 1, size=B).astype(np.int32)
    lens[0], lens[-1] = T, 7
    cap = 6 if tpi == 16 else 48
    idx = np.full((B, Hkv, cap), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        units = -(-int(lens[b]) // tpi)
        n = int(rng.integers(1, min(cap, units) + 1))
        idx[b, 0, :n] = np.sort(rng.choice(units, size=n, replace=False))
        cnt[b, 0] = n
    assert _attn_check(ksa, oracle, q, K, V, lens, idx, cnt, tpi) == 0


def _list_with_runs(rng, n_units, cap, tpi, past_end=0):
    """Ascending distinct units: a recency window ending at the last unit, runs of 15 to
    100 tokens at unaligned starts, scattered singles up to cap, and `past_end` units
    beyond the row's end."""
    w = min(n_units, cap // 3)
    picks = set(range(n_units - w, n_units + past_end))
    for ln in (15, 16, 17, 33, 48, 100):
        u = -(-ln // tpi)
        s = int(rng.integers(0, max(1, n_units - w - u)))
        picks.update(range(s, min(s + u, n_units)))
    rest = np.setdiff1d(np.arange(n_units), np.fromiter(picks, np.int64))
    extra = cap - len(picks)
    if extra > 0:
        picks.update(rng.choice(rest, size=min(extra, len(rest)), replace=False).tolist())
    out = np.sort(np.fromiter(picks, np.int64)).astype(np.int32)
    assert len(out) <= cap
    return out


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("tpi", [1, 4])
def test_token_list_runs_of_consecutive_rows(ksa, oracle, D, tpi):
    """Token lists holding runs (a recency window, adjacent picks, runs that start and end
    inside a stage) next to scattered picks; one row's list runs past its end."""
    rng = np.random.default_rng(520 + D + tpi)
    B, Hq, Hkv = 3, 16, 4
    T = 3000
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([3000, 1999, 2500], np.int32)
    cap = 900 // tpi
    idx = np.full((B, cap), -1, np.int32)
    cnt = np.zeros((B,), np.int32)
    for b in range(B):
        lst = _list_with_runs(rng, -(-int(lens[b]) // tpi), cap, tpi, past_end=2 if b == 1 else 0)
        idx[b, :len(lst)] = lst
        cnt[b] = len(lst)
    st = _attn_check(ksa, oracle, q, K, V, lens, idx, cnt, tpi, shared=True)
    assert st == 2  # KSA_FLAG_INDEX_SKIPPED, from row 1's entries past its end


@pytest.mark.parametrize("Hkv", [1, 2])
def test_paged_token_list_runs(ksa, oracle, Hkv):
    """Paged pools with runs of consecutive tokens that cross page boundaries, on pages in
    sequence (with one kv-head, consecutive pool rows) and on shuffled pages: the result
    equals the contiguous cache's bit for bit and the oracle's."""
    rng = np.random.default_rng(1350 + Hkv)
    B, Hq, D, bs, mb = 2, 8, 128, 16, 60
    T = mb * bs
    lens = np.array([T, 37 * bs + 5], np.int32)
    n_pages = B * mb + 7
    K_pages = rand_bits(rng, (n_pages, Hkv, bs, D))
    V_pages = rand_bits(rng, (n_pages, Hkv, bs, D))
    # row 0's pages in sequence, row 1's in sequence for its first half, then shuffled
    tbl = np.zeros((B, mb), np.int32)
    tbl[0] = np.arange(mb)
    tail = mb + np.arange(mb)
    tail[mb // 2:] = rng.permutation(tail[mb // 2:])
    tbl[1] = tail
    K = oracle.gather_pages(K_pages, tbl, lens)
    V = oracle.gather_pages(V_pages, tbl, lens)
    q = rand_bits(rng, (B, Hq, D))
    cap = 400
    lst = np.full((B, cap), -1, np.int32)
    n_t = np.zeros((B,), np.int32)
    for b in range(B):
        pick = _list_with_runs(rng, int(lens[b]), cap, 1)
        lst[b, :len(pick)] = pick
        n_t[b] = len(pick)
    qd, Ld = to_dev_bf16(q), torch.from_numpy(lens).to(DEV)
    Kp, Vp = to_dev_bf16(K_pages), to_dev_bf16(V_pages)
    Kc, Vc = to_dev_bf16(K), to_dev_bf16(V)
    td = torch.from_numpy(tbl).to(DEV)
    lst_d, n_d = torch.from_numpy(lst).to(DEV), torch.from_numpy(n_t).to(DEV)
    st = status_tensor()
    out_p, _ = ksa.ksa_sparse_decode_attn_paged(qd, Kp, Vp, td, Ld, lst_d, n_d, tokens_per_idx=1,
                                                idx_shared=True, dev_status=st)
    out_c, _ = ksa.ksa_sparse_decode_attn(qd, Kc, Vc, Ld, lst_d, n_d, tokens_per_idx=1,
                                          idx_shared=True)
    assert torch.equal(out_p, out_c)
    ref, _, _ = oracle.attention(q, K, V, lens, lst, n_t, 1, True)
    assert_out_close(out_p.cpu().numpy(), ref)
    assert st.item() == 0


def test_attention_edge_cases(ksa, oracle):
    rng = np.random.default_rng(600)
    B, Hq, Hkv, D, T, bs = 3, 4, 2, 128, 256, 16
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([256, 100, 256], np.int32)
    # row 0: empty lists; row 1: one single block; row 2: every block (== dense)
    idx = np.full((B, Hkv, 16), -1, np.int32)
    cnt = np.array([[0, 0], [1, 1], [16, 16]], np.int32)
    idx[1, :, 0] = [6, 0]
    idx[2] = np.arange(16)[None, :]
    assert _attn_check(ksa, oracle, q, K, V, lens, idx, cnt, bs) == 0
    # all blocks selected == dense
    dense_ref, _, _ = oracle.attention(q[2:], K[2:], V[2:], lens[2:])
    blk_ref, _, _ = oracle.attention(q[2:], K[2:], V[2:], lens[2:], idx[2:], cnt[2:], bs)
    np.testing.assert_allclose(blk_ref, dense_ref, rtol=0, atol=1e-12)


def test_attention_flags_bad_entries(ksa, oracle):
    rng = np.random.default_rng(610)
    B, Hq, Hkv, D, T, bs = 1, 4, 1, 128, 128, 16
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([100], np.int32)
    idx = np.array([[[1, -5, 3, 7, 2]]], np.int32)  # -5 invalid, block 7 starts past L=100
    cnt = np.array([[5]], np.int32)
    st = _attn_check(ksa, oracle, q, K, V, lens, idx, cnt, bs)
    assert st & 2  # KSA_FLAG_INDEX_SKIPPED


def test_device_status_read_back_and_clear(ksa, oracle):
    """ksa_get_device_status returns the bits a step's calls collected in one word, and
    clears it on request."""
    rng = np.random.default_rng(611)
    B, Hq, Hkv, D, T, bs = 1, 4, 1, 128, 128, 16
    q, K, V = (to_dev_bf16(rand_bits(rng, s)) for s in [(B, Hq, D), (B, Hkv, T, D),
                                                         (B, Hkv, T, D)])
    lens = torch.tensor([100], dtype=torch.int32, device=DEV)
    idx = torch.tensor([[[1, -5, 3]]], dtype=torch.int32, device=DEV)  # -5 names no block
    cnt = torch.tensor([[3]], dtype=torch.int32, device=DEV)
    st = status_tensor()
    ksa.ksa_sparse_decode_attn(q, K, V, lens, idx, cnt, tokens_per_idx=bs, dev_status=st)
    assert ksa.ksa_get_device_status(st) == ksa.FLAG_INDEX_SKIPPED
    assert ksa.ksa_get_device_status(st, clear=True) == ksa.FLAG_INDEX_SKIPPED
    assert ksa.ksa_get_device_status(st) == 0
    ksa.ksa_sparse_decode_attn(q, K, V, lens, idx[:, :, :1].contiguous(), cnt * 0 + 1,
                               tokens_per_idx=bs, dev_status=st)
    assert ksa.ksa_get_device_status(st) == 0  # a clean call adds nothing


def test_seq_len_out_of_range_is_clamped_and_flagged(ksa, oracle):
    rng = np.random.default_rng(620)
    B, Hq, Hkv, D, T = 2, 4, 2, 64, 96
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([500, 0], np.int32)
    qd, Kd, Vd = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V)
    st = status_tensor()
    out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, torch.from_numpy(lens).to(DEV),
                                        dev_status=st)
    assert st.item() & 1  # KSA_FLAG_SEQ_LEN_CLAMPED
    ref, _, _ = oracle.attention(q, K, V, np.array([T, 0], np.int32))
    assert_out_close(out.cpu().numpy(), ref)


# ---------------------------------------------------------------------------
# A6 unified selection


@pytest.mark.parametrize("L,P,budget,R", [(300, 50, 64, 16), (1500, 400, 300, 75),
                                           (2500, 2600, 500, 125), (900, 120, 900, 225),
                                           (4100, 1000, 1000, 1000), (5000, 800, 1200, 0),
                                           (11000, 2000, 3000, 750), (15500, 3000, 4000, 1000),
                                           (24500, 4000, 4000, 1000),
                                           (30000, 3000, 4000, 1000)])
def test_unified_select_exact(ksa, oracle, L, P, budget, R):
    rng = np.random.default_rng(700 + L)
    B, Hq, Hkv, D = 3, 16, 4, 128
    T = L + 37
    q = dyadic_bits(rng, (B, Hq, D))
    K = dyadic_bits(rng, (B, Hkv, T, D))
    lens = np.array([L, max(1, L // 3), max(1, budget - 5)], np.int32)
    idx, cnt = ksa.ksa_unified_select(to_dev_bf16(q), to_dev_bf16(K),
                                      torch.from_numpy(lens).to(DEV), P, budget, R)
    ref_idx, ref_cnt = oracle.unified_select(q, K, lens, P, budget, R)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)


@pytest.mark.parametrize("Hq,Hkv", [(20, 4), (48, 8), (63, 9), (64, 8)])
def test_unified_select_head_counts(ksa, oracle, Hq, Hkv):
    # the shared set adds the heads' pick bits sixteen at a time, the rest one at a
    # time; vote counts up to 63 stay exact; 64 heads and more count votes per token
    rng = np.random.default_rng(720 + Hq)
    B, D, L = 2, 64, 3000
    T = L + 5
    q = dyadic_bits(rng, (B, Hq, D))
    K = dyadic_bits(rng, (B, Hkv, T, D))
    lens = np.array([L, L - 777], np.int32)
    idx, cnt = ksa.ksa_unified_select(to_dev_bf16(q), to_dev_bf16(K),
                                      torch.from_numpy(lens).to(DEV), 600, 800, 200)
    ref_idx, ref_cnt = oracle.unified_select(q, K, lens, 600, 800, 200)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)


def test_unified_default_window_is_quarter(ksa, oracle):
    rng = np.random.default_rng(710)
    B, Hq, Hkv, D, T = 1, 8, 2, 64, 1200
    q = dyadic_bits(rng, (B, Hq, D))
    K = dyadic_bits(rng, (B, Hkv, T, D))
    lens = np.array([T], np.int32)
    idx, cnt = ksa.ksa_unified_select(to_dev_bf16(q), to_dev_bf16(K),
                                      torch.from_numpy(lens).to(DEV), 200, 400)
    ref_idx, _ = oracle.unified_select(q, K, lens, 200, 400, 100)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)


# ---------------------------------------------------------------------------
# whole decode step on the named workloads


def _decode_step(ksa, inp, k):
    sh = inp.shape
    S = ksa.ksa_build_block_summaries(inp.K, inp.seq_lens, sh.block_size)
    ksa.ksa_build_block_summaries(inp.K, inp.seq_lens, sh.block_size, ksa.SUMMARY_LAST_BLOCK,
                                  summaries=S)
    idx, cnt = ksa.ksa_select_blocks(inp.q, S, inp.seq_lens, sh.block_size, sh.capacity, k)
    lse = torch.empty((sh.batch, sh.num_q_heads), dtype=torch.float32, device=DEV)
    out, _ = ksa.ksa_sparse_decode_attn(inp.q, inp.K, inp.V, inp.seq_lens, idx, cnt,
                                        tokens_per_idx=sh.block_size, lse=lse)
    return idx, cnt, out, lse


def _check_rows(oracle, inp, rows, idx, cnt, out, lse, k):
    sh = inp.shape
    for b in rows:
        L = int(inp.seq_lens[b].item())
        qb, Kb, Vb = host_bits(inp.q[b:b + 1]), host_bits(inp.K[b:b + 1]), host_bits(inp.V[b:b + 1])
        lens = np.array([L], np.int32)
        ref_idx, ref_cnt = oracle.select_blocks(qb, Kb, lens, sh.block_size, k)
        assert np.array_equal(cnt[b].cpu().numpy(), ref_cnt[0]), b
        assert np.array_equal(idx[b].cpu().numpy(), ref_idx[0]), b
        ref, ref_lse, _ = oracle.attention(qb, Kb, Vb, lens, ref_idx, ref_cnt, sh.block_size)
        assert_out_close(out[b:b + 1].cpu().numpy(), ref, what=f"row {b}")
        np.testing.assert_allclose(lse[b:b + 1].cpu().numpy(), ref_lse, rtol=0, atol=LSE_TOL)


def _plant(oracle, inp, rows, k):
    sh = inp.shape
    for b in rows:
        L = int(inp.seq_lens[b].item())
        Kb, _ = gap_fix_row(oracle, host_bits(inp.q[b]), host_bits(inp.K[b]), L, sh.block_size, k)
        inp.K[b] = to_dev_bf16(Kb)


def test_decode_step_tiny(ksa, oracle):
    inp = synth.tiny_inputs(device=DEV)
    rows = [0]
    _plant(oracle, inp, rows, synth.TINY.k_blocks)
    res = _decode_step(ksa, inp, synth.TINY.k_blocks)
    _check_rows(oracle, inp, rows, *res, synth.TINY.k_blocks)


def test_decode_step_qwen3_0_6b_full_size(ksa, oracle):
    inp = synth.qwen3_0_6b_inputs(device=DEV)
    rows = sample_rows(inp.shape.batch, 5)
    _plant(oracle, inp, rows, inp.shape.k_blocks)
    res = _decode_step(ksa, inp, inp.shape.k_blocks)
    _check_rows(oracle, inp, rows, *res, inp.shape.k_blocks)


def test_decode_step_qwen3_8b_full_size(ksa, oracle):
    inp = synth.qwen3_8b_inputs(device=DEV, poison_tail=64.0)
    rows = sample_rows(inp.shape.batch, 6)
    _plant(oracle, inp, rows, inp.shape.k_blocks)
    res = _decode_step(ksa, inp, inp.shape.k_blocks)
    _check_rows(oracle, inp, rows, *res, inp.shape.k_blocks)


def _fused_step(ksa, inp, k, one_call=False, stale_last_block=True):
    """The decode step as bench.py times it: ksa_decode_step (one_call), or the fused
    selection call (last-block refresh + scoring + top-k) then the attention call.  The
    summaries are prefilled from the cache as it was before the newest token (seq_lens - 1;
    blocks never built hold NaN), so the step must refresh the block the newest token
    landed in before it scores."""
    sh = inp.shape
    B, Hq, Hkv, D, T, bs = (sh.batch, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, sh.capacity,
                            sh.block_size)
    S = torch.full((B, Hkv, -(-T // bs), D), float("nan"), dtype=torch.float32, device=DEV)
    before = (inp.seq_lens - 1).clamp_min(1) if stale_last_block else inp.seq_lens
    ksa.ksa_build_block_summaries(inp.K, before, bs, summaries=S)
    st = status_tensor()
    if one_call:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
        idx, cnt, out, _ = ksa.ksa_decode_step(inp.q, inp.K, inp.V, S, inp.seq_lens, bs, k,
                                               lse=lse, dev_status=st)
        assert st.item() == 0
        return idx, cnt, out, lse
    ws_sel = torch.zeros((ksa.ksa_select_blocks_workspace(B, Hq, Hkv, D, T, bs, k),),
                         dtype=torch.uint8, device=DEV)
    ws_att = torch.zeros((ksa.ksa_sparse_decode_attn_workspace(B, Hq, Hkv, D, T, k, bs),),
                         dtype=torch.uint8, device=DEV)
    idx, cnt = ksa.ksa_decode_select_blocks(inp.q, inp.K, S, inp.seq_lens, bs, k,
                                            workspace=ws_sel, dev_status=st)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    out, _ = ksa.ksa_sparse_decode_attn(inp.q, inp.K, inp.V, inp.seq_lens, idx, cnt,
                                        tokens_per_idx=bs, lse=lse, workspace=ws_att,
                                        dev_status=st)
    assert st.item() == 0
    return idx, cnt, out, lse


@pytest.mark.parametrize("one_call", [True, False], ids=["decode_step", "two_calls"])
@pytest.mark.parametrize("which", ["qwen3-0.6b", "qwen3-8b"])
def test_fused_decode_step_full_size(ksa, oracle, which, one_call):
    """The decode step at the full Qwen3-0.6B (batch 64, 512 blocks, k 32) and Qwen3-8B
    (batch 32, 1024-2048 blocks, k 128) shapes, through ksa_decode_step (what bench.py times)
    and through the two calls, planted score gap on the sampled rows: indices bit-exact,
    outputs within 2e-3 of the oracle."""
    if which == "qwen3-0.6b":
        inp = synth.qwen3_0_6b_inputs(device=DEV)
    else:
        inp = synth.qwen3_8b_inputs(device=DEV, poison_tail=64.0)
    rows = sample_rows(inp.shape.batch, 11, extra=3)
    _plant(oracle, inp, rows, inp.shape.k_blocks)
    res = _fused_step(ksa, inp, inp.shape.k_blocks, one_call)
    _check_rows(oracle, inp, rows, *res, inp.shape.k_blocks)


@pytest.mark.parametrize("context,budget", [(131072, 8192), (32768, 256), (4096, 8192)])
def test_sweep_points_fused_step(ksa, oracle, context, budget):
    """Sparse points of the throughput sweep (Hq 32, Hkv 8, D 128, bs 16) at their own
    context and budget, two rows each, through ksa_decode_step (one launch up to 2048
    blocks per row, the two calls' launches beyond):
    128K / 8192 tokens (k = 512 of 8192 blocks), 32K / 256 (k = 16), and 4K / 8192, where
    k = 512 covers all 256 blocks so the step must equal dense attention."""
    sh = synth.dataclasses.replace(synth.sweep_shape(context, budget), batch=2)
    inp = synth.sweep_inputs(sh, seed=1005 + context + budget, device=DEV)
    k = sh.k_blocks
    rows = [0, 1]
    _plant(oracle, inp, rows, k)
    idx, cnt, out, lse = _fused_step(ksa, inp, k, one_call=True)
    _check_rows(oracle, inp, rows, idx, cnt, out, lse, k)
    nb = -(-context // sh.block_size)
    if k >= nb:
        assert torch.all(cnt == nb)
        dense = torch.empty_like(out)
        dense_lse = torch.empty_like(lse)
        ksa.ksa_sparse_decode_attn(inp.q, inp.K, inp.V, inp.seq_lens, out=dense, lse=dense_lse)
        assert_out_close(out.cpu().numpy(), dense.cpu().numpy(), what="k covers every block")
        np.testing.assert_allclose(lse.cpu().numpy(), dense_lse.cpu().numpy(), rtol=0,
                                   atol=LSE_TOL)


def test_append_kv_writes_the_newest_slot(ksa, oracle):
    """ksa_append_kv: K[b, g, L_b - 1] and V[b, g, L_b - 1] take the new rows bit for bit and
    nothing else changes; a row whose seq_len is outside [1, T] is left alone and flagged.
    The paged form writes the same rows into the pages the block table names."""
    rng = np.random.default_rng(1600)
    B, Hkv, T, D, bs = 4, 3, 96, 128, 16
    K, V = rand_bits(rng, (B, Hkv, T, D)), rand_bits(rng, (B, Hkv, T, D))
    kn, vn = rand_bits(rng, (B, Hkv, D)), rand_bits(rng, (B, Hkv, D))
    lens = np.array([1, 50, 96, 97], np.int32)  # the last is out of range
    Kd, Vd = to_dev_bf16(K), to_dev_bf16(V)
    st = status_tensor()
    ksa.ksa_append_kv(to_dev_bf16(kn), to_dev_bf16(vn), Kd, Vd, torch.from_numpy(lens).to(DEV),
                      dev_status=st)
    wantK, wantV = K.copy(), V.copy()
    for b in range(3):
        wantK[b, :, lens[b] - 1] = kn[b]
        wantV[b, :, lens[b] - 1] = vn[b]
    assert np.array_equal(host_bits(Kd), wantK) and np.array_equal(host_bits(Vd), wantV)
    assert st.item() == ksa.FLAG_SEQ_LEN_CLAMPED
    # paged: a shuffled pool with a spare page; row 3's slot names a page outside the pool
    mb = T // bs
    P = B * mb + 1
    perm = rng.permutation(P)[:B * mb].astype(np.int32).reshape(B, mb)
    perm[3, (30 - 1) // bs] = P + 5
    plens = np.array([1, 50, 96, 30], np.int32)
    pages_k = rand_bits(rng, (P, Hkv, bs, D))
    pages_v = rand_bits(rng, (P, Hkv, bs, D))
    Kp, Vp = to_dev_bf16(pages_k), to_dev_bf16(pages_v)
    st.zero_()
    ksa.ksa_append_kv_paged(to_dev_bf16(kn), to_dev_bf16(vn), Kp, Vp,
                            torch.from_numpy(perm).to(DEV), torch.from_numpy(plens).to(DEV),
                            dev_status=st)
    wk, wv = pages_k.copy(), pages_v.copy()
    for b in range(3):
        t = plens[b] - 1
        wk[perm[b, t // bs], :, t % bs] = kn[b]
        wv[perm[b, t // bs], :, t % bs] = vn[b]
    assert np.array_equal(host_bits(Kp), wk) and np.array_equal(host_bits(Vp), wv)
    assert st.item() == ksa.FLAG_INDEX_SKIPPED


def test_lessismore_full_size(ksa, oracle):
    sh = synth.LESSISMORE
    inp = synth.lessismore_inputs(device=DEV)
    tok, cnt = ksa.ksa_unified_select(inp.q_sel, inp.K_sel, inp.seq_lens, sh.per_head_topk,
                                      sh.token_budget, sh.recent_tokens)
    rows = sample_rows(sh.batch, 7, extra=1)
    for b in rows:
        ref_idx, ref_cnt = oracle.unified_select(host_bits(inp.q_sel[b:b + 1]),
                                                 host_bits(inp.K_sel[b:b + 1]),
                                                 np.array([sh.seq_len], np.int32),
                                                 sh.per_head_topk, sh.token_budget,
                                                 sh.recent_tokens)
        assert cnt[b].item() == ref_cnt[0] == sh.token_budget
        assert np.array_equal(tok[b].cpu().numpy(), ref_idx[0]), b
    for (q, K, V) in inp.layers:
        out, _ = ksa.ksa_sparse_decode_attn(q, K, V, inp.seq_lens, tok, cnt, tokens_per_idx=1,
                                            idx_shared=True)
        for b in rows[:2]:
            ref, _, _ = oracle.attention(host_bits(q[b:b + 1]), host_bits(K[b:b + 1]),
                                         host_bits(V[b:b + 1]), np.array([sh.seq_len], np.int32),
                                         tok[b:b + 1].cpu().numpy(), cnt[b:b + 1].cpu().numpy(),
                                         1, True)
            assert_out_close(out[b:b + 1].cpu().numpy(), ref, what=f"row {b}")


def test_dense_full_context_sampled(ksa, oracle):
    """k = all: the dense path on a 32K-context sweep shape (few rows)."""
    sh = synth.dataclasses.replace(synth.sweep_shape(32768, 1024), batch=4)
    inp = synth.sweep_inputs(sh, device=DEV)
    out, _ = ksa.ksa_sparse_decode_attn(inp.q, inp.K, inp.V, inp.seq_lens)
    for b in (0, 3):
        ref, _, _ = oracle.attention(host_bits(inp.q[b:b + 1]), host_bits(inp.K[b:b + 1]),
                                     host_bits(inp.V[b:b + 1]), np.array([32768], np.int32))
        assert_out_close(out[b:b + 1].cpu().numpy(), ref, what=f"row {b}")


@pytest.mark.parametrize("mode", ["dense", "blocks", "tokens"])
def test_long_pipelines(ksa, oracle, mode):
    """Few rows, long selections: every CTA cycles its stage buffers dozens of
    times (the pipeline's barrier phases wrap many times)."""
    rng = np.random.default_rng(800)
    B, Hq, Hkv, D, T, bs = 1, 8, 2, 128, 32768, 16
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([T - 5], np.int32)
    if mode == "dense":
        assert _attn_check(ksa, oracle, q, K, V, lens) == 0
    elif mode == "blocks":
        nb = -(-lens[0] // bs)
        idx = np.stack([np.sort(rng.choice(nb, size=1024, replace=False)) for _ in range(Hkv)])
        idx[:, -1] = nb - 1  # keep the partial tail block
        idx = np.sort(idx, axis=1)[None].astype(np.int32)
        cnt = np.full((B, Hkv), 1024, np.int32)
        assert _attn_check(ksa, oracle, q, K, V, lens, idx, cnt, bs) == 0
    else:
        idx = np.sort(rng.choice(lens[0], size=8192, replace=False))[None].astype(np.int32)
        cnt = np.array([8192], np.int32)
        assert _attn_check(ksa, oracle, q, K, V, lens, idx, cnt, 1, shared=True) == 0


@pytest.mark.parametrize("mode", ["dense", "blocks", "tokens"])
def test_long_rows_repeat_calls(ksa, oracle, mode):
    """Rows of 1536-2048 stages, each split between many CTAs, over 24K+ stages in all.  Every
    output matches the oracle; three calls on one workspace give the same bits (the split and
    the merge order are fixed); the row semaphores are zero again after every call."""
    rng = np.random.default_rng(810)
    B, Hq, Hkv, D, T, bs = 4, 8, 4, 128, 32768, 16
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([T, T - 5, 25000, 30001], np.int32)
    idx = cnt = None
    tpi, shared = 1, False
    if mode == "blocks":  # 1536 of each row's blocks: 1536 stages a row
        tpi = bs
        idx = np.zeros((B, Hkv, 1536), np.int32)
        for b in range(B):
            nb = -(-int(lens[b]) // bs)
            for g in range(Hkv):
                idx[b, g] = np.sort(rng.choice(nb, size=1536, replace=False))
        cnt = np.full((B, Hkv), 1536, np.int32)
    elif mode == "tokens":  # one shared set of 24576 tokens a row: 1536 stages a row
        shared = True
        idx = np.stack([np.sort(rng.choice(int(lens[b]), size=24576, replace=False))
                        for b in range(B)]).astype(np.int32)
        cnt = np.full((B,), 24576, np.int32)
    qd, Kd, Vd = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V)
    Ld = torch.from_numpy(lens).to(DEV)
    idx_d = None if idx is None else torch.from_numpy(idx).to(DEV)
    cnt_d = None if cnt is None else torch.from_numpy(cnt).to(DEV)
    cap = T if mode == "dense" else idx.shape[-1]
    ws = torch.zeros((ksa.lib().ksa_sparse_decode_attn_workspace(
        ctypes.byref(ksa.Shape(B, Hq, Hkv, D, T, bs)), cap, tpi),), dtype=torch.uint8, device=DEV)
    head = (B * Hq * 4 + 255) // 256 * 256  # the semaphores
    outs = []
    for _ in range(3):
        st = status_tensor()
        out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, Ld, idx_d, cnt_d, tokens_per_idx=tpi,
                                            idx_shared=shared, workspace=ws, dev_status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert int(ws[:head].count_nonzero()) == 0
        outs.append(out.cpu().numpy())
    assert all(np.array_equal(outs[0].view(np.uint32), o.view(np.uint32)) for o in outs[1:])
    ref, _, _ = oracle.attention(q, K, V, lens, idx, cnt, tpi, shared)
    assert_out_close(outs[0], ref)


@pytest.mark.parametrize("D,bs,k,nblk", [(128, 16, 8, 40), (64, 32, 6, 40), (64, 16, 12, 1100)])
def test_decode_select_fuses_last_block_refresh(ksa, oracle, D, bs, k, nblk):
    """ksa_decode_select_blocks == LAST_BLOCK refresh followed by selection:
    the same summaries bit for bit, the same blocks, and the oracle's blocks
    (1100 blocks: rows too long to rank inside the scoring launch)."""
    rng = np.random.default_rng(900 + D + nblk)
    B, Hq, Hkv = 4, 8, 2
    T = nblk * bs + 9
    lens = np.array([T, 3 * bs + 1, 5, 20 * bs], np.int32)  # rows 1 and 2 keep every block
    q = rand_bits(rng, (B, Hq, D))
    K_new = rand_bits(rng, (B, Hkv, T, D))
    for b in range(B):
        K_new[b], _ = gap_fix_row(oracle, q[b], K_new[b], int(lens[b]), bs, k)
    K_old = K_new.copy()  # the cache before this step's token: the last block differs
    for b in range(B):
        jl = (lens[b] - 1) // bs
        K_old[b, :, jl * bs:lens[b]] = rand_bits(rng, (Hkv, lens[b] - jl * bs, D))
    qd, Ld = to_dev_bf16(q), torch.from_numpy(lens).to(DEV)
    S0 = ksa.ksa_build_block_summaries(to_dev_bf16(K_old), Ld, bs)
    Kn = to_dev_bf16(K_new)
    S_a = S0.clone()
    ksa.ksa_build_block_summaries(Kn, Ld, bs, ksa.SUMMARY_LAST_BLOCK, summaries=S_a)
    idx_a, cnt_a = ksa.ksa_select_blocks(qd, S_a, Ld, bs, T, k)
    S_b = S0.clone()
    st = status_tensor()
    idx_b, cnt_b = ksa.ksa_decode_select_blocks(qd, Kn, S_b, Ld, bs, k, dev_status=st)
    assert torch.equal(S_a.view(torch.int32), S_b.view(torch.int32))  # bits (see above)
    assert torch.equal(idx_a, idx_b) and torch.equal(cnt_a, cnt_b)
    ref_idx, ref_cnt = oracle.select_blocks(q, K_new, lens, bs, k)
    assert np.array_equal(idx_b.cpu().numpy(), ref_idx)
    assert np.array_equal(cnt_b.cpu().numpy(), ref_cnt)
    assert st.item() == 0


def test_select_many_rows_persistent_units(ksa, oracle):
    """Ragged rows split between scoring warps: each row is ranked by the warp
    that completes it, and the per-row counters come back to zero."""
    rng = np.random.default_rng(950)
    B, Hq, Hkv, D, bs, k = 48, 16, 8, 128, 16, 16
    T = 200 * bs
    lens = rng.integers(10, T + 1, size=B).astype(np.int32)
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    for b in range(B):
        K[b], _ = gap_fix_row(oracle, q[b], K[b], int(lens[b]), bs, k)
    qd, Kd, Ld = to_dev_bf16(q), to_dev_bf16(K), torch.from_numpy(lens).to(DEV)
    S = ksa.ksa_build_block_summaries(Kd, Ld, bs)
    ws = torch.zeros((ksa.ksa_select_blocks_workspace(B, Hq, Hkv, D, T, bs, k),),
                     dtype=torch.uint8, device=DEV)
    ref_idx, ref_cnt = oracle.select_blocks(q, K, lens, bs, k)
    for _ in range(2):  # the workspace semaphores must come back to zero
        idx, cnt = ksa.ksa_select_blocks(qd, S, Ld, bs, T, k, workspace=ws)
        assert np.array_equal(idx.cpu().numpy(), ref_idx)
        assert np.array_equal(cnt.cpu().numpy(), ref_cnt)


# ---------------------------------------------------------------------------
# bf16-stored block summaries

DELTA_BF16 = 0.05  # one bf16 unit in one stored mean moves a score by at most ~0.02 here


@pytest.mark.parametrize("D,bs", [(128, 16), (64, 32)])
def test_summaries_bf16_storage(ksa, oracle, D, bs):
    """bf16 storage = the fp32 mean rounded to nearest even, bit for bit; and within one
    bf16 unit of the oracle's rounding of the exact mean.  LAST_BLOCK writes one block."""
    rng = np.random.default_rng(1100 + D)
    B, Hkv, T = 3, 2, 9 * bs + 3
    K = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([T, 1, 2 * bs + 5], np.int32)
    Kd, Ld = to_dev_bf16(K), torch.from_numpy(lens).to(DEV)
    S32 = ksa.ksa_build_block_summaries(Kd, Ld, bs)
    S16 = ksa.ksa_build_block_summaries(Kd, Ld, bs, summary_dtype=torch.bfloat16)
    assert S16.dtype == torch.bfloat16
    ref = oracle.block_summaries_bf16(K, lens, bs).astype(np.int32)
    got = S16.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.int32)
    want = S32.to(torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16).astype(np.int32)
    for b in range(B):
        nb = -(-lens[b] // bs)
        assert np.array_equal(got[b, :, :nb], want[b, :, :nb])
        assert np.abs(got[b, :, :nb] - ref[b, :, :nb]).max() <= 1
    S2 = torch.full_like(S16, float("nan"))
    ksa.ksa_build_block_summaries(Kd, Ld, bs, ksa.SUMMARY_LAST_BLOCK, summaries=S2)
    S2 = S2.float().cpu().numpy()
    for b in range(B):
        nb = -(-lens[b] // bs)
        np.testing.assert_array_equal(S2[b, :, nb - 1], S16[b, :, nb - 1].float().cpu().numpy())
        assert np.all(np.isnan(S2[b, :, :nb - 1])) and np.all(np.isnan(S2[b, :, nb:]))


@pytest.mark.parametrize("D,bs,k,nblk", [(128, 16, 8, 40), (64, 32, 6, 300), (128, 16, 32, 1100)])
def test_select_blocks_bf16_summaries(ksa, oracle, D, bs, k, nblk):
    """Selection from bf16-stored summaries: the oracle's blocks for bf16-stored means,
    with a planted gap; the fused decode-step form refreshes the last block in bf16."""
    rng = np.random.default_rng(1200 + nblk)
    B, Hq, Hkv = 3, 8, 2
    T = nblk * bs + 7
    lens = np.array([T, 13 * bs + 1, 3 * bs], np.int32)
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    for b in range(B):
        K[b], _ = gap_fix_row(oracle, q[b], K[b], int(lens[b]), bs, k, delta=DELTA_BF16,
                              summary_bf16=True)
        assert min_boundary_gap(oracle, q[b], K[b], int(lens[b]), bs, k,
                                summary_bf16=True) >= DELTA_BF16
    qd, Kd, Ld = to_dev_bf16(q), to_dev_bf16(K), torch.from_numpy(lens).to(DEV)
    st = status_tensor()
    S = ksa.ksa_build_block_summaries(Kd, Ld, bs, summary_dtype=torch.bfloat16, dev_status=st)
    idx, cnt = ksa.ksa_select_blocks(qd, S, Ld, bs, T, k, dev_status=st)
    ref_idx, ref_cnt = oracle.select_blocks(q, K, lens, bs, k, summary_bf16=True)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    # fused form: stale last blocks in the summaries, refreshed (in bf16) by the call
    S_old = S.clone()
    for b in range(B):
        jl = (lens[b] - 1) // bs
        S_old[b, :, jl] = 0
    idx2, cnt2 = ksa.ksa_decode_select_blocks(qd, Kd, S_old, Ld, bs, k, dev_status=st)
    # bit patterns: blocks past a row's end hold unwritten memory, possibly NaN patterns
    assert torch.equal(S_old.view(torch.int16), S.view(torch.int16))
    assert torch.equal(idx2, idx) and torch.equal(cnt2, cnt)
    assert st.item() == 0


# one e4m3 step of one stored element (1/8 of its binade, at the block's scale) moves a score
# by |group query sum| x step: here at most ~0.12; the planted gap is twice that
DELTA_FP8 = 0.25


def _fp8_values(S8):
    """Decoded fp8 summaries [B, Hkv, nb, D] (fp64, host): the e4m3 values times the scales."""
    vals = S8.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return vals * ksa_scales(S8)[..., None]


def ksa_scales(S8):
    import block_top_sparse_ksa_b200 as k
    return k.fp8_summary_scales(S8).cpu().to(torch.float64).numpy()


def test_summaries_fp8_storage(ksa, oracle):
    """fp8 storage (D = 128): a block's scale is 2^e, e the smallest exponent with
    max|mean| <= 448 2^e, and its values are the fp32 means times 2^-e rounded to the nearest
    e4m3 value -- bit for bit what torch's float8_e4m3fn cast makes of the GPU's own fp32
    means -- and against the oracle's rounding of the exact means the scales agree and a
    value differs by at most one e4m3 step.  LAST_BLOCK writes one block and its scale."""
    rng = np.random.default_rng(1150)
    B, Hkv, D, bs = 3, 2, 128, 16
    T = 9 * bs + 3
    nbm = -(-T // bs)
    # keys of very different sizes from block to block (scales 2^-8 .. 2^7)
    mag = np.exp2(rng.integers(-8, 8, (B, Hkv, nbm, 1, 1))).repeat(bs, 3).reshape(B, Hkv, -1, 1)
    K = bf16_bits(rng.standard_normal((B, Hkv, nbm * bs, D)) * mag)[:, :, :T]
    K = np.ascontiguousarray(K)
    lens = np.array([T, 1, 2 * bs + 5], np.int32)
    Kd, Ld = to_dev_bf16(K), torch.from_numpy(lens).to(DEV)
    S32 = ksa.ksa_build_block_summaries(Kd, Ld, bs)
    S8 = ksa.ksa_build_block_summaries(Kd, Ld, bs, summary_dtype="fp8")
    assert S8.dtype == torch.uint8 and tuple(S8.shape) == (B, Hkv, nbm, D)
    scales = ksa_scales(S8)
    want_bytes = (S32.cpu().double() / torch.from_numpy(scales)[..., None]).float().to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    got_bytes = S8.cpu().numpy()
    ref = oracle.store_fp8(oracle.block_summaries(K, lens, bs))
    got = _fp8_values(S8)
    for b in range(B):
        nb = -(-lens[b] // bs)
        m32 = np.abs(S32[b, :, :nb].cpu().double().numpy()).max(-1)
        e = np.vectorize(oracle.e4m3_scale_exp)(m32)
        np.testing.assert_array_equal(scales[b, :, :nb], np.exp2(e))
        assert np.array_equal(got_bytes[b, :, :nb], want_bytes[b, :, :nb])
        d = np.abs(got[b, :, :nb] - ref[b, :, :nb]) / scales[b, :, :nb, None]
        big = np.maximum(np.abs(got[b, :, :nb]), np.abs(ref[b, :, :nb])) / scales[b, :, :nb, None]
        step = np.exp2(np.floor(np.log2(np.maximum(big, 2.0 ** -6))) - 3)
        assert np.all(d <= step), d.max()
        assert np.mean(d > 0) < 1e-3
    S2 = ksa.alloc_summaries(B, Hkv, nbm, D, "fp8")
    S2.fill_(0x7F)  # e4m3 NaN everywhere
    ksa.fp8_summary_scales(S2).fill_(float("nan"))
    ksa.ksa_build_block_summaries(Kd, Ld, bs, ksa.SUMMARY_LAST_BLOCK, summaries=S2)
    sc2 = ksa_scales(S2)
    for b in range(B):
        nb = -(-lens[b] // bs)
        assert np.array_equal(S2[b, :, nb - 1].cpu().numpy(), got_bytes[b, :, nb - 1])
        np.testing.assert_array_equal(sc2[b, :, nb - 1], scales[b, :, nb - 1])
        assert np.all(S2[b, :, :nb - 1].cpu().numpy() == 0x7F)
        assert np.all(np.isnan(sc2[b, :, :nb - 1]))


@pytest.mark.parametrize("bs,k,nblk", [(16, 8, 40), (32, 6, 300), (16, 32, 1100)])
def test_select_blocks_fp8_summaries(ksa, oracle, bs, k, nblk):
    """Selection from fp8-stored summaries: the oracle's blocks for fp8-stored means, with a
    planted gap; the fused decode-step form refreshes the last block (values and scale)."""
    rng = np.random.default_rng(1250 + nblk)
    B, Hq, Hkv, D = 3, 8, 2, 128
    T = nblk * bs + 7
    lens = np.array([T, 13 * bs + 1, 3 * bs], np.int32)
    q = rand_bits(rng, (B, Hq, D))
    K = rand_bits(rng, (B, Hkv, T, D))
    for b in range(B):
        K[b], _ = gap_fix_row(oracle, q[b], K[b], int(lens[b]), bs, k, delta=DELTA_FP8,
                              summary_fp8=True)
        assert min_boundary_gap(oracle, q[b], K[b], int(lens[b]), bs, k,
                                summary_fp8=True) >= DELTA_FP8
    qd, Kd, Ld = to_dev_bf16(q), to_dev_bf16(K), torch.from_numpy(lens).to(DEV)
    st = status_tensor()
    S = ksa.ksa_build_block_summaries(Kd, Ld, bs, summary_dtype="fp8", dev_status=st)
    idx, cnt = ksa.ksa_select_blocks(qd, S, Ld, bs, T, k, dev_status=st)
    ref_idx, ref_cnt = oracle.select_blocks(q, K, lens, bs, k, summary_fp8=True)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    # fused form: stale last blocks (values and scales), refreshed in fp8 by the call
    S_old = ksa.alloc_summaries(B, Hkv, S.shape[2], D, "fp8")
    S_old.copy_(S)
    sc_old = ksa.fp8_summary_scales(S_old)
    sc_old.copy_(ksa.fp8_summary_scales(S))
    for b in range(B):
        jl = (lens[b] - 1) // bs
        S_old[b, :, jl] = 0
        sc_old[b, :, jl] = 0.0
    idx2, cnt2 = ksa.ksa_decode_select_blocks(qd, Kd, S_old, Ld, bs, k, dev_status=st)
    assert torch.equal(S_old, S)
    assert torch.equal(sc_old.view(torch.int32), ksa.fp8_summary_scales(S).view(torch.int32))
    assert torch.equal(idx2, idx) and torch.equal(cnt2, cnt)
    assert st.item() == 0


# ---------------------------------------------------------------------------
# paged K/V cache (page = block)


def _paged_case(rng, B, Hkv, D, bs, mb, extra_pages):
    """A page pool larger than needed, blocks placed on random distinct pages."""
    P = B * mb + extra_pages
    K_pages = rand_bits(rng, (P, Hkv, bs, D))
    V_pages = rand_bits(rng, (P, Hkv, bs, D))
    tbl = rng.permutation(P)[:B * mb].astype(np.int32).reshape(B, mb)
    return K_pages, V_pages, tbl


def _scatter(K, tbl, pages, bs):
    for b in range(K.shape[0]):
        for j in range(tbl.shape[1]):
            pages[tbl[b, j]] = K[b, :, j * bs:(j + 1) * bs]


@pytest.mark.parametrize("D,bs,k", [(128, 16, 8), (64, 32, 5)])
def test_paged_kv_matches_gathered_cache(ksa, oracle, D, bs, k):
    """Every paged entry point equals its contiguous form on the gathered cache, bit for bit,
    and the oracle on it: summaries, the fused decode selection, and attention over block
    lists, token lists and the dense set."""
    rng = np.random.default_rng(1300 + D)
    B, Hq, Hkv, mb = 3, 8, 2, 40
    T = mb * bs
    lens = np.array([T, 13 * bs + 1, 5], np.int32)
    K_pages, V_pages, tbl = _paged_case(rng, B, Hkv, D, bs, mb, extra_pages=17)
    q = rand_bits(rng, (B, Hq, D))
    K = oracle.gather_pages(K_pages, tbl, lens)
    for b in range(B):  # plant the score gap on the logical cache, then write it back
        K[b], _ = gap_fix_row(oracle, q[b], K[b], int(lens[b]), bs, k)
    _scatter(K, tbl, K_pages, bs)
    K = oracle.gather_pages(K_pages, tbl, lens)
    V = oracle.gather_pages(V_pages, tbl, lens)
    qd, Ld = to_dev_bf16(q), torch.from_numpy(lens).to(DEV)
    Kp, Vp = to_dev_bf16(K_pages), to_dev_bf16(V_pages)
    Kc, Vc = to_dev_bf16(K), to_dev_bf16(V)
    td = torch.from_numpy(tbl).to(DEV)
    st = status_tensor()
    S_p = ksa.ksa_build_block_summaries_paged(Kp, td, Ld, dev_status=st)
    S_c = ksa.ksa_build_block_summaries(Kc, Ld, bs)
    for b in range(B):
        nb = -(-lens[b] // bs)
        assert torch.equal(S_p[b, :, :nb], S_c[b, :, :nb])
    # fused decode selection from stale last blocks
    S_old = S_p.clone()
    for b in range(B):
        S_old[b, :, (lens[b] - 1) // bs] = 0.0
    idx, cnt = ksa.ksa_decode_select_blocks_paged(qd, Kp, td, S_old, Ld, k, dev_status=st)
    for b in range(B):
        nb = -(-lens[b] // bs)
        assert torch.equal(S_old[b, :, :nb], S_p[b, :, :nb])
    ref_idx, ref_cnt = oracle.select_blocks(q, K, lens, bs, k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    # attention: block list
    out_p, _ = ksa.ksa_sparse_decode_attn_paged(qd, Kp, Vp, td, Ld, idx, cnt, tokens_per_idx=bs,
                                                dev_status=st)
    out_c, _ = ksa.ksa_sparse_decode_attn(qd, Kc, Vc, Ld, idx, cnt, tokens_per_idx=bs)
    assert torch.equal(out_p, out_c)
    ref, _, _ = oracle.attention(q, K, V, lens, ref_idx, ref_cnt, bs)
    assert_out_close(out_p.cpu().numpy(), ref)
    # token list shared by the kv-heads, and the dense set
    lst = np.full((B, 64), -1, np.int32)
    n_t = np.zeros((B,), np.int32)
    for b in range(B):
        pick = np.sort(rng.choice(int(lens[b]), size=min(64, int(lens[b])), replace=False))
        lst[b, :len(pick)] = pick
        n_t[b] = len(pick)
    lst_d, n_d = torch.from_numpy(lst).to(DEV), torch.from_numpy(n_t).to(DEV)
    out_p, _ = ksa.ksa_sparse_decode_attn_paged(qd, Kp, Vp, td, Ld, lst_d, n_d, tokens_per_idx=1,
                                                idx_shared=True, dev_status=st)
    out_c, _ = ksa.ksa_sparse_decode_attn(qd, Kc, Vc, Ld, lst_d, n_d, tokens_per_idx=1,
                                          idx_shared=True)
    assert torch.equal(out_p, out_c)
    out_p, _ = ksa.ksa_sparse_decode_attn_paged(qd, Kp, Vp, td, Ld, dev_status=st)
    out_c, _ = ksa.ksa_sparse_decode_attn(qd, Kc, Vc, Ld)
    assert torch.equal(out_p, out_c)
    ref, _, _ = oracle.attention(q, K, V, lens)
    assert_out_close(out_p.cpu().numpy(), ref)
    assert st.item() == 0


def test_paged_kv_bad_page_ids_are_flagged_not_read(ksa, oracle):
    """A block whose page id is outside the pool is never read: its summary is zero, its
    tokens are left out of attention, and the status word says so."""
    rng = np.random.default_rng(1400)
    B, Hq, Hkv, D, bs, mb, k = 2, 4, 2, 128, 16, 12, 4
    lens = np.array([mb * bs, 7 * bs], np.int32)
    K_pages, V_pages, tbl = _paged_case(rng, B, Hkv, D, bs, mb, extra_pages=3)
    P = K_pages.shape[0]
    bad = tbl.copy()
    bad[0, 3] = P          # one past the pool
    bad[1, 6] = -5         # negative: the last block of row 1
    qd, Ld = to_dev_bf16(rand_bits(rng, (B, Hq, D))), torch.from_numpy(lens).to(DEV)
    Kp, Vp, td = to_dev_bf16(K_pages), to_dev_bf16(V_pages), torch.from_numpy(bad).to(DEV)
    st = status_tensor()
    S = ksa.ksa_build_block_summaries_paged(Kp, td, Ld, dev_status=st)
    assert st.item() & ksa.FLAG_INDEX_SKIPPED
    assert not S[0, :, 3].any() and not S[1, :, 6].any()
    st.zero_()
    idx, cnt = ksa.ksa_decode_select_blocks_paged(qd, Kp, td, S, Ld, k, dev_status=st)
    assert st.item() & ksa.FLAG_INDEX_SKIPPED  # the refresh of row 1's last block
    st.zero_()
    all_idx = torch.arange(mb, dtype=torch.int32, device=DEV).repeat(B, Hkv, 1)
    all_cnt = torch.tensor([[mb] * Hkv, [7] * Hkv], dtype=torch.int32, device=DEV)
    out, lse = ksa.ksa_sparse_decode_attn_paged(qd, Kp, Vp, td, Ld, all_idx, all_cnt,
                                                tokens_per_idx=bs,
                                                lse=torch.empty((B, Hq), device=DEV),
                                                dev_status=st)
    assert st.item() & ksa.FLAG_INDEX_SKIPPED
    assert torch.isfinite(out).all()
    # the same attention over a table whose bad blocks are simply not selected
    keep = [j for j in range(mb) if j != 3]
    sel = torch.tensor(keep + [-1], dtype=torch.int32, device=DEV).repeat(1, Hkv, 1)
    cnt0 = torch.tensor([[len(keep)] * Hkv], dtype=torch.int32, device=DEV)
    out0, _ = ksa.ksa_sparse_decode_attn_paged(qd[:1], Kp, Vp, td[:1], Ld[:1], sel, cnt0,
                                               tokens_per_idx=bs)
    # (another batch splits the work differently, so fp32 sums differ in the last bits)
    torch.testing.assert_close(out[:1], out0, atol=1e-5, rtol=1e-5)


# ---------------------------------------------------------------------------
# attention-recall diagnostic


def test_aggregation_comparison_bounds(ksa, oracle):
    """Unified, per-head and random-head sets of the same budget, scored by recall in the
    selection layer: each head's own top-k carries the most softmax mass any k tokens can,
    so the per-head recall bounds the other two head by head, and equals the random-head
    recall for the drawn head.  With one kv-head and identical query heads all three sets
    coincide."""
    from block_top_sparse_ksa_b200 import recall
    shape = synth.dataclasses.replace(synth.LESSISMORE, batch=2, num_q_heads=8, num_kv_heads=2,
                                      capacity=600, seq_len=600, per_head_topk=120,
                                      token_budget=120, recent_tokens=30)
    inp = synth.lessismore_inputs(seed=5, device=DEV, shape=shape)
    k, B = 120, 2
    heads = np.array([6, 1], np.int32)
    uni, ucnt = ksa.ksa_unified_select(inp.q_sel, inp.K_sel, inp.seq_lens, k, k, 0)
    ph, phc = ksa.ksa_select_tokens_per_head(inp.q_sel, inp.K_sel, inp.seq_lens, k)
    rh, rhc = ksa.ksa_select_tokens_one_head(inp.q_sel, inp.K_sel, inp.seq_lens, heads, k)
    args = (inp.q_sel, inp.K_sel, inp.K_sel, inp.seq_lens)
    r_uni = recall.attention_recall(*args, uni, ucnt, idx_shared=ksa.IDX_SHARED)
    r_ph = recall.attention_recall(*args, ph, phc, idx_shared=ksa.IDX_PER_Q_HEAD)
    r_rh = recall.attention_recall(*args, rh, rhc, idx_shared=ksa.IDX_SHARED)
    tol = 1e-4
    assert np.all(r_ph >= r_uni - tol) and np.all(r_ph >= r_rh - tol)
    for b in range(B):
        assert abs(r_rh[b, heads[b]] - r_ph[b, heads[b]]) <= tol
    res = recall.aggregation_comparison(inp, k, seed=3)
    assert res["per_head"]["selection_layer"] >= res["unified"]["selection_layer"] - tol
    assert res["per_head"]["selection_layer"] >= res["random_head"]["selection_layer"] - tol
    one = synth.dataclasses.replace(shape, num_kv_heads=1)
    inp1 = synth.lessismore_inputs(seed=6, device=DEV, shape=one)
    inp1.q_sel.copy_(inp1.q_sel[:, :1].clone().expand_as(inp1.q_sel))
    res1 = recall.aggregation_comparison(inp1, k, seed=3)
    vals = [res1[n]["selection_layer"] for n in ("unified", "per_head", "random_head")]
    assert max(vals) - min(vals) <= tol, vals


# recall = exp(lse_sel - lse_all) from two attention launches; each lse is within 1e-4 of the
# oracle's, so the recall is within (e^{2e-4} - 1) * recall <= 2.1e-4 of the oracle's recall
RECALL_TOL = 2.5e-4


@pytest.mark.parametrize("layout", ["blocks", "shared_tokens", "per_q_head"])
def test_attention_recall_matches_oracle(ksa, oracle, layout):
    """The GPU recall of a selection against the oracle's: the share of each head's dense
    softmax weight on the selected tokens, element by element; the dense set recalls 1 and
    an empty selection 0."""
    from block_top_sparse_ksa_b200.recall import attention_recall
    rng = np.random.default_rng(1500)
    B, Hq, Hkv, D, T, bs = 2, 8, 2, 64, 320, 16
    lens = np.array([T, 123], np.int32)
    q, K, V = (rand_bits(rng, s) for s in [(B, Hq, D), (B, Hkv, T, D), (B, Hkv, T, D)])
    nb = -(-lens // bs)
    if layout == "blocks":
        tpi, shared, k = bs, ksa.IDX_PER_KV_HEAD, 6
        idx = np.stack([np.stack([np.sort(rng.choice(int(nb[b]), size=k, replace=False))
                                  for _ in range(Hkv)]) for b in range(B)]).astype(np.int32)
        cnt = np.full((B, Hkv), k, np.int32)
    elif layout == "shared_tokens":
        tpi, shared, k = 1, ksa.IDX_SHARED, 40
        idx = np.stack([np.sort(rng.choice(int(lens[b]), size=k, replace=False))
                        for b in range(B)]).astype(np.int32)
        cnt = np.array([k, k - 7], np.int32)
    else:
        tpi, shared, k = 1, ksa.IDX_PER_Q_HEAD, 25
        idx = np.stack([np.stack([np.sort(rng.choice(int(lens[b]), size=k, replace=False))
                                  for _ in range(Hq)]) for b in range(B)]).astype(np.int32)
        cnt = np.full((B, Hq), k, np.int32)
    qd, Kd, Vd, Ld = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V), torch.from_numpy(lens).to(DEV)
    rec = attention_recall(qd, Kd, Vd, Ld, torch.from_numpy(idx).to(DEV),
                           torch.from_numpy(cnt).to(DEV), tokens_per_idx=tpi, idx_shared=shared)
    ref = oracle.attention_recall(q, K, lens, idx, cnt, tpi, shared)
    assert np.all(ref > 0.0) and np.all(ref < 1.0)
    np.testing.assert_allclose(rec, ref, rtol=0, atol=RECALL_TOL)
    all_idx = torch.arange(int(nb.max()), dtype=torch.int32, device=DEV).repeat(B, Hkv, 1)
    all_cnt = torch.from_numpy(np.repeat(nb[:, None], Hkv, 1).astype(np.int32)).to(DEV)
    assert np.allclose(attention_recall(qd, Kd, Vd, Ld, all_idx, all_cnt, tokens_per_idx=bs),
                       1.0, atol=RECALL_TOL)
    none = torch.zeros((B, Hkv), dtype=torch.int32, device=DEV)
    assert np.all(attention_recall(qd, Kd, Vd, Ld, all_idx, none, tokens_per_idx=bs) == 0.0)


def test_recency_sweep_matches_oracle(ksa, oracle):
    """The LessIsMore recency-share sweep (0 to 100% of the budget given to the recent
    window) on a small seeded shape: for every share the GPU's unified set equals the
    oracle's, and the mean recall of that set in the selection layer and in each sparse
    layer equals the oracle's recall of the oracle's set."""
    from block_top_sparse_ksa_b200 import recall
    shape = synth.dataclasses.replace(synth.LESSISMORE, batch=2, num_q_heads=8, num_kv_heads=2,
                                      capacity=1500, seq_len=1500, per_head_topk=300,
                                      token_budget=300, recent_tokens=75)
    inp = synth.lessismore_inputs(seed=21, device=DEV, shape=shape)
    ratios = [0.0, 0.25, 0.5, 0.75, 1.0]
    rows = recall.recency_sweep(inp, ratios)
    q_sel, K_sel = host_bits(inp.q_sel), host_bits(inp.K_sel)
    lens = inp.seq_lens.cpu().numpy()
    layers = [tuple(host_bits(t) for t in layer) for layer in inp.layers]
    for ratio, row in zip(ratios, rows):
        R = int(round(ratio * shape.token_budget))
        assert row["recent_tokens"] == R
        tok, cnt = oracle.unified_select(q_sel, K_sel, lens, shape.per_head_topk,
                                         shape.token_budget, R)
        g_tok, g_cnt = ksa.ksa_unified_select(inp.q_sel, inp.K_sel, inp.seq_lens,
                                              shape.per_head_topk, shape.token_budget, R)
        assert np.array_equal(g_tok.cpu().numpy(), tok) and np.array_equal(g_cnt.cpu().numpy(),
                                                                           cnt)
        want = oracle.attention_recall(q_sel, K_sel, lens, tok, cnt, 1, 1).mean()
        assert abs(row["selection_layer"] - want) <= RECALL_TOL, (ratio, row, want)
        for got, (q, K, _) in zip(row["sparse_layers"], layers):
            want = oracle.attention_recall(q, K, lens, tok, cnt, 1, 1).mean()
            assert abs(got - want) <= RECALL_TOL, (ratio, got, want)


def test_select_window_matches_oracle(ksa, oracle):
    """Local attention as a block selection: the oracle's last min(k, NB_b) blocks."""
    lens = np.array([1000, 1, 33, 16 * 7], np.int32)
    Ld = torch.from_numpy(lens).to(DEV)
    for bs in (16, 64):
        for k in (1, 5, 100):
            idx, cnt = ksa.ksa_select_window(Ld, 3, bs, 1000, k)
            ref_idx, ref_cnt = oracle.select_window(lens, 3, bs, k)
            assert np.array_equal(idx.cpu().numpy(), ref_idx)
            assert np.array_equal(cnt.cpu().numpy(), ref_cnt)


# ---------------------------------------------------------------------------
# per-head token top-k and attention with one list per query head


@pytest.mark.parametrize("L,k", [(300, 40), (1500, 400), (90, 200)])
def test_tokens_per_head_and_per_query_head_attention(ksa, oracle, L, k):
    """Dyadic q, K: exact scores, exact ties.  Every head's list equals the oracle's; the
    attention over per-query-head lists equals the oracle run head by head."""
    rng = np.random.default_rng(1600 + L)
    B, Hq, Hkv, D = 2, 8, 2, 128
    G = Hq // Hkv
    T = L + 13
    q = dyadic_bits(rng, (B, Hq, D))
    K = dyadic_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([L, max(1, L // 3)], np.int32)
    qd, Kd, Vd, Ld = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V), torch.from_numpy(lens).to(DEV)
    st = status_tensor()
    idx, cnt = ksa.ksa_select_tokens_per_head(qd, Kd, Ld, k, dev_status=st)
    ref_idx, ref_cnt = oracle.select_tokens_per_head(q, K, lens, k)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, Ld, idx, cnt, tokens_per_idx=1,
                                        idx_shared=ksa.IDX_PER_Q_HEAD, lse=lse, dev_status=st)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for h in range(Hq):
        g = h // G
        ref, ref_lse, _ = oracle.attention(q[:, h:h + 1], K[:, g:g + 1], V[:, g:g + 1], lens,
                                           ref_idx[:, h:h + 1], ref_cnt[:, h:h + 1], 1)
        assert_out_close(out[:, h], ref[:, 0])
        np.testing.assert_allclose(lse[:, h], ref_lse[:, 0], rtol=0, atol=LSE_TOL)
    assert st.item() == 0


@pytest.mark.parametrize("L,k", [(300, 40), (1500, 400), (90, 200)])
def test_random_head_selection_and_shared_attention(ksa, oracle, L, k):
    """Random-head aggregation: dyadic q, K give exact scores and ties; each row's shared set
    equals the oracle's for the drawn head, and attention over it (shared by all heads)
    equals the oracle's."""
    rng = np.random.default_rng(1700 + L)
    B, Hq, Hkv, D = 3, 8, 2, 128
    T = L + 13
    q = dyadic_bits(rng, (B, Hq, D))
    K = dyadic_bits(rng, (B, Hkv, T, D))
    V = rand_bits(rng, (B, Hkv, T, D))
    lens = np.array([L, max(1, L // 3), max(1, L - 7)], np.int32)
    heads = rng.integers(0, Hq, size=B).astype(np.int32)  # the random draw: an input
    qd, Kd, Vd, Ld = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V), torch.from_numpy(lens).to(DEV)
    st = status_tensor()
    idx, cnt = ksa.ksa_select_tokens_one_head(qd, Kd, Ld, heads, k, dev_status=st)
    ref_idx, ref_cnt = oracle.select_tokens_one_head(q, K, lens, heads, k)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, Ld, idx, cnt, tokens_per_idx=1,
                                        idx_shared=ksa.IDX_SHARED, lse=lse, dev_status=st)
    ref, ref_lse, _ = oracle.attention(q, K, V, lens, ref_idx, ref_cnt, 1, True)
    assert_out_close(out.cpu().numpy(), ref)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_TOL)
    assert st.item() == 0


@pytest.mark.parametrize("tpi", [4, 16, 64, 256])
def test_per_query_head_lists_of_blocks(ksa, oracle, tpi):
    """Lists per query head whose entries name runs of tpi tokens: runs of 16 or more go
    through the TMA producer (256, the largest run allowed, is 16 stages per entry), shorter
    ones through cp.async.  Ragged counts, one empty head, a partial last run; checked head
    by head against the oracle."""
    rng = np.random.default_rng(1800 + tpi)
    B, Hq, Hkv, D = 2, 8, 2, 128
    G = Hq // Hkv
    T = 64 * tpi
    q, K, V = (rand_bits(rng, s) for s in [(B, Hq, D), (B, Hkv, T, D), (B, Hkv, T, D)])
    lens = np.array([T - tpi // 2, 23 * tpi + 1], np.int32)
    cap = 12
    idx = np.full((B, Hq, cap), -1, np.int32)
    cnt = np.zeros((B, Hq), np.int32)
    for b in range(B):
        n_runs = -(-int(lens[b]) // tpi)
        for h in range(Hq):
            n = 0 if (b, h) == (1, 3) else int(rng.integers(1, cap + 1))
            pick = np.sort(rng.choice(n_runs, size=n, replace=False))
            if n and b == 0 and h == 0:
                pick[-1] = n_runs - 1  # the partial last run
                pick = np.unique(pick)
                n = len(pick)
            idx[b, h, :n] = pick
            cnt[b, h] = n
    qd, Kd, Vd, Ld = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V), torch.from_numpy(lens).to(DEV)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    st = status_tensor()
    out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, Ld, torch.from_numpy(idx).to(DEV),
                                        torch.from_numpy(cnt).to(DEV), tokens_per_idx=tpi,
                                        idx_shared=ksa.IDX_PER_Q_HEAD, lse=lse, dev_status=st)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for h in range(Hq):
        g = h // G
        ref, ref_lse, _ = oracle.attention(q[:, h:h + 1], K[:, g:g + 1], V[:, g:g + 1], lens,
                                           idx[:, h:h + 1], cnt[:, h:h + 1], tpi)
        assert_out_close(out[:, h], ref[:, 0], what=f"head {h}")
        fin = np.isfinite(ref_lse[:, 0])
        np.testing.assert_allclose(lse[fin, h], ref_lse[fin, 0], rtol=0, atol=LSE_TOL)
        assert np.all(np.isneginf(lse[~fin, h]))
    assert out[1, 3].max() == 0.0 and out[1, 3].min() == 0.0  # the empty head
    assert st.item() == 0


@pytest.mark.parametrize("layout", ["blocks", "shared_tokens", "dense"])
def test_outputs_lie_in_the_hull_of_the_selected_values(ksa, oracle, layout):
    """An invariant that needs no oracle: every output coordinate lies between the smallest
    and largest value of that coordinate over the selected V rows (softmax weights are
    non-negative and sum to 1), up to the fp32 accumulation tolerance."""
    rng = np.random.default_rng(1900 + len(layout))
    B, Hq, Hkv, D, T, bs = 3, 8, 2, 128, 1024, 16
    G = Hq // Hkv
    q, K, V = (rand_bits(rng, s, 2.0) for s in [(B, Hq, D), (B, Hkv, T, D), (B, Hkv, T, D)])
    lens = np.array([T, 517, 40], np.int32)
    qd, Kd, Vd, Ld = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V), torch.from_numpy(lens).to(DEV)
    Vv = bf16_value(V)
    sel = np.zeros((B, Hkv, T), bool)
    if layout == "blocks":
        k = 9
        idx = np.full((B, Hkv, k), -1, np.int32)
        cnt = np.zeros((B, Hkv), np.int32)
        for b in range(B):
            nb = -(-int(lens[b]) // bs)
            for g in range(Hkv):
                pick = np.sort(rng.choice(nb, size=min(k, nb), replace=False))
                idx[b, g, :len(pick)] = pick
                cnt[b, g] = len(pick)
                for j in pick:
                    sel[b, g, j * bs:min((j + 1) * bs, lens[b])] = True
        out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, Ld, torch.from_numpy(idx).to(DEV),
                                            torch.from_numpy(cnt).to(DEV), tokens_per_idx=bs)
    elif layout == "shared_tokens":
        k = 30
        idx = np.stack([np.sort(rng.choice(int(lens[b]), size=k, replace=False))
                        for b in range(B)]).astype(np.int32)
        cnt = np.full((B,), k, np.int32)
        for b in range(B):
            sel[b, :, idx[b]] = True
        out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, Ld, torch.from_numpy(idx).to(DEV),
                                            torch.from_numpy(cnt).to(DEV), tokens_per_idx=1,
                                            idx_shared=ksa.IDX_SHARED)
    else:
        for b in range(B):
            sel[b, :, :lens[b]] = True
        out, _ = ksa.ksa_sparse_decode_attn(qd, Kd, Vd, Ld)
    out = out.cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            rows = Vv[b, h // G][sel[b, h // G]]
            assert np.all(out[b, h] >= rows.min(0) - 2e-3), (b, h)
            assert np.all(out[b, h] <= rows.max(0) + 2e-3), (b, h)


@pytest.mark.parametrize("mode", ["dense", "blocks"])
def test_nan_poisoned_partials_are_never_read_stale(ksa, oracle, mode):
    """The workspace's split-row partial region starts as NaN (its semaphores zero, as the
    API asks): rows split over a hundred or more CTAs still match the oracle, so every
    partial the merge reads was written by this call."""
    rng = np.random.default_rng(2000 + len(mode))
    B, Hq, Hkv, D, T, bs = 2, 8, 2, 128, 32768, 16
    q, K, V = (rand_bits(rng, s) for s in [(B, Hq, D), (B, Hkv, T, D), (B, Hkv, T, D)])
    lens = np.array([T, T - 1000], np.int32)
    idx = cnt = None
    tpi = 1
    cap = T
    if mode == "blocks":
        tpi, cap = bs, 1500
        idx = np.full((B, Hkv, cap), -1, np.int32)
        cnt = np.zeros((B, Hkv), np.int32)
        for b in range(B):
            nb = -(-int(lens[b]) // bs)
            for g in range(Hkv):
                idx[b, g] = np.sort(rng.choice(nb, size=cap, replace=False))
                cnt[b, g] = cap
    need = ksa.lib().ksa_sparse_decode_attn_workspace(
        ctypes.byref(ksa.Shape(B, Hq, Hkv, D, T, bs)), cap, tpi)
    head = (B * Hq * 4 + 255) // 256 * 256
    ws = torch.zeros((need,), dtype=torch.uint8, device=DEV)
    ws[head:].view(torch.float32).fill_(float("nan"))
    qd, Kd, Vd, Ld = to_dev_bf16(q), to_dev_bf16(K), to_dev_bf16(V), torch.from_numpy(lens).to(DEV)
    st = status_tensor()
    out, _ = ksa.ksa_sparse_decode_attn(
        qd, Kd, Vd, Ld, None if idx is None else torch.from_numpy(idx).to(DEV),
        None if cnt is None else torch.from_numpy(cnt).to(DEV), tokens_per_idx=tpi,
        workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got = out.cpu().numpy()
    assert np.all(np.isfinite(got))
    ref, _, _ = oracle.attention(q, K, V, lens, idx, cnt, tpi)
    assert_out_close(got, ref)
