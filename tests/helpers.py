"""Test helpers: planted score gaps, tolerances, row sampling.

The gap planting uses the fp64 oracle to score blocks and nudges keys so that
the k-th and (k+1)-th block scores of every (row, kv-head) differ by at least
DELTA; then the selected block set is unique and can be compared bit-exactly.
It only edits inputs: nothing here comes from the CUDA library.
"""
from __future__ import annotations

import numpy as np

from oracle.oracle import bf16_bits, bf16_value

# Minimum planted gap between the k-th and (k+1)-th block scores.  The GPU
# scores carry fp32 rounding of order 1e-6 |s|, far below this.
DELTA = 1e-2

# Output tolerance (fp32 output, bf16 inputs, fp32 accumulation).
ABS_TOL = 2e-3
REL_TOL = 1e-2
LSE_TOL = 1e-4


def _row_scores(oracle, q_row, K, lens, bs, summary_bf16, summary_fp8=False):
    S = oracle.block_summaries(K[None], lens, bs)
    if summary_bf16:  # the scores the bf16-stored means give
        S = bf16_value(oracle.round_bf16(S))
    if summary_fp8:  # ... or the fp8-stored ones
        S = oracle.store_fp8(S)
    return oracle.block_scores(q_row[None], S, lens, bs)[0]  # [Hkv, nb]


def gap_fix_row(oracle, q_row: np.ndarray, K_row: np.ndarray, L: int, bs: int, k: int,
                delta: float = DELTA, max_iter: int = 20, summary_bf16: bool = False,
                summary_fp8: bool = False):
    """Plant a score gap >= delta at the top-k boundary of every kv-head of one row.

    q_row: uint16 [Hq, D] bits; K_row: uint16 [Hkv, T, D] bits (edited copy returned).
    Selected blocks that sit within delta of the best unselected score have all
    their valid keys moved along the group's query-sum direction until the
    boundary gap is at least delta (scored from bf16- or fp8-stored means when
    summary_bf16 / summary_fp8).  Returns (K_row, number of blocks moved)."""
    K = K_row.copy()
    Hq, D = q_row.shape
    Hkv, T, _ = K.shape
    G = Hq // Hkv
    qv = bf16_value(q_row)
    lens = np.array([L], np.int32)
    moved = 0
    for _ in range(max_iter):
        s = _row_scores(oracle, q_row, K, lens, bs, summary_bf16, summary_fp8)
        nb = -(-L // bs)
        if nb <= k:
            return K, moved
        ok = True
        for g in range(Hkv):
            sg = s[g, :nb]
            order = np.lexsort((np.arange(nb), -sg))  # score desc, index asc
            sel, rest = order[:k], order[k:]
            top_rest = sg[rest].max()
            low = sel[sg[sel] < top_rest + delta]
            if len(low) == 0:
                continue
            ok = False
            qs = qv[g * G:(g + 1) * G].sum(0)
            nrm = np.linalg.norm(qs)
            u = qs / nrm
            for j in low:
                need = (top_rest + 2 * delta - sg[j]) / nrm + 4.0 / 256
                t0, t1 = j * bs, min(j * bs + bs, L)
                K[g, t0:t1] = bf16_bits(bf16_value(K[g, t0:t1]) + need * u[None, :])
                moved += 1
        if ok:
            return K, moved
    raise AssertionError("could not plant the score gap")


def min_boundary_gap(oracle, q_row, K_row, L, bs, k, summary_bf16: bool = False,
                     summary_fp8: bool = False) -> float:
    lens = np.array([L], np.int32)
    s = _row_scores(oracle, q_row, K_row, lens, bs, summary_bf16, summary_fp8)
    nb = -(-L // bs)
    if nb <= k:
        return np.inf
    gaps = []
    for g in range(s.shape[0]):
        srt = np.sort(s[g, :nb])[::-1]
        gaps.append(srt[k - 1] - srt[k])
    return float(min(gaps))


def assert_out_close(got: np.ndarray, ref: np.ndarray, what: str = "out",
                     bf16_output: bool = False) -> None:
    """Spec tolerance: max|d| <= 2e-3 and max|d| / max|ref| <= 1e-2.
    bf16 output adds half an ulp of bf16 (2^-8 relative) to the absolute bound."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    d = np.abs(got - ref)
    if bf16_output:
        bound = ABS_TOL + 2.0 ** -8 * np.abs(ref)
        assert np.all(d <= bound), f"{what}: max excess {np.max(d - bound):.3e}"
    else:
        assert d.max() <= ABS_TOL, f"{what}: max abs err {d.max():.3e}"
        scale = max(np.abs(ref).max(), 1e-30)
        assert d.max() / scale <= REL_TOL, f"{what}: rel err {d.max() / scale:.3e}"


def sample_rows(B: int, seed: int, extra: int = 2):
    rng = np.random.default_rng(seed)
    rows = {0, B // 2, B - 1}
    if B > 3:
        rows.update(int(x) for x in rng.choice(B, size=min(extra, B), replace=False))
    return sorted(rows)
