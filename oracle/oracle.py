"""Python face of the fp64 CPU oracle (``ksa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product library
never imports this module and shares no code with it.

Arrays are numpy.  bf16 tensors are passed as ``uint16`` bit patterns (the C
side widens them to fp64 exactly).  Each wrapper names the step of the method
it computes; the definitions and the readings taken where the sources are
silent are written out in ``ksa_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ksa_oracle.c")
_LIB = os.path.join(_HERE, "libksa_oracle.so")

_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (strict IEEE: no fast-math, no contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
               "-shared", "-o", out, src, "-lm"]
        subprocess.run(cmd, check=True)
    return out


class Oracle:
    """ctypes binding of one compiled oracle library."""

    def __init__(self, path: str | None = None):
        self.lib = ctypes.CDLL(path or build())
        L = self.lib
        c_int, c_double = ctypes.c_int, ctypes.c_double
        nullable_f64 = ctypes.c_void_p
        L.ksa_oracle_block_summaries.argtypes = [c_int] * 5 + [_u16p, _i32p, _f64p]
        L.ksa_oracle_block_scores.argtypes = [c_int] * 6 + [_u16p, _f64p, _i32p, _f64p]
        L.ksa_oracle_topk.argtypes = [c_int, _f64p, c_int, _i32p]
        L.ksa_oracle_topk.restype = c_int
        L.ksa_oracle_select_blocks.argtypes = ([c_int] * 6 + [_u16p, _u16p, _i32p, c_int,
                                                _i32p, _i32p, nullable_f64])
        L.ksa_oracle_select_blocks_ex.argtypes = ([c_int] * 6 + [_u16p, _u16p, _i32p, c_int,
                                                   c_int, _i32p, _i32p, nullable_f64])
        L.ksa_oracle_select_tokens_per_head.argtypes = ([c_int] * 5 + [_u16p, _u16p, _i32p,
                                                        c_int, _i32p, _i32p])
        L.ksa_oracle_select_tokens_one_head.argtypes = ([c_int] * 5 + [_u16p, _u16p, _i32p,
                                                        _i32p, c_int, _i32p, _i32p])
        L.ksa_oracle_select_window.argtypes = [c_int] * 3 + [_i32p, c_int, _i32p, _i32p]
        L.ksa_oracle_gather_pages.argtypes = [c_int] * 6 + [_u16p, _i32p, _i32p, _u16p]
        L.ksa_oracle_round_bf16.argtypes = [c_double]
        L.ksa_oracle_round_bf16.restype = ctypes.c_uint16
        L.ksa_oracle_round_bf16_array.argtypes = [ctypes.c_size_t, _f64p, _u16p]
        L.ksa_oracle_round_e4m3.argtypes = [c_double]
        L.ksa_oracle_round_e4m3.restype = c_double
        L.ksa_oracle_e4m3_scale_exp.argtypes = [c_double]
        L.ksa_oracle_e4m3_scale_exp.restype = c_int
        L.ksa_oracle_store_fp8_blocks.argtypes = [ctypes.c_size_t, c_int, _f64p]
        L.ksa_oracle_attention.argtypes = ([c_int] * 5 + [_u16p, _u16p, _u16p, _i32p,
                                           ctypes.c_void_p, ctypes.c_void_p, c_int, c_int,
                                           c_int, c_double, _f64p, nullable_f64,
                                           nullable_f64])
        L.ksa_oracle_attention_recall.argtypes = ([c_int] * 5 + [_u16p, _u16p, _i32p, _i32p,
                                                  _i32p, c_int, c_int, c_int, c_double, _f64p])
        L.ksa_oracle_unified_select.argtypes = ([c_int] * 5 + [_u16p, _u16p, _i32p, c_int,
                                                c_int, c_int, _i32p, _i32p,
                                                ctypes.c_void_p])
        L.ksa_oracle_set_threads.argtypes = [c_int]
        L.ksa_oracle_max_threads.restype = c_int

    # -- threads ------------------------------------------------------------
    def set_threads(self, n: int) -> None:
        self.lib.ksa_oracle_set_threads(int(n))

    def max_threads(self) -> int:
        return int(self.lib.ksa_oracle_max_threads())

    # -- A1 -----------------------------------------------------------------
    def block_summaries(self, K: np.ndarray, seq_lens: np.ndarray, bs: int) -> np.ndarray:
        """Mean key of every block: K uint16 [B,Hkv,T,D] -> fp64 [B,Hkv,ceil(T/bs),D]."""
        K = np.ascontiguousarray(K, dtype=np.uint16)
        B, Hkv, T, D = K.shape
        nb = -(-T // bs)
        S = np.zeros((B, Hkv, nb, D), np.float64)
        self.lib.ksa_oracle_block_summaries(B, Hkv, T, D, bs, K,
                                            np.ascontiguousarray(seq_lens, np.int32), S)
        return S

    def gather_pages(self, pages: np.ndarray, block_table: np.ndarray,
                     seq_lens: np.ndarray) -> np.ndarray:
        """Logical cache of a paged one: pages uint16 [P,Hkv,bs,D], block_table int32
        [B,max_blocks] -> uint16 [B,Hkv,max_blocks*bs,D] (zero past L_b and for bad pages)."""
        pages = np.ascontiguousarray(pages, dtype=np.uint16)
        tbl = np.ascontiguousarray(block_table, dtype=np.int32)
        P, Hkv, bs, D = pages.shape
        B, mb = tbl.shape
        K = np.empty((B, Hkv, mb * bs, D), np.uint16)
        self.lib.ksa_oracle_gather_pages(B, Hkv, D, bs, mb, P, pages, tbl,
                                         np.ascontiguousarray(seq_lens, np.int32), K)
        return K

    def round_bf16(self, x) -> np.ndarray:
        """Nearest bf16 (ties to even) of fp64 values -> uint16 bit patterns, same shape."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty(x.shape, np.uint16)
        self.lib.ksa_oracle_round_bf16_array(x.size, x.reshape(-1), out.reshape(-1))
        return out

    def round_e4m3(self, x) -> np.ndarray:
        """Nearest fp8 e4m3 value (ties to even, held at +-448) of fp64 values, same shape."""
        x = np.asarray(x, dtype=np.float64)
        return np.vectorize(self.lib.ksa_oracle_round_e4m3, otypes=[np.float64])(x)

    def e4m3_scale_exp(self, amax: float) -> int:
        """Smallest e with amax <= 448 * 2^e (0 for amax == 0)."""
        return int(self.lib.ksa_oracle_e4m3_scale_exp(float(amax)))

    def store_fp8(self, S: np.ndarray) -> np.ndarray:
        """The stored values of block means [..., D] as fp8 e4m3 with a power-of-two scale
        per block (a copy, fp64)."""
        S = np.ascontiguousarray(S, dtype=np.float64).copy()
        D = S.shape[-1]
        self.lib.ksa_oracle_store_fp8_blocks(S.size // D, D, S.reshape(-1))
        return S

    def block_summaries_bf16(self, K: np.ndarray, seq_lens: np.ndarray, bs: int) -> np.ndarray:
        """The block means stored as bf16 -> uint16 bits [B,Hkv,ceil(T/bs),D]."""
        return self.round_bf16(self.block_summaries(K, seq_lens, bs))

    # -- A2 -----------------------------------------------------------------
    def block_scores(self, q: np.ndarray, S: np.ndarray, seq_lens: np.ndarray,
                     bs: int) -> np.ndarray:
        """Group-summed query against each block mean -> fp64 [B,Hkv,nb] (-inf past NB_b)."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        S = np.ascontiguousarray(S, dtype=np.float64)
        B, Hq, D = q.shape
        _, Hkv, nb, _ = S.shape
        s = np.empty((B, Hkv, nb), np.float64)
        self.lib.ksa_oracle_block_scores(B, Hq, Hkv, D, nb, bs, q, S,
                                         np.ascontiguousarray(seq_lens, np.int32), s)
        return s

    # -- A3 -----------------------------------------------------------------
    def topk(self, s: np.ndarray, k: int) -> np.ndarray:
        """Indices of the k largest entries (ties -> lower index), ascending."""
        s = np.ascontiguousarray(s, dtype=np.float64)
        out = np.full(max(k, 1), -1, np.int32)
        m = self.lib.ksa_oracle_topk(s.shape[0], s, k, out)
        return out[:m].copy()

    def select_blocks(self, q, K, seq_lens, bs: int, k: int, want_scores: bool = False,
                      summary_bf16: bool = False, summary_fp8: bool = False):
        """A1+A2+A3: (block_idx [B,Hkv,k] ascending -1 padded, num_sel [B,Hkv][, scores]).
        summary_bf16 / summary_fp8: the block means are stored as bf16 / as fp8 e4m3 with a
        power-of-two scale per block before scoring."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        K = np.ascontiguousarray(K, dtype=np.uint16)
        B, Hq, D = q.shape
        _, Hkv, T, _ = K.shape
        idx = np.empty((B, Hkv, k), np.int32)
        cnt = np.empty((B, Hkv), np.int32)
        scores = np.empty((B, Hkv, -(-T // bs)), np.float64) if want_scores else None
        self.lib.ksa_oracle_select_blocks_ex(
            B, Hq, Hkv, D, T, bs, q, K, np.ascontiguousarray(seq_lens, np.int32), k,
            2 if summary_fp8 else int(bool(summary_bf16)), idx, cnt,
            scores.ctypes.data if want_scores else None)
        return (idx, cnt, scores) if want_scores else (idx, cnt)

    def select_tokens_per_head(self, q, K, seq_lens, k: int):
        """Each query head's own top-k tokens (ties -> lower t), ascending, -1 padded:
        (token_idx [B,Hq,k], num_sel [B,Hq])."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        K = np.ascontiguousarray(K, dtype=np.uint16)
        B, Hq, D = q.shape
        _, Hkv, T, _ = K.shape
        idx = np.empty((B, Hq, k), np.int32)
        cnt = np.empty((B, Hq), np.int32)
        self.lib.ksa_oracle_select_tokens_per_head(B, Hq, Hkv, D, T, q, K,
                                                   np.ascontiguousarray(seq_lens, np.int32),
                                                   k, idx, cnt)
        return idx, cnt

    def select_tokens_one_head(self, q, K, seq_lens, head_of_row, k: int):
        """Random-head aggregation: row b's set is head head_of_row[b]'s own top-k tokens,
        shared by every head: (token_idx [B,k], num_sel [B])."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        K = np.ascontiguousarray(K, dtype=np.uint16)
        B, Hq, D = q.shape
        _, Hkv, T, _ = K.shape
        heads = np.ascontiguousarray(head_of_row, np.int32)
        if heads.shape != (B,) or heads.min() < 0 or heads.max() >= Hq:
            raise ValueError("head_of_row must hold one head in [0, Hq) per row")
        idx = np.empty((B, k), np.int32)
        cnt = np.empty((B,), np.int32)
        self.lib.ksa_oracle_select_tokens_one_head(B, Hq, Hkv, D, T, q, K,
                                                   np.ascontiguousarray(seq_lens, np.int32),
                                                   heads, k, idx, cnt)
        return idx, cnt

    def select_window(self, seq_lens, num_kv_heads: int, bs: int, k: int):
        """Local attention as a block selection: the last min(k, NB_b) blocks, ascending."""
        lens = np.ascontiguousarray(seq_lens, np.int32)
        B = lens.shape[0]
        idx = np.empty((B, num_kv_heads, k), np.int32)
        cnt = np.empty((B, num_kv_heads), np.int32)
        self.lib.ksa_oracle_select_window(B, num_kv_heads, bs, lens, k, idx, cnt)
        return idx, cnt

    # -- A4/A5/A7/A8 --------------------------------------------------------
    def attention(self, q, K, V, seq_lens, idx=None, num_idx=None, tokens_per_idx: int = 1,
                  shared: bool = False, scale: float = 0.0):
        """Softmax attention over the selected tokens -> (out fp64 [B,Hq,D], lse [B,Hq], wsum [B,Hq])."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        K = np.ascontiguousarray(K, dtype=np.uint16)
        V = np.ascontiguousarray(V, dtype=np.uint16)
        B, Hq, D = q.shape
        _, Hkv, T, _ = K.shape
        out = np.empty((B, Hq, D), np.float64)
        lse = np.empty((B, Hq), np.float64)
        wsum = np.empty((B, Hq), np.float64)
        if idx is None:
            idx_p = cnt_p = None
            cap = 0
            keep = ()
        else:
            idx = np.ascontiguousarray(idx, np.int32)
            num_idx = np.ascontiguousarray(num_idx, np.int32)
            cap = idx.shape[-1]
            idx_p, cnt_p = idx.ctypes.data, num_idx.ctypes.data
            keep = (idx, num_idx)  # noqa: F841  (keep buffers alive through the call)
        self.lib.ksa_oracle_attention(B, Hq, Hkv, D, T, q, K, V,
                                      np.ascontiguousarray(seq_lens, np.int32), idx_p, cnt_p,
                                      cap, tokens_per_idx, int(shared), float(scale), out,
                                      lse.ctypes.data, wsum.ctypes.data)
        del keep
        return out, lse, wsum

    def attention_recall(self, q, K, seq_lens, idx, num_idx, tokens_per_idx: int = 1,
                         shared: int = 0, scale: float = 0.0) -> np.ndarray:
        """Share of each query head's dense softmax weight on the selected tokens -> fp64
        [B,Hq].  shared: 0 lists per kv-head [B,Hkv,cap], 1 one list per row [B,cap],
        2 one list per query head [B,Hq,cap]."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        K = np.ascontiguousarray(K, dtype=np.uint16)
        B, Hq, D = q.shape
        _, Hkv, T, _ = K.shape
        idx = np.ascontiguousarray(idx, np.int32)
        num_idx = np.ascontiguousarray(num_idx, np.int32)
        rec = np.empty((B, Hq), np.float64)
        self.lib.ksa_oracle_attention_recall(B, Hq, Hkv, D, T, q, K,
                                             np.ascontiguousarray(seq_lens, np.int32), idx,
                                             num_idx, idx.shape[-1], tokens_per_idx, int(shared),
                                             float(scale), rec)
        return rec

    # -- A6 -----------------------------------------------------------------
    def unified_select(self, q, K, seq_lens, per_head_topk: int, token_budget: int,
                       recent_tokens: int, want_votes: bool = False):
        """LessIsMore selection -> (token_idx [B,budget] ascending -1 padded, num_sel [B][, votes])."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        K = np.ascontiguousarray(K, dtype=np.uint16)
        B, Hq, D = q.shape
        _, Hkv, T, _ = K.shape
        idx = np.empty((B, token_budget), np.int32)
        cnt = np.empty((B,), np.int32)
        votes = np.zeros((B, T), np.int32) if want_votes else None
        self.lib.ksa_oracle_unified_select(
            B, Hq, Hkv, D, T, q, K, np.ascontiguousarray(seq_lens, np.int32), per_head_topk,
            token_budget, recent_tokens, idx, cnt, votes.ctypes.data if want_votes else None)
        return (idx, cnt, votes) if want_votes else (idx, cnt)


_DEFAULT: Oracle | None = None


def get() -> Oracle:
    """The process-wide oracle instance (compiled on first use)."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT


def bf16_bits(x) -> np.ndarray:
    """Round an fp32/fp64 numpy array to bf16 (nearest-even) and return its bit pattern."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_value(bits) -> np.ndarray:
    """The exact value (fp64) of a bf16 bit pattern array."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
