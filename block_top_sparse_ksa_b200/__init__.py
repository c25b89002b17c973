"""block_top_sparse_ksa_b200 -- Python binding of libksa (include/ksa.h).

Block top-k sparse decode attention over a GQA KV cache and LessIsMore unified
token selection on NVIDIA B200.  This module only marshals arguments: it takes
torch CUDA tensors (device memory) and the current torch CUDA stream, and calls
the C ABI.  Every step of the computation runs in libksa's CUDA kernels; there
is no CPU or PyTorch fallback.  If ``libksa.so`` is missing, loading fails with
an error that says how to build it.

Layouts (row-major, contiguous):
  q [B, Hq, D] bf16;  K, V [B, Hkv, T, D] bf16;  seq_lens [B] int32;
  summaries [B, Hkv, ceil(T/bs), D] fp32 or bf16, or fp8: a uint8 tensor of
  that shape (the e4m3 values) whose storage holds the per-block fp32 scales
  right after it (alloc_summaries, fp8_summary_scales);  block_idx [B, Hkv, k]
  int32.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

__all__ = [
    "KsaError", "Shape", "lib", "library_path", "ksa_build_block_summaries",
    "ksa_select_blocks", "ksa_sparse_decode_attn", "ksa_unified_select",
    "ksa_select_blocks_workspace", "ksa_sparse_decode_attn_workspace",
    "ksa_sparse_decode_attn_noalloc", "ksa_decode_select_blocks",
    "ksa_unified_select_workspace", "ksa_status_string", "ksa_last_error", "ksa_version",
    "ksa_build_block_summaries_ex", "ksa_select_blocks_ex", "ksa_decode_select_blocks_ex",
    "ksa_build_block_summaries_paged", "ksa_decode_select_blocks_paged",
    "ksa_sparse_decode_attn_paged", "Pages", "ksa_select_window", "ksa_select_tokens_per_head",
    "ksa_select_tokens_per_head_workspace", "ksa_select_tokens_one_head",
    "ksa_select_tokens_one_head_workspace", "ksa_get_device_status", "IDX_PER_KV_HEAD",
    "IDX_SHARED", "IDX_PER_Q_HEAD", "ksa_append_kv", "ksa_append_kv_paged", "ksa_decode_step",
    "ksa_decode_step_workspace",
    "SUMMARY_ALL", "SUMMARY_LAST_BLOCK", "SUMMARIES_F32", "SUMMARIES_BF16", "SUMMARIES_FP8",
    "OUT_F32", "OUT_BF16", "alloc_summaries", "fp8_summary_scales",
    "FLAG_SEQ_LEN_CLAMPED",
    "FLAG_INDEX_SKIPPED", "FLAG_NONFINITE_SCORE", "FLAG_WAIT_TIMEOUT",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libksa.so")

SUMMARY_ALL, SUMMARY_LAST_BLOCK = 0, 1
SUMMARIES_F32, SUMMARIES_BF16, SUMMARIES_FP8 = 0, 1, 2
IDX_PER_KV_HEAD, IDX_SHARED, IDX_PER_Q_HEAD = 0, 1, 2
OUT_F32, OUT_BF16 = 0, 1
FLAG_SEQ_LEN_CLAMPED, FLAG_INDEX_SKIPPED, FLAG_NONFINITE_SCORE, FLAG_WAIT_TIMEOUT = 1, 2, 4, 8
_STATUS = {0: "KSA_OK", 1: "KSA_ERR_INVALID_ARG", 2: "KSA_ERR_UNSUPPORTED",
           3: "KSA_ERR_WORKSPACE", 4: "KSA_ERR_CUDA"}


class KsaError(RuntimeError):
    """A libksa call returned a non-OK status."""

    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("block_size", ctypes.c_int32)]


class Pages(ctypes.Structure):
    """ksa_pages: the block table of a paged K/V cache (page = block)."""
    _fields_ = [("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "ksa_build_block_summaries": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _i32, _vp, _vp, _vp]),
    "ksa_build_block_summaries_ex": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _i32, _i32, _vp,
                                            _vp, _vp]),
    "ksa_select_blocks_ex": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _i32, _vp, _i32, _vp, _vp,
                                    _vp, _sz, _vp, _vp]),
    "ksa_decode_select_blocks_ex": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _i32, _vp, _i32,
                                           _vp, _vp, _vp, _sz, _vp, _vp]),
    "ksa_build_block_summaries_paged": (_i32, [ctypes.POINTER(Shape), _vp, ctypes.POINTER(Pages),
                                               _vp, _i32, _i32, _vp, _vp, _vp]),
    "ksa_decode_select_blocks_paged": (_i32, [ctypes.POINTER(Shape), _vp, _vp,
                                              ctypes.POINTER(Pages), _vp, _i32, _vp, _i32, _vp,
                                              _vp, _vp, _sz, _vp, _vp]),
    "ksa_sparse_decode_attn_paged": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp,
                                            ctypes.POINTER(Pages), _vp, _vp, _vp, _i32, _i32,
                                            _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp, _vp]),
    "ksa_decode_step_workspace": (_sz, [ctypes.POINTER(Shape), _i32]),
    "ksa_decode_step": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _i32, _vp, _i32, _vp,
                               _vp, _f32, _i32, _vp, _vp, _vp, _sz, _vp, _vp]),
    "ksa_append_kv": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ksa_append_kv_paged": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp,
                                   ctypes.POINTER(Pages), _vp, _vp, _vp]),
    "ksa_select_window": (_i32, [ctypes.POINTER(Shape), _vp, _i32, _vp, _vp, _vp, _vp]),
    "ksa_select_tokens_per_head_workspace": (_sz, [ctypes.POINTER(Shape), _i32]),
    "ksa_select_tokens_one_head_workspace": (_sz, [ctypes.POINTER(Shape), _i32]),
    "ksa_get_device_status": (_i32, [_vp, _vp, _i32, ctypes.POINTER(ctypes.c_uint32)]),
    "ksa_select_tokens_one_head": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _i32, _vp,
                                          _vp, _vp, _sz, _vp, _vp]),
    "ksa_select_tokens_per_head": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _i32, _vp, _vp,
                                          _vp, _sz, _vp, _vp]),
    "ksa_select_blocks_workspace": (_sz, [ctypes.POINTER(Shape), _i32]),
    "ksa_select_blocks": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _i32, _vp, _vp, _vp, _sz,
                                 _vp, _vp]),
    "ksa_decode_select_blocks": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _i32, _vp,
                                        _vp, _vp, _sz, _vp, _vp]),
    "ksa_sparse_decode_attn_workspace": (_sz, [ctypes.POINTER(Shape), _i32, _i32]),
    "ksa_sparse_decode_attn": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                      _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp, _vp]),
    "ksa_sparse_decode_attn_noalloc": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp,
                                              _vp, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp,
                                              _vp]),
    "ksa_unified_select_workspace": (_sz, [ctypes.POINTER(Shape), _i32, _i32]),
    "ksa_unified_select": (_i32, [ctypes.POINTER(Shape), _vp, _vp, _vp, _i32, _i32, _i32, _vp,
                                  _vp, _vp, _sz, _vp, _vp]),
    "ksa_status_string": (ctypes.c_char_p, [_i32]),
    "ksa_last_error": (ctypes.c_char_p, []),
    "ksa_version": (_i32, []),
}

_LIB: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded libksa (raises if it was never built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(library_path):
            raise RuntimeError(
                f"{library_path} is missing: build it with "
                "`python -m block_top_sparse_ksa_b200.build` (needs nvcc)")
        handle = ctypes.CDLL(library_path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def ksa_status_string(status: int) -> str:
    return lib().ksa_status_string(int(status)).decode()


def ksa_last_error() -> str:
    return lib().ksa_last_error().decode()


def ksa_version() -> int:
    return int(lib().ksa_version())


# ---------------------------------------------------------------------------
# marshalling helpers


def _check(status: int) -> None:
    if status != 0:
        raise KsaError(status, ksa_last_error())


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _shape(B, Hq, Hkv, D, T, bs=16) -> Shape:
    return Shape(int(B), int(Hq), int(Hkv), int(D), int(T), int(bs))


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)


def _summary_dtype(summaries: torch.Tensor) -> int:
    """KSA_SUMMARIES_* code of a summaries tensor (fp32, bf16, or uint8 for fp8)."""
    if summaries.dtype == torch.float32:
        return SUMMARIES_F32
    if summaries.dtype == torch.bfloat16:
        return SUMMARIES_BF16
    if summaries.dtype == torch.uint8:
        room = summaries.untyped_storage().nbytes() - summaries.storage_offset()
        if summaries.dim() != 4 or room < summaries.numel() * (summaries.shape[-1] + 4) // (
                summaries.shape[-1]):
            raise ValueError("fp8 summaries: a [B, Hkv, nb, D] uint8 tensor whose storage holds "
                             "B*Hkv*nb fp32 scales after it (see alloc_summaries)")
        return SUMMARIES_FP8
    raise TypeError(f"summaries must be float32, bfloat16 or uint8 (fp8), not {summaries.dtype}")


def alloc_summaries(B: int, Hkv: int, nb: int, D: int, dtype="fp32", device="cuda",
                    fill: Optional[float] = None) -> torch.Tensor:
    """Block-summary storage [B, Hkv, nb, D]: dtype torch.float32 / "fp32", torch.bfloat16 /
    "bf16", or "fp8" (uint8 e4m3 values, the nb fp32 scales per (row, kv-head) stored right
    after them in the same allocation).  `fill`: an initial value for fp32/bf16 storage."""
    if dtype in (torch.float32, "fp32", "f32"):
        S = torch.empty((B, Hkv, nb, D), dtype=torch.float32, device=device)
    elif dtype in (torch.bfloat16, "bf16"):
        S = torch.empty((B, Hkv, nb, D), dtype=torch.bfloat16, device=device)
    elif dtype == "fp8":
        n = B * Hkv * nb
        return torch.zeros((n * (D + 4),), dtype=torch.uint8, device=device)[:n * D].view(
            B, Hkv, nb, D)
    else:
        raise ValueError(f"unknown summary dtype {dtype!r}")
    if fill is not None:
        S.fill_(fill)
    return S


def fp8_summary_scales(S: torch.Tensor) -> torch.Tensor:
    """The per-block fp32 scales [B, Hkv, nb] stored after fp8 summaries S."""
    B, Hkv, nb, D = S.shape
    n = B * Hkv * nb
    raw = torch.as_strided(S, (n * 4,), (1,), S.storage_offset() + S.numel())
    return raw.view(torch.float32).view(B, Hkv, nb)


def ksa_build_block_summaries(K: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                              mode: int = SUMMARY_ALL, summaries: Optional[torch.Tensor] = None,
                              dev_status: Optional[torch.Tensor] = None, stream=None,
                              summary_dtype=torch.float32) -> torch.Tensor:
    """Block mean keys S [B, Hkv, ceil(T/bs), D] (all blocks, or the last one), stored as
    fp32, bf16 or fp8: the given tensor's type, else `summary_dtype` (torch.float32,
    torch.bfloat16 or "fp8"; see alloc_summaries)."""
    _dev(K, "K", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hkv, T, D = K.shape
    nb = -(-T // block_size)
    if summaries is None:
        summaries = alloc_summaries(B, Hkv, nb, D, summary_dtype, K.device)
    _dev(summaries, "summaries", summaries.dtype)
    sh = _shape(B, Hkv, Hkv, D, T, block_size)
    _check(lib().ksa_build_block_summaries_ex(
        ctypes.byref(sh), _ptr(K), _ptr(seq_lens), int(mode), _summary_dtype(summaries),
        _ptr(summaries), _ptr(dev_status), _stream(stream)))
    return summaries


ksa_build_block_summaries_ex = ksa_build_block_summaries


def _workspace(ws: Optional[torch.Tensor], sh: Shape, args, kind: str, device) -> torch.Tensor:
    """The caller's workspace as given (the library checks its size), or a fresh zero-filled
    one of the size the matching *_workspace query returns (see include/ksa.h)."""
    if ws is not None:
        if not ws.is_cuda or not ws.is_contiguous():
            raise TypeError("workspace must be a contiguous CUDA tensor")
        return ws
    if kind == "select":
        need = lib().ksa_select_blocks_workspace(ctypes.byref(sh), args)
    else:
        need = lib().ksa_sparse_decode_attn_workspace(ctypes.byref(sh), *args)
    return torch.zeros((max(int(need), 1),), dtype=torch.uint8, device=device)


def ksa_select_blocks_workspace(B: int, Hq: int, Hkv: int, D: int, T: int, block_size: int,
                                k_blocks: int) -> int:
    sh = _shape(B, Hq, Hkv, D, T, block_size)
    return int(lib().ksa_select_blocks_workspace(ctypes.byref(sh), int(k_blocks)))


def ksa_select_blocks(q: torch.Tensor, summaries: torch.Tensor, seq_lens: torch.Tensor,
                      block_size: int, capacity: int, k_blocks: int,
                      block_idx: Optional[torch.Tensor] = None,
                      num_sel: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None,
                      dev_status: Optional[torch.Tensor] = None, stream=None):
    """Top-k blocks per (row, kv-head): (block_idx [B,Hkv,k] ascending -1 padded, num_sel [B,Hkv]).
    The summaries' dtype (fp32 or bf16) selects their storage type."""
    _dev(q, "q", torch.bfloat16)
    _dev(summaries, "summaries", summaries.dtype)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    Hkv = summaries.shape[1]
    if block_idx is None:
        block_idx = torch.empty((B, Hkv, k_blocks), dtype=torch.int32, device=q.device)
    if num_sel is None:
        num_sel = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    sh = _shape(B, Hq, Hkv, D, capacity, block_size)
    ws = _workspace(workspace, sh, int(k_blocks), "select", q.device)
    _check(lib().ksa_select_blocks_ex(ctypes.byref(sh), _ptr(q), _ptr(summaries),
                                      _summary_dtype(summaries), _ptr(seq_lens), int(k_blocks),
                                      _ptr(block_idx), _ptr(num_sel), _ptr(ws),
                                      ws.numel() * ws.element_size(), _ptr(dev_status),
                                      _stream(stream)))
    return block_idx, num_sel


ksa_select_blocks_ex = ksa_select_blocks


def ksa_decode_select_blocks(q: torch.Tensor, K: torch.Tensor, summaries: torch.Tensor,
                             seq_lens: torch.Tensor, block_size: int, k_blocks: int,
                             block_idx: Optional[torch.Tensor] = None,
                             num_sel: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None,
                             dev_status: Optional[torch.Tensor] = None, stream=None):
    """Refresh every row's last-block summary from K, then select (one launch)."""
    _dev(q, "q", torch.bfloat16)
    _dev(K, "K", torch.bfloat16)
    _dev(summaries, "summaries", summaries.dtype)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    _, Hkv, T, _ = K.shape
    if block_idx is None:
        block_idx = torch.empty((B, Hkv, k_blocks), dtype=torch.int32, device=q.device)
    if num_sel is None:
        num_sel = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    sh = _shape(B, Hq, Hkv, D, T, block_size)
    ws = _workspace(workspace, sh, int(k_blocks), "select", q.device)
    _check(lib().ksa_decode_select_blocks_ex(
        ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(summaries), _summary_dtype(summaries),
        _ptr(seq_lens), int(k_blocks), _ptr(block_idx), _ptr(num_sel), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))
    return block_idx, num_sel


ksa_decode_select_blocks_ex = ksa_decode_select_blocks


def ksa_decode_step_workspace(B: int, Hq: int, Hkv: int, D: int, T: int, block_size: int,
                              k_blocks: int) -> int:
    sh = _shape(B, Hq, Hkv, D, T, block_size)
    return int(lib().ksa_decode_step_workspace(ctypes.byref(sh), int(k_blocks)))


def ksa_decode_step(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, summaries: torch.Tensor,
                    seq_lens: torch.Tensor, block_size: int, k_blocks: int,
                    block_idx: Optional[torch.Tensor] = None,
                    num_sel: Optional[torch.Tensor] = None, scale: float = 0.0,
                    out_dtype: int = OUT_F32, out: Optional[torch.Tensor] = None,
                    lse: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None,
                    dev_status: Optional[torch.Tensor] = None, stream=None):
    """One decode step in one call: last-block refresh, scoring, top-k and attention over the
    kept blocks -> (block_idx [B,Hkv,k], num_sel [B,Hkv], out [B,Hq,D], lse or None)."""
    _dev(q, "q", torch.bfloat16)
    _dev(K, "K", torch.bfloat16)
    _dev(V, "V", torch.bfloat16)
    _dev(summaries, "summaries", summaries.dtype)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    _, Hkv, T, _ = K.shape
    if block_idx is None:
        block_idx = torch.empty((B, Hkv, k_blocks), dtype=torch.int32, device=q.device)
    if num_sel is None:
        num_sel = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    odt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((B, Hq, D), dtype=odt, device=q.device)
    _dev(out, "out", odt)
    if lse is not None:
        _dev(lse, "lse", torch.float32)
    sh = _shape(B, Hq, Hkv, D, T, block_size)
    if workspace is None:  # zero-filled once (see include/ksa.h)
        need = lib().ksa_decode_step_workspace(ctypes.byref(sh), int(k_blocks))
        workspace = torch.zeros((max(int(need), 1),), dtype=torch.uint8, device=q.device)
    elif not workspace.is_cuda or not workspace.is_contiguous():
        raise TypeError("workspace must be a contiguous CUDA tensor")
    _check(lib().ksa_decode_step(
        ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(V), _ptr(summaries), _summary_dtype(summaries),
        _ptr(seq_lens), int(k_blocks), _ptr(block_idx), _ptr(num_sel), float(scale),
        int(out_dtype), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))
    return block_idx, num_sel, out, lse


def ksa_sparse_decode_attn(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                           seq_lens: torch.Tensor, idx: Optional[torch.Tensor] = None,
                           num_idx: Optional[torch.Tensor] = None, tokens_per_idx: int = 1,
                           idx_shared: int = IDX_PER_KV_HEAD, scale: float = 0.0,
                           out_dtype: int = OUT_F32, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None,
                           dev_status: Optional[torch.Tensor] = None, stream=None):
    """Softmax attention over the selected tokens (dense when idx is None): (out, lse)."""
    _dev(q, "q", torch.bfloat16)
    _dev(K, "K", torch.bfloat16)
    _dev(V, "V", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    _, Hkv, T, _ = K.shape
    cap = 0
    if idx is not None:
        _dev(idx, "idx", torch.int32)
        _dev(num_idx, "num_idx", torch.int32)
        cap = idx.shape[-1]
    odt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((B, Hq, D), dtype=odt, device=q.device)
    _dev(out, "out", odt)
    if lse is not None:
        _dev(lse, "lse", torch.float32)
    sh = _shape(B, Hq, Hkv, D, T, max(1, tokens_per_idx))
    ws = _workspace(workspace, sh, (int(cap), int(tokens_per_idx)), "attn", q.device)
    _check(lib().ksa_sparse_decode_attn(
        ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(V), _ptr(seq_lens), _ptr(idx), _ptr(num_idx),
        int(cap), int(tokens_per_idx), int(idx_shared), float(scale), int(out_dtype),
        _ptr(out), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status),
        _stream(stream)))
    return out, lse


def ksa_sparse_decode_attn_noalloc(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                                   seq_lens: torch.Tensor, idx: Optional[torch.Tensor] = None,
                                   num_idx: Optional[torch.Tensor] = None,
                                   tokens_per_idx: int = 1, idx_shared: int = IDX_PER_KV_HEAD,
                                   scale: float = 0.0, out_dtype: int = OUT_F32,
                                   out: Optional[torch.Tensor] = None,
                                   lse: Optional[torch.Tensor] = None,
                                   dev_status: Optional[torch.Tensor] = None, stream=None):
    """ksa_sparse_decode_attn on the library's fixed scratch (no workspace argument).

    For callers that must not allocate device memory; see include/ksa.h.  Calls
    that may overlap on the GPU share the scratch and race."""
    _dev(q, "q", torch.bfloat16)
    _dev(K, "K", torch.bfloat16)
    _dev(V, "V", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    _, Hkv, T, _ = K.shape
    cap = 0
    if idx is not None:
        _dev(idx, "idx", torch.int32)
        _dev(num_idx, "num_idx", torch.int32)
        cap = idx.shape[-1]
    odt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((B, Hq, D), dtype=odt, device=q.device)
    _dev(out, "out", odt)
    if lse is not None:
        _dev(lse, "lse", torch.float32)
    sh = _shape(B, Hq, Hkv, D, T, max(1, tokens_per_idx))
    _check(lib().ksa_sparse_decode_attn_noalloc(
        ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(V), _ptr(seq_lens), _ptr(idx), _ptr(num_idx),
        int(cap), int(tokens_per_idx), int(idx_shared), float(scale), int(out_dtype),
        _ptr(out), _ptr(lse), _ptr(dev_status), _stream(stream)))
    return out, lse


def ksa_sparse_decode_attn_workspace(B: int, Hq: int, Hkv: int, D: int, T: int,
                                     idx_capacity: int = 0, tokens_per_idx: int = 1) -> int:
    sh = _shape(B, Hq, Hkv, D, T, max(1, tokens_per_idx))
    return int(lib().ksa_sparse_decode_attn_workspace(ctypes.byref(sh), int(idx_capacity),
                                                      int(tokens_per_idx)))


def ksa_unified_select_workspace(B: int, Hq: int, Hkv: int, D: int, T: int, per_head_topk: int,
                                 token_budget: int) -> int:
    sh = _shape(B, Hq, Hkv, D, T)
    return int(lib().ksa_unified_select_workspace(ctypes.byref(sh), int(per_head_topk),
                                                  int(token_budget)))


def ksa_unified_select(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor,
                       per_head_topk: int, token_budget: int, recent_tokens: int = -1,
                       token_idx: Optional[torch.Tensor] = None,
                       num_sel: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None,
                       dev_status: Optional[torch.Tensor] = None, stream=None):
    """LessIsMore selection: (token_idx [B, budget] ascending -1 padded, num_sel [B])."""
    _dev(q, "q", torch.bfloat16)
    _dev(K, "K", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    _, Hkv, T, _ = K.shape
    if workspace is None:  # the unified workspace needs no initialisation
        need = ksa_unified_select_workspace(B, Hq, Hkv, D, T, per_head_topk, token_budget)
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    if token_idx is None:
        token_idx = torch.empty((B, token_budget), dtype=torch.int32, device=q.device)
    if num_sel is None:
        num_sel = torch.empty((B,), dtype=torch.int32, device=q.device)
    sh = _shape(B, Hq, Hkv, D, T)
    _check(lib().ksa_unified_select(
        ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(seq_lens), int(per_head_topk),
        int(token_budget), int(recent_tokens), _ptr(token_idx), _ptr(num_sel), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))
    return token_idx, num_sel


# ---------------------------------------------------------------------------
# paged K/V cache: pools [num_pages, Hkv, block_size, D] bf16 and a block table
# [B, max_blocks] int32 naming the page of each logical block


def _pages(block_table: torch.Tensor, num_pages: int) -> Pages:
    _dev(block_table, "block_table", torch.int32)
    return Pages(ctypes.c_void_p(block_table.data_ptr()), int(block_table.shape[1]),
                 int(num_pages))


def ksa_build_block_summaries_paged(K_pages: torch.Tensor, block_table: torch.Tensor,
                                    seq_lens: torch.Tensor, mode: int = SUMMARY_ALL,
                                    summaries: Optional[torch.Tensor] = None,
                                    dev_status: Optional[torch.Tensor] = None, stream=None,
                                    summary_dtype=torch.float32) -> torch.Tensor:
    """ksa_build_block_summaries on a paged key cache; the page size is the block size."""
    _dev(K_pages, "K_pages", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    P, Hkv, bs, D = K_pages.shape
    B, mb = block_table.shape
    if summaries is None:
        summaries = alloc_summaries(B, Hkv, mb, D, summary_dtype, K_pages.device)
    _dev(summaries, "summaries", summaries.dtype)
    sh = _shape(B, Hkv, Hkv, D, mb * bs, bs)
    pg = _pages(block_table, P)
    _check(lib().ksa_build_block_summaries_paged(
        ctypes.byref(sh), _ptr(K_pages), ctypes.byref(pg), _ptr(seq_lens), int(mode),
        _summary_dtype(summaries), _ptr(summaries), _ptr(dev_status), _stream(stream)))
    return summaries


def ksa_decode_select_blocks_paged(q: torch.Tensor, K_pages: torch.Tensor,
                                   block_table: torch.Tensor, summaries: torch.Tensor,
                                   seq_lens: torch.Tensor, k_blocks: int,
                                   block_idx: Optional[torch.Tensor] = None,
                                   num_sel: Optional[torch.Tensor] = None,
                                   workspace: Optional[torch.Tensor] = None,
                                   dev_status: Optional[torch.Tensor] = None, stream=None):
    """ksa_decode_select_blocks on a paged key cache."""
    _dev(q, "q", torch.bfloat16)
    _dev(K_pages, "K_pages", torch.bfloat16)
    _dev(summaries, "summaries", summaries.dtype)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    P, Hkv, bs, _ = K_pages.shape
    mb = block_table.shape[1]
    if block_idx is None:
        block_idx = torch.empty((B, Hkv, k_blocks), dtype=torch.int32, device=q.device)
    if num_sel is None:
        num_sel = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    sh = _shape(B, Hq, Hkv, D, mb * bs, bs)
    pg = _pages(block_table, P)
    ws = _workspace(workspace, sh, int(k_blocks), "select", q.device)
    _check(lib().ksa_decode_select_blocks_paged(
        ctypes.byref(sh), _ptr(q), _ptr(K_pages), ctypes.byref(pg), _ptr(summaries),
        _summary_dtype(summaries), _ptr(seq_lens), int(k_blocks), _ptr(block_idx), _ptr(num_sel),
        _ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))
    return block_idx, num_sel


def ksa_sparse_decode_attn_paged(q: torch.Tensor, K_pages: torch.Tensor, V_pages: torch.Tensor,
                                 block_table: torch.Tensor, seq_lens: torch.Tensor,
                                 idx: Optional[torch.Tensor] = None,
                                 num_idx: Optional[torch.Tensor] = None, tokens_per_idx: int = 1,
                                 idx_shared: int = IDX_PER_KV_HEAD, scale: float = 0.0,
                                 out_dtype: int = OUT_F32, out: Optional[torch.Tensor] = None,
                                 lse: Optional[torch.Tensor] = None,
                                 workspace: Optional[torch.Tensor] = None,
                                 dev_status: Optional[torch.Tensor] = None, stream=None):
    """ksa_sparse_decode_attn on a paged K/V cache: (out, lse)."""
    _dev(q, "q", torch.bfloat16)
    _dev(K_pages, "K_pages", torch.bfloat16)
    _dev(V_pages, "V_pages", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    P, Hkv, bs, _ = K_pages.shape
    mb = block_table.shape[1]
    odt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((B, Hq, D), dtype=odt, device=q.device)
    _dev(out, "out", odt)
    if lse is not None:
        _dev(lse, "lse", torch.float32)
    cap = 0
    if idx is not None:
        _dev(idx, "idx", torch.int32)
        _dev(num_idx, "num_idx", torch.int32)
        cap = idx.shape[-1]
    sh = _shape(B, Hq, Hkv, D, mb * bs, bs)
    pg = _pages(block_table, P)
    ws = _workspace(workspace, sh, (int(cap), int(tokens_per_idx)), "attn", q.device)
    _check(lib().ksa_sparse_decode_attn_paged(
        ctypes.byref(sh), _ptr(q), _ptr(K_pages), _ptr(V_pages), ctypes.byref(pg),
        _ptr(seq_lens), _ptr(idx), _ptr(num_idx), int(cap), int(tokens_per_idx),
        int(idx_shared), float(scale), int(out_dtype), _ptr(out), _ptr(lse), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))
    return out, lse


def ksa_append_kv(k_new: torch.Tensor, v_new: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                  seq_lens: torch.Tensor, dev_status: Optional[torch.Tensor] = None,
                  stream=None) -> None:
    """Write the new token's rows: K[b, g, L_b - 1] = k_new[b, g], V likewise (k_new, v_new
    [B, Hkv, D] bf16; seq_lens already counts the new token)."""
    _dev(k_new, "k_new", torch.bfloat16)
    _dev(v_new, "v_new", torch.bfloat16)
    _dev(K, "K", torch.bfloat16)
    _dev(V, "V", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hkv, T, D = K.shape
    if tuple(k_new.shape) != (B, Hkv, D) or tuple(v_new.shape) != (B, Hkv, D):
        raise ValueError(f"k_new and v_new must be [{B}, {Hkv}, {D}]")
    sh = _shape(B, Hkv, Hkv, D, T)
    _check(lib().ksa_append_kv(ctypes.byref(sh), _ptr(k_new), _ptr(v_new), _ptr(K), _ptr(V),
                               _ptr(seq_lens), _ptr(dev_status), _stream(stream)))


def ksa_append_kv_paged(k_new: torch.Tensor, v_new: torch.Tensor, K_pages: torch.Tensor,
                        V_pages: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor,
                        dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ksa_append_kv on a paged K/V cache (pools [num_pages, Hkv, bs, D], block table
    [B, max_blocks])."""
    _dev(k_new, "k_new", torch.bfloat16)
    _dev(v_new, "v_new", torch.bfloat16)
    _dev(K_pages, "K_pages", torch.bfloat16)
    _dev(V_pages, "V_pages", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    P, Hkv, bs, D = K_pages.shape
    B, mb = block_table.shape
    if tuple(k_new.shape) != (B, Hkv, D) or tuple(v_new.shape) != (B, Hkv, D):
        raise ValueError(f"k_new and v_new must be [{B}, {Hkv}, {D}]")
    sh = _shape(B, Hkv, Hkv, D, mb * bs, bs)
    pg = _pages(block_table, P)
    _check(lib().ksa_append_kv_paged(ctypes.byref(sh), _ptr(k_new), _ptr(v_new), _ptr(K_pages),
                                     _ptr(V_pages), ctypes.byref(pg), _ptr(seq_lens),
                                     _ptr(dev_status), _stream(stream)))


def ksa_select_window(seq_lens: torch.Tensor, num_kv_heads: int, block_size: int, capacity: int,
                      k_blocks: int, block_idx: Optional[torch.Tensor] = None,
                      num_sel: Optional[torch.Tensor] = None,
                      dev_status: Optional[torch.Tensor] = None, stream=None):
    """Local attention as a block selection: (block_idx [B,Hkv,k] ascending -1 padded,
    num_sel [B,Hkv]) = each row's last min(k, NB_b) blocks."""
    _dev(seq_lens, "seq_lens", torch.int32)
    B = seq_lens.shape[0]
    if block_idx is None:
        block_idx = torch.empty((B, num_kv_heads, k_blocks), dtype=torch.int32,
                                device=seq_lens.device)
    if num_sel is None:
        num_sel = torch.empty((B, num_kv_heads), dtype=torch.int32, device=seq_lens.device)
    sh = _shape(B, num_kv_heads, num_kv_heads, 64, capacity, block_size)
    _check(lib().ksa_select_window(ctypes.byref(sh), _ptr(seq_lens), int(k_blocks),
                                   _ptr(block_idx), _ptr(num_sel), _ptr(dev_status),
                                   _stream(stream)))
    return block_idx, num_sel


def ksa_select_tokens_per_head_workspace(B: int, Hq: int, Hkv: int, D: int, T: int,
                                         k_tokens: int) -> int:
    sh = _shape(B, Hq, Hkv, D, T)
    return int(lib().ksa_select_tokens_per_head_workspace(ctypes.byref(sh), int(k_tokens)))


def ksa_select_tokens_per_head(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor,
                               k_tokens: int, token_idx: Optional[torch.Tensor] = None,
                               num_sel: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None,
                               dev_status: Optional[torch.Tensor] = None, stream=None):
    """Each query head's own top-k tokens: (token_idx [B,Hq,k] ascending -1 padded,
    num_sel [B,Hq]); attend with idx_shared=IDX_PER_Q_HEAD, tokens_per_idx=1."""
    _dev(q, "q", torch.bfloat16)
    _dev(K, "K", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    _, Hkv, T, _ = K.shape
    if workspace is None:  # no initialisation needed
        need = ksa_select_tokens_per_head_workspace(B, Hq, Hkv, D, T, k_tokens)
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    if token_idx is None:
        token_idx = torch.empty((B, Hq, k_tokens), dtype=torch.int32, device=q.device)
    if num_sel is None:
        num_sel = torch.empty((B, Hq), dtype=torch.int32, device=q.device)
    sh = _shape(B, Hq, Hkv, D, T)
    _check(lib().ksa_select_tokens_per_head(
        ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(seq_lens), int(k_tokens), _ptr(token_idx),
        _ptr(num_sel), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(dev_status), _stream(stream)))
    return token_idx, num_sel


def ksa_select_tokens_one_head_workspace(B: int, Hq: int, Hkv: int, D: int, T: int,
                                         k_tokens: int) -> int:
    sh = _shape(B, Hq, Hkv, D, T)
    return int(lib().ksa_select_tokens_one_head_workspace(ctypes.byref(sh), int(k_tokens)))


def ksa_select_tokens_one_head(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor,
                               head_of_row, k_tokens: int,
                               token_idx: Optional[torch.Tensor] = None,
                               num_sel: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None,
                               dev_status: Optional[torch.Tensor] = None, stream=None):
    """Random-head aggregation: row b's set is query head head_of_row[b]'s own top-k tokens,
    shared by every head: (token_idx [B,k] ascending -1 padded, num_sel [B]); attend with
    idx_shared=IDX_SHARED, tokens_per_idx=1.  head_of_row: B heads in [0, Hq) on the host
    (a list, a numpy array or a CPU tensor), drawn by the caller."""
    _dev(q, "q", torch.bfloat16)
    _dev(K, "K", torch.bfloat16)
    _dev(seq_lens, "seq_lens", torch.int32)
    B, Hq, D = q.shape
    _, Hkv, T, _ = K.shape
    heads = (head_of_row.detach().cpu().numpy() if isinstance(head_of_row, torch.Tensor)
             else np.asarray(head_of_row))
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    if heads.shape != (B,):
        raise ValueError(f"head_of_row must hold {B} heads, got shape {heads.shape}")
    if workspace is None:  # no initialisation needed
        need = ksa_select_tokens_one_head_workspace(B, Hq, Hkv, D, T, k_tokens)
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    if token_idx is None:
        token_idx = torch.empty((B, k_tokens), dtype=torch.int32, device=q.device)
    if num_sel is None:
        num_sel = torch.empty((B,), dtype=torch.int32, device=q.device)
    _dev(token_idx, "token_idx", torch.int32)
    _dev(num_sel, "num_sel", torch.int32)
    if token_idx.numel() < B * k_tokens or num_sel.numel() < B:
        raise ValueError("token_idx must hold [B, k_tokens] and num_sel [B] entries")
    sh = _shape(B, Hq, Hkv, D, T)
    _check(lib().ksa_select_tokens_one_head(
        ctypes.byref(sh), _ptr(q), _ptr(K), _ptr(seq_lens),
        heads.ctypes.data_as(ctypes.c_void_p), int(k_tokens), _ptr(token_idx), _ptr(num_sel),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
        _stream(stream)))
    return token_idx, num_sel


def ksa_get_device_status(dev_status: torch.Tensor, clear: bool = False, stream=None) -> int:
    """The KSA_FLAG_* bits collected in a device status word (waits for `stream`); with clear,
    the word is zeroed afterwards on the stream."""
    if not isinstance(dev_status, torch.Tensor) or not dev_status.is_cuda:
        raise TypeError("dev_status must be a CUDA tensor")
    if dev_status.element_size() * dev_status.numel() < 4:
        raise ValueError("dev_status must hold one 32-bit word")
    flags = ctypes.c_uint32(0)
    _check(lib().ksa_get_device_status(_ptr(dev_status), _stream(stream), int(bool(clear)),
                                       ctypes.byref(flags)))
    return int(flags.value)
