"""ksa_sparse_decode_attn_noalloc: the attention entry point for callers that
cannot allocate device memory (a serving loop with no new device memory after
start-up, or a layer handed only its input and output buffers and no
allocator).  It runs on a fixed scratch
area inside the library instead of a caller workspace.

Its output must match ksa_sparse_decode_attn's (same tolerance as the parity
tests), on two calls in a row: the second call sees the scratch exactly as the
first left it.  This file sorts last so that a stopping run has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.helpers import LSE_TOL, assert_out_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ksa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_top_sparse_ksa_b200 as k
    k.lib()
    return k


def _inputs(B, Hq, Hkv, D, T, bs, k, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    q = torch.randn((B, Hq, D), generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn((B, Hkv, T, D), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((B, Hkv, T, D), generator=g, device="cuda").to(torch.bfloat16)
    lens = torch.randint(T // 2, T + 1, (B,), generator=g, device="cuda").to(torch.int32)
    nb = (lens.long() + bs - 1) // bs
    keys = torch.rand((B, Hkv, T // bs), generator=g, device="cuda")
    keys = torch.where(torch.arange(T // bs, device="cuda")[None, None] < nb[:, None, None],
                       keys, torch.full_like(keys, 2.0))
    idx = torch.sort(torch.argsort(keys, dim=-1)[..., :k], dim=-1).values.to(torch.int32)
    cnt = torch.full((B, Hkv), k, dtype=torch.int32, device="cuda")
    return q, K, V, lens, idx.contiguous(), cnt


def _raw_noalloc(ksa, q, K, V, lens, idx, cnt, bs, out, lse):
    """Call the C ABI directly (ctypes), the way a C caller would."""
    B, Hq, D = q.shape
    _, Hkv, T, _ = K.shape
    sh = ksa.Shape(B, Hq, Hkv, D, T, bs)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ksa.lib().ksa_sparse_decode_attn_noalloc(
        ctypes.byref(sh), p(q), p(K), p(V), p(lens), p(idx), p(cnt), idx.shape[-1], bs, 0, 0.0,
        0, p(out), p(lse), None, stream)


@pytest.mark.parametrize("B,Hq,Hkv,D,T,bs,k", [
    (16, 16, 8, 128, 4096, 32, 16),   # many rows: most rows held by one CTA
    (1, 8, 2, 128, 32768, 16, 1024),  # two long rows split over many CTAs (partials + semaphores)
    (3, 8, 4, 64, 2048, 16, 40),      # D = 64
    (8, 16, 8, 128, 16384, 16, 512),  # 32768 stages, ~74 per CTA: most rows split in two
])
def test_noalloc_matches_workspace_entry_point_twice(ksa, B, Hq, Hkv, D, T, bs, k):
    q, K, V, lens, idx, cnt = _inputs(B, Hq, Hkv, D, T, bs, k, seed=B * 1000 + T)
    ref, ref_lse = ksa.ksa_sparse_decode_attn(
        q, K, V, lens, idx, cnt, tokens_per_idx=bs,
        lse=torch.empty((B, Hq), dtype=torch.float32, device="cuda"))
    for call in range(2):
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        assert _raw_noalloc(ksa, q, K, V, lens, idx, cnt, bs, out, lse) == 0, ksa.ksa_last_error()
        torch.cuda.synchronize()
        assert_out_close(out.cpu().numpy(), ref.cpu().numpy(), what=f"call {call}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=0, atol=LSE_TOL)


def test_noalloc_binding_and_size_limit(ksa):
    q, K, V, lens, idx, cnt = _inputs(2, 4, 2, 128, 1024, 16, 8, seed=7)
    ref, _ = ksa.ksa_sparse_decode_attn(q, K, V, lens, idx, cnt, tokens_per_idx=16)
    out, _ = ksa.ksa_sparse_decode_attn_noalloc(q, K, V, lens, idx, cnt, tokens_per_idx=16)
    assert_out_close(out.cpu().numpy(), ref.cpu().numpy())
    # a shape whose workspace exceeds the fixed scratch is refused before any work
    big = ksa.Shape(65536, 64, 64, 128, 16, 16)  # 4M row semaphores alone need 16 MiB, twice the 8 MiB scratch
    fake = ctypes.c_void_p(0x1000)
    st = ksa.lib().ksa_sparse_decode_attn_noalloc(
        ctypes.byref(big), fake, fake, fake, fake, None, None, 0, 1, 0, 0.0, 0, fake, None, None,
        None)
    assert st == 2  # KSA_ERR_UNSUPPORTED
    assert "scratch" in ksa.ksa_last_error()
