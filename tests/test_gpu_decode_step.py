"""ksa_decode_step: one decode step in one call -- the last-block summary refresh, block
scoring, top-k and attention over the kept blocks (Kinetics press summary, section 5:
block top-k), issued as the launches of ksa_decode_select_blocks followed by
ksa_sparse_decode_attn on one workspace.  Its results must equal the two calls' bit for
bit, on repeated calls over one workspace too.  (Parity with the oracle is in
test_gpu_parity.py.)"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ksa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_top_sparse_ksa_b200 as k
    k.lib()
    return k


def _inputs(B, Hq, Hkv, D, T, bs, seed, block_offset=0.3):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = torch.randn((B, Hq, D), generator=g, device=DEV).to(torch.bfloat16)
    K = torch.randn((B, Hkv, T, D), generator=g, device=DEV)
    nb = -(-T // bs)
    off = torch.randn((B, Hkv, nb, 1, D), generator=g, device=DEV) * block_offset
    K = (K + off.expand(B, Hkv, nb, bs, D).reshape(B, Hkv, nb * bs, D)[:, :, :T]).to(
        torch.bfloat16)
    V = torch.randn((B, Hkv, T, D), generator=g, device=DEV).to(torch.bfloat16)
    lens = torch.randint(T // 2, T + 1, (B,), generator=g, device=DEV).to(torch.int32)
    lens[0] = T              # a full row
    if B > 2:
        lens[1] = 1          # a one-token row
        lens[2] = min(T, bs * 3 + 1)  # a short row with a one-token tail block
    return q, K, V, lens


def _prefill(ksa, K, lens, bs, sdt):
    """Summaries of the cache before the newest token; blocks never built hold NaN."""
    B, Hkv, T, D = K.shape
    S = torch.full((B, Hkv, -(-T // bs), D), float("nan"), dtype=sdt, device=DEV)
    ksa.ksa_build_block_summaries(K, (lens - 1).clamp_min(1), bs, summaries=S)
    return S


def _two_calls(ksa, q, K, V, S, lens, bs, k, out_dtype):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx, cnt = ksa.ksa_decode_select_blocks(q, K, S, lens, bs, k, dev_status=st)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=DEV)
    out, _ = ksa.ksa_sparse_decode_attn(q, K, V, lens, idx, cnt, tokens_per_idx=bs,
                                        out_dtype=out_dtype, lse=lse, dev_status=st)
    return idx, cnt, out, lse, st


def _one_call(ksa, q, K, V, S, lens, bs, k, out_dtype, ws=None):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=DEV)
    idx, cnt, out, _ = ksa.ksa_decode_step(q, K, V, S, lens, bs, k, out_dtype=out_dtype,
                                           lse=lse, workspace=ws, dev_status=st)
    return idx, cnt, out, lse, st


CASES = [
    # B, Hq, Hkv, D, T, bs, k, summaries, out dtype
    (3, 8, 2, 128, 40 * 16 + 7, 16, 8, torch.float32, 0),     # ragged capacity
    (4, 16, 8, 128, 4096, 32, 16, torch.float32, 0),          # the Qwen3-0.6B layout, short
    (3, 8, 4, 64, 2048, 16, 40, torch.float32, 1),            # D 64, bf16 output
    (5, 32, 8, 128, 32768, 16, 128, torch.float32, 0),        # 2048 blocks
    (3, 16, 8, 128, 8192, 32, 32, torch.bfloat16, 0),         # bf16 summaries
    (3, 8, 2, 128, 1100 * 16, 16, 50, torch.float32, 0),      # 1100 blocks
    (2, 8, 2, 128, 3000 * 16, 16, 64, torch.float32, 0),      # 3000 blocks
    (4, 8, 2, 128, 512, 16, 64, torch.float32, 0),            # k covers every block
    (64, 16, 8, 128, 16384, 32, 32, torch.float32, 0),        # Qwen3-0.6B step shape
    # between half and all of the resident attention CTAs' worth of rows (148 SMs x 3): the
    # attention grid is one CTA per row
    (32, 32, 8, 128, 8192, 16, 64, torch.float32, 0),         # 256 rows, 512 blocks
    (32, 32, 8, 128, 32768, 16, 128, torch.float32, 0),       # the Qwen3-8B step shape
    (28, 8, 8, 128, 4096, 16, 128, torch.float32, 1),         # rows kept whole and ranked
    (150, 8, 2, 64, 4096, 16, 24, torch.bfloat16, 0),         # D 64, bf16 summaries
    (55, 16, 8, 128, 10000, 32, 20, torch.bfloat16, 0),       # 440 rows
    (28, 8, 8, 64, 5200 * 16, 16, 64, torch.float32, 0),      # 5200 blocks
]


@pytest.mark.parametrize("B,Hq,Hkv,D,T,bs,k,sdt,odt", CASES,
                         ids=[f"B{c[0]}-D{c[3]}-T{c[4]}-bs{c[5]}-k{c[6]}-"
                              f"{'bf16' if c[7] == torch.bfloat16 else 'f32'}S-out{c[8]}"
                              for c in CASES])
def test_decode_step_equals_the_two_calls(ksa, B, Hq, Hkv, D, T, bs, k, sdt, odt):
    q, K, V, lens = _inputs(B, Hq, Hkv, D, T, bs, seed=B * 7919 + T)
    S0 = _prefill(ksa, K, lens, bs, sdt)
    S1, S2 = S0.clone(), S0.clone()
    ref = _two_calls(ksa, q, K, V, S1, lens, bs, k, odt)
    got = _one_call(ksa, q, K, V, S2, lens, bs, k, odt)
    torch.cuda.synchronize()
    names = ("block_idx", "num_sel", "out", "lse")
    for name, a, b in zip(names, got[:4], ref[:4]):
        assert torch.equal(a, b), name
    assert torch.equal(S2.view(torch.int32) if sdt == torch.float32 else S2.view(torch.int16),
                       S1.view(torch.int32) if sdt == torch.float32 else S1.view(torch.int16))
    assert got[4].item() == 0 and ref[4].item() == 0
    assert torch.isfinite(got[2].float()).all()


@pytest.mark.parametrize("B", [16, 32])
def test_decode_step_repeated_calls_on_one_workspace(ksa, B):
    """Calls back to back on one workspace, alternating two query sets and two caches: each
    result equals the first result for its inputs (every call leaves the workspace's
    semaphores as it found them).  With 32 rows of 8 kv-heads the attention grid is one
    CTA per row."""
    Hq, Hkv, D, T, bs, k = 32, 8, 128, 16384, 16, 64
    qa, Ka, Va, la = _inputs(B, Hq, Hkv, D, T, bs, seed=1)
    qb, Kb, Vb, lb = _inputs(B, Hq, Hkv, D, T, bs, seed=2)
    Sa = _prefill(ksa, Ka, la, bs, torch.float32)
    Sb = _prefill(ksa, Kb, lb, bs, torch.float32)
    ws = torch.zeros((ksa.ksa_decode_step_workspace(B, Hq, Hkv, D, T, bs, k),),
                     dtype=torch.uint8, device=DEV)
    first = {}
    for i in range(6):
        which = "a" if i % 2 == 0 else "b"
        q, K, V, lens, S = (qa, Ka, Va, la, Sa) if which == "a" else (qb, Kb, Vb, lb, Sb)
        res = _one_call(ksa, q, K, V, S, lens, bs, k, 0, ws=ws)
        torch.cuda.synchronize()
        assert res[4].item() == 0
        res = [t.clone() for t in res[:4]]
        if which not in first:
            first[which] = res
        else:
            for a, b in zip(res, first[which]):
                assert torch.equal(a, b)
    assert not torch.equal(first["a"][2], first["b"][2])


@pytest.mark.parametrize("B,Hkv", [(4, 2), (32, 8)])
def test_decode_step_flags_bad_lengths_and_nan_scores(ksa, B, Hkv):
    """Device-side data errors flag the status word as in the two calls: a seq_len outside
    [1, T] is clamped, a NaN summary ranks lowest."""
    Hq, D, T, bs, k = 8 * Hkv // 2, 128, 2048, 16, 8
    q, K, V, lens = _inputs(B, Hq, Hkv, D, T, bs, seed=3)
    S = _prefill(ksa, K, lens, bs, torch.float32)
    lens[3] = T + 5
    S[0, 1, 3] = float("nan")
    ref = _two_calls(ksa, q, K, V, S.clone(), lens, bs, k, 0)
    got = _one_call(ksa, q, K, V, S.clone(), lens, bs, k, 0)
    torch.cuda.synchronize()
    flags = ksa.FLAG_SEQ_LEN_CLAMPED | ksa.FLAG_NONFINITE_SCORE
    assert got[4].item() == ref[4].item() == flags
    for a, b in zip(got[:4], ref[:4]):
        assert torch.equal(a, b)
    assert 3 not in got[0][0, 1].tolist()
