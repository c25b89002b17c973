"""A decode step recorded into a CUDA graph and replayed.

A serving loop records its decode step once and replays it every token.  The
step's launches take plain device pointers and a caller-owned workspace, so a
replay must reproduce the eager results bit for bit.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ksa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import block_top_sparse_ksa_b200 as k
    k.lib()
    return k


def _inputs(B, Hq, Hkv, D, T, bs, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    q = torch.randn((B, Hq, D), generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn((B, Hkv, T, D), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((B, Hkv, T, D), generator=g, device="cuda").to(torch.bfloat16)
    lens = torch.randint(T // 2, T + 1, (B,), generator=g, device="cuda").to(torch.int32)
    return q, K, V, lens


def test_decode_step_replays_as_a_cuda_graph(ksa):
    """A whole decode step -- the fused last-block refresh, scoring and top-k, then the
    attention -- recorded once into a CUDA graph and replayed: every replay reproduces the
    eagerly computed indices, counts, outputs and lse bit for bit."""
    B, Hq, Hkv, D, T, bs, k = 8, 16, 8, 128, 4096, 32, 16
    q, K, V, lens = _inputs(B, Hq, Hkv, D, T, bs, seed=99)
    S = ksa.ksa_build_block_summaries(K, lens, bs)
    ws = torch.zeros((ksa.ksa_select_blocks_workspace(B, Hq, Hkv, D, T, bs, k),),
                     dtype=torch.uint8, device="cuda")
    idx = torch.empty((B, Hkv, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    ws_att = torch.zeros((ksa.ksa_sparse_decode_attn_workspace(B, Hq, Hkv, D, T, k, bs),),
                         dtype=torch.uint8, device="cuda")
    out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")

    def step():
        ksa.ksa_decode_select_blocks(q, K, S, lens, bs, k, block_idx=idx, num_sel=cnt,
                                     workspace=ws)
        ksa.ksa_sparse_decode_attn(q, K, V, lens, idx, cnt, tokens_per_idx=bs, out=out, lse=lse,
                                   workspace=ws_att)

    # eager run on a side stream: the reference (and every launch's one-time setup, such as
    # the kernels' shared-memory limits, happens before the capture)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    ref = [t.clone() for t in (idx, cnt, out, lse)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        idx.fill_(-7)
        cnt.fill_(-7)
        out.fill_(-7.0)
        lse.fill_(-7.0)
        graph.replay()
        torch.cuda.synchronize()
        for got, want in zip((idx, cnt, out, lse), ref):
            assert torch.equal(got, want)
    del graph
