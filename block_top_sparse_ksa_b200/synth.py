"""Seeded synthetic decode workloads (shared by the tests and the benchmark).

This module only draws random numbers and lays them out: it holds none of the
method's arithmetic (no block means, no scores, no selection, no softmax), so
the CUDA path and the CPU oracle can both be fed from it without sharing any
step of the computation.

Shapes and value recipes stand in for the workloads the sources describe:
Qwen3-0.6B and Qwen3-8B shaped decode attention at 16K-32K context (the
Kinetics block top-k throughput runs) and a 20K-token, 32-head, top-4000
trace (the LessIsMore locality analysis).  No dataset or trained weight is
used; everything is drawn from ``torch.Generator`` seeded per workload.

All K/V caches are ``[B, Hkv, T, D]`` bf16, queries ``[B, Hq, D]`` bf16,
sequence lengths ``[B]`` int32.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

GiB = 1 << 30


@dataclasses.dataclass
class DecodeShape:
    """One decode-attention layer: sizes of the cache and of the selection."""

    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    capacity: int  # T, tokens the cache can hold per row
    block_size: int  # bs
    k_blocks: int  # K' blocks kept per (row, kv-head)
    min_len: int  # sequence lengths drawn uniformly in [min_len, max_len]
    max_len: int

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_blocks(self) -> int:
        return -(-self.capacity // self.block_size)


@dataclasses.dataclass
class UnifiedShape:
    """LessIsMore: one selection layer followed by ``sparse_layers`` layers."""

    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    capacity: int
    seq_len: int
    per_head_topk: int
    token_budget: int
    recent_tokens: int
    sparse_layers: int


# Workloads named by what they are.  Sizes follow the sources' shapes.
TINY = DecodeShape("tiny-block-topk-b1-h4kv2-d64-L2048-bs16-k8", 1, 4, 2, 64, 2048, 16, 8,
                   2048, 2048)
QWEN3_0_6B = DecodeShape("qwen3-0.6b-decode-b64-L16384-bs32-k32", 64, 16, 8, 128, 16384, 32,
                         32, 16384, 16384)
QWEN3_8B = DecodeShape("qwen3-8b-decode-b32-L16k..32k-bs16-k128", 32, 32, 8, 128, 32768, 16,
                       128, 16384, 32768)
LESSISMORE = UnifiedShape("lessismore-qwen3-8b-b16-L20000-P4000-budget4000-R1000", 16, 32, 8,
                          128, 20000, 20000, 4000, 4000, 1000, 3)


def sweep_shape(context: int, budget_tokens: int, cache_bytes: int = 40 * GiB) -> DecodeShape:
    """Throughput sweep point: Hq 32, Hkv 8, D 128, bs 16, batch sized so K+V ~ cache_bytes."""
    hkv, d, bs = 8, 128, 16
    batch = max(1, cache_bytes // (hkv * d * 2 * 2 * context))
    k = max(1, budget_tokens // bs)
    return DecodeShape(f"sweep-L{context}-budget{budget_tokens}-b{batch}", batch, 32, hkv, d,
                       context, bs, k, context, context)


# ---------------------------------------------------------------------------
# primitive draws


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen, device, std: float = 1.0) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std


def unit_group_direction(q_bf16: torch.Tensor, num_kv_heads: int) -> torch.Tensor:
    """Unit vector along the sum of each kv-group's queries: [B, Hkv, D] fp32.

    Used only to plant query-aligned keys (input construction)."""
    B, Hq, D = q_bf16.shape
    qs = q_bf16.float().view(B, num_kv_heads, Hq // num_kv_heads, D).sum(2)
    return qs / qs.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def draw_seq_lens(shape: DecodeShape, gen, device) -> torch.Tensor:
    if shape.min_len == shape.max_len:
        return torch.full((shape.batch,), shape.max_len, dtype=torch.int32, device=device)
    return torch.randint(shape.min_len, shape.max_len + 1, (shape.batch,), generator=gen,
                         device=device, dtype=torch.int64).to(torch.int32)


@dataclasses.dataclass
class DecodeInputs:
    shape: DecodeShape
    q: torch.Tensor  # [B, Hq, D] bf16
    K: torch.Tensor  # [B, Hkv, T, D] bf16
    V: torch.Tensor  # [B, Hkv, T, D] bf16
    seq_lens: torch.Tensor  # [B] int32
    planted: Optional[torch.Tensor] = None  # [B, Hkv, n_plant] block ids that got aligned keys


def make_decode_inputs(shape: DecodeShape, seed: int, device="cpu", *, recipe: str = "iid",
                       plant_blocks: int = 0, plant_scale: float = 0.5,
                       group_noise: Optional[float] = None, block_offset_std: float = 0.0,
                       poison_tail: Optional[float] = None) -> DecodeInputs:
    """Draw one decode layer.

    recipe pieces (combined as the workload asks):
      * q, K, V ~ N(0, 1), rounded to bf16;
      * group_noise: q_h = q_group + N(0, group_noise^2) for the heads of a kv-group;
      * block_offset_std: every (row, kv-head, block) adds one offset vector
        ~ N(0, block_offset_std^2) to all its keys;
      * plant_blocks: that many seeded blocks per (row, kv-head) get every key
        shifted by plant_scale * u_g (u_g = unit vector of the group's query sum);
      * poison_tail: cache slots t >= L_b hold this constant (K and V) so a read
        past the sequence end shows up in the results.
    """
    del recipe
    dev = torch.device(device)
    gen = _gen(seed, dev)
    B, Hq, Hkv, D, T, bs = (shape.batch, shape.num_q_heads, shape.num_kv_heads,
                            shape.head_dim, shape.capacity, shape.block_size)
    G = Hq // Hkv
    seq_lens = draw_seq_lens(shape, gen, dev)
    if group_noise is None:
        q = _randn((B, Hq, D), gen, dev)
    else:
        base = _randn((B, Hkv, 1, D), gen, dev)
        q = (base + _randn((B, Hkv, G, D), gen, dev, group_noise)).view(B, Hq, D)
    q = q.to(torch.bfloat16)
    nb = shape.max_blocks
    planted = None
    if plant_blocks > 0:
        keys = torch.rand((B, Hkv, nb), generator=gen, device=dev)
        # only blocks that hold tokens of the row can be planted
        nb_row = (seq_lens.to(torch.int64) + bs - 1) // bs
        keys = torch.where(torch.arange(nb, device=dev)[None, None, :] < nb_row[:, None, None],
                           keys, torch.full_like(keys, 2.0))
        planted = torch.argsort(keys, dim=-1)[..., :plant_blocks].to(torch.int32)
        u = unit_group_direction(q, Hkv)  # [B, Hkv, D]
    K = torch.empty((B, Hkv, T, D), dtype=torch.bfloat16, device=dev)
    V = torch.empty((B, Hkv, T, D), dtype=torch.bfloat16, device=dev)
    for b in range(B):  # one row at a time keeps the fp32 scratch small
        kb = _randn((Hkv, T, D), gen, dev)
        if block_offset_std > 0.0:
            off = _randn((Hkv, nb, 1, D), gen, dev, block_offset_std)
            kb = kb + off.expand(Hkv, nb, bs, D).reshape(Hkv, nb * bs, D)[:, :T]
        if planted is not None:
            shift = torch.zeros((Hkv, nb, D), device=dev)
            shift.scatter_(1, planted[b].long()[..., None].expand(-1, -1, D),
                           (plant_scale * u[b])[:, None, :].expand(-1, plant_blocks, -1))
            kb = kb + shift.repeat_interleave(bs, dim=1)[:, :T]
        K[b] = kb.to(torch.bfloat16)
        V[b] = _randn((Hkv, T, D), gen, dev).to(torch.bfloat16)
    if poison_tail is not None:
        t = torch.arange(T, device=dev)
        mask = t[None, :] >= seq_lens.to(dev)[:, None]  # [B, T]
        K.masked_fill_(mask[:, None, :, None], poison_tail)
        V.masked_fill_(mask[:, None, :, None], poison_tail)
    return DecodeInputs(shape, q, K, V, seq_lens, planted)


def make_queries(shape: DecodeShape, seed: int, count: int, device="cpu",
                 group_noise: Optional[float] = None) -> torch.Tensor:
    """``count`` independent query sets [count, B, Hq, D] bf16 (one per decode step)."""
    dev = torch.device(device)
    gen = _gen(seed, dev)
    B, Hq, Hkv, D = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim
    if group_noise is None:
        q = _randn((count, B, Hq, D), gen, dev)
    else:
        base = _randn((count, B, Hkv, 1, D), gen, dev)
        q = (base + _randn((count, B, Hkv, Hq // Hkv, D), gen, dev, group_noise)).view(
            count, B, Hq, D)
    return q.to(torch.bfloat16)


# Standard recipes of the named workloads -----------------------------------


def tiny_inputs(seed: int = 1001, device="cpu", **kw) -> DecodeInputs:
    """q,K,V ~ N(0,1) -> bf16; 4 blocks per (row, kv-head) get keys + 0.5 u_g."""
    return make_decode_inputs(TINY, seed, device, plant_blocks=4, plant_scale=0.5, **kw)


def qwen3_0_6b_inputs(seed: int = 1002, device="cpu", shape: DecodeShape = QWEN3_0_6B,
                      **kw) -> DecodeInputs:
    """K,V ~ N(0,1); 5% of blocks query-aligned (+0.5 u_g); q_h = q_g + N(0, 0.1^2)."""
    n_plant = max(1, round(0.05 * shape.max_blocks))
    return make_decode_inputs(shape, seed, device, plant_blocks=n_plant, plant_scale=0.5,
                              group_noise=0.1, **kw)


def qwen3_8b_inputs(seed: int = 1003, device="cpu", shape: DecodeShape = QWEN3_8B,
                    **kw) -> DecodeInputs:
    """L_b ~ U[16384, 32768]; K = N(0,1) + per-block offset N(0, 0.3^2); V, q ~ N(0,1)."""
    return make_decode_inputs(shape, seed, device, block_offset_std=0.3, **kw)


def sweep_inputs(shape: DecodeShape, seed: int = 1005, device="cpu", **kw) -> DecodeInputs:
    """Sweep point: q, K, V ~ N(0,1)."""
    return make_decode_inputs(shape, seed, device, **kw)


def dyadic(x: torch.Tensor, step: float = 0.25, lim: float = 4.0) -> torch.Tensor:
    """Snap to multiples of ``step`` clipped to [-lim, lim] (exact in bf16).

    With step 1/4 and |x| <= 4 every product is a multiple of 1/16 and every
    dot product over D <= 128 is an integer multiple of 1/16 below 2^15/16, so
    it is exact in fp32 whatever the summation order."""
    return (torch.round(x / step) * step).clamp(-lim, lim)


@dataclasses.dataclass
class UnifiedInputs:
    shape: UnifiedShape
    q_sel: torch.Tensor  # [B, Hq, D] bf16, selection layer (dyadic)
    K_sel: torch.Tensor  # [B, Hkv, T, D] bf16, selection layer (dyadic)
    seq_lens: torch.Tensor  # [B] int32
    layers: list  # [(q, K, V)] for the sparse layers, N(0,1) bf16


def lessismore_inputs(seed: int = 1004, device="cpu", shape: UnifiedShape = LESSISMORE,
                      with_layers: bool = True) -> UnifiedInputs:
    """Selection layer with dyadic q, K (exact scores on any hardware), then
    ``sparse_layers`` layers with independent N(0,1) q, K, V."""
    dev = torch.device(device)
    gen = _gen(seed, dev)
    B, Hq, Hkv, D, T = (shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim,
                        shape.capacity)
    seq_lens = torch.full((B,), shape.seq_len, dtype=torch.int32, device=dev)
    q_sel = dyadic(_randn((B, Hq, D), gen, dev)).to(torch.bfloat16)
    K_sel = torch.empty((B, Hkv, T, D), dtype=torch.bfloat16, device=dev)
    for b in range(B):
        K_sel[b] = dyadic(_randn((Hkv, T, D), gen, dev)).to(torch.bfloat16)
    layers = []
    if with_layers:
        for _ in range(shape.sparse_layers):
            q = _randn((B, Hq, D), gen, dev).to(torch.bfloat16)
            K = torch.empty((B, Hkv, T, D), dtype=torch.bfloat16, device=dev)
            V = torch.empty((B, Hkv, T, D), dtype=torch.bfloat16, device=dev)
            for b in range(B):
                K[b] = _randn((Hkv, T, D), gen, dev).to(torch.bfloat16)
                V[b] = _randn((Hkv, T, D), gen, dev).to(torch.bfloat16)
            layers.append((q, K, V))
    return UnifiedInputs(shape, q_sel, K_sel, seq_lens, layers)


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")

