"""Attention recall of a token selection, and the LessIsMore recency-ratio sweep.

LessIsMore (evaluation of the unified selection and of the recency window)
rates a selection by how much of each head's full attention it keeps.  For
query head h of row b and a selected token set T_sel,

    recall[b, h] = sum_{t in T_sel} softmax(z)_t,   z_t = scale * <q_h, K_t>, t < L_b,

and since softmax(z)_t = exp(z_t - lse(all)), the sum is exactly

    recall = exp(lse(T_sel) - lse(all)).

So recall takes two launches of the attention kernel -- the dense set and the
selection, of which only the log-sum-exps are used -- and no kernel of its
own.  The sweep varies the recency share of a fixed LessIsMore budget from 0
to 100% and reports the recall of the shared set in the selection layer and
in the sparse layers that reuse it.  Inputs are the seeded synthetic caches of
``synth``; no model is involved.

    python -m block_top_sparse_ksa_b200.recall [--batch 4] [--ratios 0,0.25,0.5,0.75,1]
"""
from __future__ import annotations

import argparse
import json
from typing import Optional, Sequence

import numpy as np
import torch

from . import (IDX_PER_Q_HEAD, IDX_SHARED, ksa_select_tokens_one_head,
               ksa_select_tokens_per_head, ksa_sparse_decode_attn, ksa_unified_select)


def attention_recall(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor,
                     idx: torch.Tensor, num_idx: torch.Tensor, tokens_per_idx: int = 1,
                     idx_shared: int = 0, scale: float = 0.0,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> np.ndarray:
    """recall [B, Hq] (fp64, host) of the selection (idx, num_idx) under the dense softmax."""
    B, Hq, D = q.shape
    lse_all = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    lse_sel = torch.empty_like(lse_all)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    ksa_sparse_decode_attn(q, K, V, seq_lens, scale=scale, out=out, lse=lse_all,
                           workspace=workspace, stream=stream)
    ksa_sparse_decode_attn(q, K, V, seq_lens, idx, num_idx, tokens_per_idx=tokens_per_idx,
                           idx_shared=idx_shared, scale=scale, out=out, lse=lse_sel,
                           workspace=workspace, stream=stream)
    a = lse_all.cpu().numpy().astype(np.float64)
    s = lse_sel.cpu().numpy().astype(np.float64)
    return np.exp(s - a)  # an empty selection has lse -inf: recall 0


def recency_sweep(inp, ratios: Sequence[float]) -> list:
    """For each recency share of the budget: mean recall of the unified set in the selection
    layer (its own q, K) and in each sparse layer (q, K, V of that layer)."""
    sh = inp.shape
    rows = []
    for ratio in ratios:
        R = int(round(ratio * sh.token_budget))
        tok, cnt = ksa_unified_select(inp.q_sel, inp.K_sel, inp.seq_lens, sh.per_head_topk,
                                      sh.token_budget, R)
        row = {"recent_share": ratio, "recent_tokens": R, "budget": sh.token_budget,
               "selection_layer": float(attention_recall(
                   inp.q_sel, inp.K_sel, inp.K_sel, inp.seq_lens, tok, cnt,
                   idx_shared=True).mean())}
        row["sparse_layers"] = [
            float(attention_recall(q, K, V, inp.seq_lens, tok, cnt, idx_shared=True).mean())
            for q, K, V in inp.layers]
        rows.append(row)
    return rows


def aggregation_comparison(inp, budget: int, seed: int = 0) -> dict:
    """The three ways LessIsMore's mechanism analysis turns the heads' choices into the set the
    layers read, each with the same token budget and no recency window: the unified vote, a
    set per query head, and one randomly drawn head's set (seeded draw, one head per row).
    Returns the mean recall of each in the selection layer and in the sparse layers."""
    B, Hq = inp.q_sel.shape[0], inp.q_sel.shape[1]
    heads = np.random.default_rng(seed).integers(0, Hq, size=B).astype(np.int32)
    sets = {
        "unified": ksa_unified_select(inp.q_sel, inp.K_sel, inp.seq_lens, budget, budget, 0)
        + (IDX_SHARED,),
        "per_head": ksa_select_tokens_per_head(inp.q_sel, inp.K_sel, inp.seq_lens, budget)
        + (IDX_PER_Q_HEAD,),
        "random_head": ksa_select_tokens_one_head(inp.q_sel, inp.K_sel, inp.seq_lens, heads,
                                                  budget) + (IDX_SHARED,),
    }
    res = {"budget": budget, "recent_tokens": 0, "heads": heads.tolist()}
    for name, (tok, cnt, layout) in sets.items():
        res[name] = {
            "selection_layer": float(attention_recall(inp.q_sel, inp.K_sel, inp.K_sel,
                                                      inp.seq_lens, tok, cnt,
                                                      idx_shared=layout).mean()),
            "sparse_layers": [float(attention_recall(q, K, V, inp.seq_lens, tok, cnt,
                                                     idx_shared=layout).mean())
                              for q, K, V in inp.layers]}
    return res


def main(argv=None) -> None:
    from . import synth
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--batch", type=int, default=4)
    p.add_argument("--ratios", default="0,0.1,0.25,0.5,0.75,1")
    p.add_argument("--seed", type=int, default=1004)
    p.add_argument("--aggregation", action="store_true",
                   help="also compare unified, per-head and random-head sets")
    args = p.parse_args(argv)
    shape = synth.dataclasses.replace(synth.LESSISMORE, batch=args.batch)
    inp = synth.lessismore_inputs(seed=args.seed, device="cuda", shape=shape)
    for row in recency_sweep(inp, [float(x) for x in args.ratios.split(",")]):
        print(json.dumps({"workload": shape.name, **row}))
    if args.aggregation:
        print(json.dumps({"workload": shape.name,
                          **aggregation_comparison(inp, shape.token_budget, args.seed)}))


if __name__ == "__main__":
    main()
