#!/usr/bin/env python
"""Throughput of block top-k sparse decode attention on B200.

One step = one decode step of one attention layer for a whole batch, one
ksa_decode_step call: block-summary maintenance (last block) + block scoring
(one launch), top-k selection (one launch), gathered split-KV attention over
the selected blocks (one launch), all in libksa's CUDA kernels.  Metric:
queries/s, one query = one sequence's decode step for one layer (all query
heads).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ksa|reference]
                  [--workload qwen3-8b|qwen3-0.6b|lessismore|tiny|sweep-L<ctx>-B<budget>|dense-L<ctx>]

The default workload is the Qwen3-8B-shaped layer at 16K-32K context (batch
32, Hq 32, Hkv 8, D 128, lengths uniform in [16384, 32768], block 16, 128
blocks kept).  The same line also carries the Qwen3-0.6B-shaped layer (batch
64, context 16384) and the 32K-context sweep point with a 1024-token budget,
timed the same way (--no-extra skips them).  With N > 1 (torchrun, one rank
per GPU) every rank runs the same per-GPU batch (weak scaling, no collective
on the data path); the step time is the max over ranks.  Rank 0 prints one
JSON line on stdout; diagnostics go to stderr.

Timing: W warm-up steps (and more, untimed, until at least --min-warmup-s of
them have run, so the clocks have settled), then K steps back to back between
two CUDA events on the launching stream, bracketed by barrier + synchronize.
Nothing else is enqueued inside the timed region.  Per-kernel durations come
from a second pass of the same steps with an event around the selection call
and the attention call.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "sparse decode-attn queries/s at 1 B200; achieved HBM GB/s vs ~8 TB/s peak"
UNIT = "queries/s"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args():
    p = argparse.ArgumentParser(description="Decode-step throughput of libksa (or of the fp64 "
                                "oracle with --impl reference); prints one JSON line.")
    p.add_argument("--gpus", type=int, default=1,
                   help="GPUs of the job (launch with torchrun for more than one)")
    p.add_argument("--steps", type=int, default=20000, help="timed steps")
    p.add_argument("--warmup", type=int, default=100, help="untimed steps before them")
    p.add_argument("--impl", choices=["ksa", "reference"], default="ksa",
                   help="ksa: the CUDA library; reference: the oracle on the host cores")
    p.add_argument("--workload", default="qwen3-8b",
                   help="qwen3-8b, qwen3-0.6b, lessismore, tiny, sweep-L<ctx>-B<budget>, "
                        "dense-L<ctx>")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the extra workloads carried in the default line")
    p.add_argument("--min-warmup-s", type=float, default=0.25,
                   help="keep running untimed warm-up steps until this much time has passed")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="wall-clock budget of the oracle CPU baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--batch", type=int, default=0,
                   help="override the per-GPU batch (small profiling cases only)")
    p.add_argument("--summaries", choices=["f32", "bf16", "fp8"], default="f32",
                   help="storage type of the block summaries (block workloads)")
    return p.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; no collective on the data path)


class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend="nccl"):
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            if torch.cuda.is_available():
                self.pg.barrier(device_ids=[self.local])
            else:
                self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return x
        dev = f"cuda:{self.local}" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, x: float) -> float:
        if self.pg is None:
            return x
        dev = f"cuda:{self.local}" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def weak_scaling(dist: Dist, queries_per_rank: int, ms_local: float, steps: int):
    """Whole-job throughput of K timed steps: every rank processed its own
    batch each step; the job took the slowest rank's time.
    Returns (queries/s over all ranks, ms per step)."""
    ms = dist.max(ms_local)
    total = dist.sum(float(queries_per_rank))
    return total / (ms / 1e3 / steps), ms / steps


# ---------------------------------------------------------------------------
# workloads


def resolve_workload(name: str, batch: int = 0):
    kind, shape = _resolve(name)
    if batch > 0:
        from block_top_sparse_ksa_b200 import synth
        shape = synth.dataclasses.replace(shape, batch=batch)
    return kind, shape


def _resolve(name: str):
    from block_top_sparse_ksa_b200 import synth
    if name == "qwen3-0.6b":
        return "block", synth.QWEN3_0_6B
    if name == "qwen3-8b":
        return "block", synth.QWEN3_8B
    if name == "tiny":
        return "block", synth.TINY
    if name == "lessismore":
        return "unified", synth.LESSISMORE
    if name.startswith("sweep-L"):
        ctx, budget = name[len("sweep-L"):].split("-B")
        return "block", synth.sweep_shape(int(ctx), int(budget))
    if name.startswith("dense-L"):
        return "dense", synth.sweep_shape(int(name[len("dense-L"):]), 256)
    raise SystemExit(f"unknown workload {name}")


def make_block_inputs(shape, device):
    from block_top_sparse_ksa_b200 import synth
    if shape.name == synth.QWEN3_0_6B.name:
        return synth.qwen3_0_6b_inputs(device=device, shape=shape)
    if shape.name == synth.QWEN3_8B.name:
        return synth.qwen3_8b_inputs(device=device, shape=shape)
    if shape.name == synth.TINY.name:
        return synth.tiny_inputs(device=device)
    return synth.sweep_inputs(shape, device=device)


def query_sets(shape, count, device):
    from block_top_sparse_ksa_b200 import synth
    noise = 0.1 if shape.name.startswith("qwen3-0.6b") else None
    return synth.make_queries(shape, 5000, count, device, group_noise=noise)


def algorithmic_bytes(shape, seq_lens, kind: str, summary_bytes: int = 4,
                      summary_extra: int = 0):
    """Per step: summaries read (when k < NB_b) + selected K/V + q + out (fp32).
    Also returns the attention kernel's share (selected K/V + q + out).
    summary_bytes: bytes per summary value (4 fp32, 2 bf16, 1 fp8); summary_extra: bytes
    per block besides the values (4: the fp8 scale)."""
    bs, Hkv, Hq, D = shape.block_size, shape.num_kv_heads, shape.num_q_heads, shape.head_dim
    k = shape.k_blocks
    summ = kv = 0
    for L in seq_lens:
        nb = -(-int(L) // bs)
        if kind == "dense":
            kv += Hkv * int(L) * D * 2 * 2
            continue
        if k < nb:
            summ += Hkv * nb * (D * summary_bytes + summary_extra)
        kv += Hkv * min(k * bs, int(L)) * D * 2 * 2
    qo = len(seq_lens) * Hq * D * (2 + 4)
    return summ + kv + qo, kv + qo, summ


# ---------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    """nvidia-smi samples every 200 ms while it runs.  mark() notes the host time at the start
    and end of the timed region; the summary keeps the samples from the warm-up before the
    first mark (clocks under the same load) to the last mark, or all samples if that window
    caught none."""
    FIELDS = ("timestamp,index,uuid,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        self.marks = []
        try:
            self.uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.t_start = time.time()
        except Exception:
            self.proc = None

    def mark(self):
        self.marks.append(time.time())

    @staticmethod
    def _when(stamp: str):
        import datetime
        try:
            return datetime.datetime.strptime(stamp, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)  # one more sample after the last mark
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 11:
                continue
            if self.uuid and self.uuid not in parts[2] and parts[2] not in self.uuid:
                continue
            rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        window = "whole run"
        if len(self.marks) >= 2:
            lo, hi = self.marks[0] - 0.25, self.marks[-1] + 0.25
            inside = [r for r in rows if (self._when(r[0]) or 0.0) >= lo
                      and (self._when(r[0]) or 0.0) <= hi]
            if inside:
                rows, window = inside, "last warm-up samples + timed region"
        sm = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        mx = [float(r[4]) for r in rows if r[4].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[7 + i]
                          and "Not" not in r[7 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "window": window}


# ---------------------------------------------------------------------------
# timed runs


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def sources_digest(paths) -> str:
    """First 16 hex digits of the SHA-256 of the files' bytes, concatenated in order."""
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str, batch: int):
    """DRAM bytes per launch from a committed ncu capture, if it stands for this batch and the
    kernel's sources are unchanged since (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
        ent = rec[kernel][workload]
        if int(ent["batch"]) != batch:
            return None
        if sources_digest(ent["sources"]) != ent["sources_sha256_16"]:
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


def warm_up(step, warmup: int, min_s: float) -> int:
    """W untimed steps, then more until min_s seconds have passed (SM clocks settle under
    load); returns the number of warm-up steps run."""
    n = 0
    t0 = time.perf_counter()
    while n < warmup or time.perf_counter() - t0 < min_s:
        step(n)
        n += 1
        if n % 64 == 0:
            torch.cuda.synchronize()  # keep the host from running far ahead of the device
    return n


def timed_steps(step, steps: int, dist, stream, side=(), join=None):
    """K steps back to back between two events on `stream`, bracketed by barrier +
    synchronize.  Streams in `side` start after the start event; `join()` (if given) makes
    `stream` wait for their last work before the end event.  Returns (device ms over all K
    steps, host enqueue us per step).  The host figure is the mean over the first 64 steps:
    later ones wait for room in the device's launch queue, so over a long run the host's
    rate only mirrors the device's."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for s in side:
        s.wait_event(start)
    nh = min(steps, 64)
    h0 = time.perf_counter()
    h1 = h0
    for i in range(steps):
        step(i)
        if i == nh - 1:
            h1 = time.perf_counter()
    if join is not None:
        join()
    end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    return start.elapsed_time(end), (h1 - h0) * 1e6 / max(nh, 1)


def kernel_pass(parts, steps: int, stream):
    """Per-launch device time: the step's launches (`parts`, callables taking the step
    index) with an event around each, over `steps` steps.  Returns mean ms per part."""
    evs = []
    for i in range(steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)]
        ev[0].record(stream)
        for j, part in enumerate(parts):
            part(i)
            ev[j + 1].record(stream)
        evs.append(ev)
    torch.cuda.synchronize()
    return [statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in evs)
            for j in range(len(parts))]


class BlockWorkload:
    """Device-resident inputs, prefilled summaries and workspaces of one block workload."""

    def __init__(self, name: str, batch: int, dev, summaries: str):
        import block_top_sparse_ksa_b200 as ksa
        self.ksa = ksa
        self.kind, self.shape = resolve_workload(name, batch)
        sh = self.shape
        torch.manual_seed(0)
        self.inp = make_block_inputs(sh, dev)
        self.nq = 16
        self.qs = query_sets(sh, self.nq, dev)
        sdt = {"bf16": torch.bfloat16, "fp8": "fp8"}.get(summaries, torch.float32)
        B, Hq, Hkv, D, T, bs, k = (sh.batch, sh.num_q_heads, sh.num_kv_heads, sh.head_dim,
                                   sh.capacity, sh.block_size, sh.k_blocks)
        self.S = ksa.ksa_build_block_summaries(self.inp.K, self.inp.seq_lens, bs,
                                               summary_dtype=sdt)  # prefill, untimed
        self.ws_sel = torch.zeros((ksa.ksa_select_blocks_workspace(B, Hq, Hkv, D, T, bs, k),),
                                  dtype=torch.uint8, device=dev)
        self.ws_att = torch.zeros((ksa.ksa_sparse_decode_attn_workspace(B, Hq, Hkv, D, T, k, bs),),
                                  dtype=torch.uint8, device=dev)
        self.ws_step = torch.zeros((ksa.ksa_decode_step_workspace(B, Hq, Hkv, D, T, bs, k),),
                                   dtype=torch.uint8, device=dev)
        self.idx = torch.empty((B, Hkv, k), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((B, Hkv), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream()
        nb_max = -(-T // bs)
        # ksa_decode_step: a scoring launch (when some row can hold more than k blocks), a
        # ranking launch, the attention launch
        self.launches_per_step = 1 if self.kind == "dense" else (2 if nb_max > k else 1) + 1

    def select(self, i, q=None):
        sh = self.shape
        self.ksa.ksa_decode_select_blocks(self.qs[i % self.nq] if q is None else q, self.inp.K,
                                          self.S, self.inp.seq_lens, sh.block_size, sh.k_blocks,
                                          block_idx=self.idx, num_sel=self.cnt,
                                          workspace=self.ws_sel, stream=self.stream)

    def attend(self, i, q=None):
        q = self.qs[i % self.nq] if q is None else q
        if self.kind == "dense":
            self.ksa.ksa_sparse_decode_attn(q, self.inp.K, self.inp.V, self.inp.seq_lens,
                                            out=self.out, workspace=self.ws_att,
                                            stream=self.stream)
        else:
            self.ksa.ksa_sparse_decode_attn(q, self.inp.K, self.inp.V, self.inp.seq_lens,
                                            self.idx, self.cnt,
                                            tokens_per_idx=self.shape.block_size, out=self.out,
                                            workspace=self.ws_att, stream=self.stream)

    def decode_step(self, i, q=None):
        sh = self.shape
        self.ksa.ksa_decode_step(self.qs[i % self.nq] if q is None else q, self.inp.K,
                                 self.inp.V, self.S, self.inp.seq_lens, sh.block_size,
                                 sh.k_blocks, block_idx=self.idx, num_sel=self.cnt, out=self.out,
                                 workspace=self.ws_step, stream=self.stream)

    def step(self, i):
        """The timed step: ksa_decode_step (dense attention for the k = all workloads)."""
        if self.kind == "dense":
            self.attend(i)
        else:
            self.decode_step(i)

    def parts(self):
        """The step's calls, one by one (for per-kernel times)."""
        return [self.attend] if self.kind == "dense" else [self.select, self.attend]


def measure_block(wl: BlockWorkload, args, dist, peak: float, peak_kind: str,
                  clocks: "ClockSampler | None" = None):
    """Warm-up, the timed steps and the per-kernel pass of one block workload."""
    sh, kind = wl.shape, wl.kind
    n_warm = warm_up(wl.step, args.warmup, args.min_warmup_s)
    if clocks is not None:
        clocks.mark()
    ms, host_us = timed_steps(wl.step, args.steps, dist, wl.stream)
    if clocks is not None:
        clocks.mark()
    value, ms_step = weak_scaling(dist, sh.batch, ms, args.steps)
    times = kernel_pass(wl.parts(), max(20, min(args.steps, 200)), wl.stream)
    t_att = times[-1]
    t_sel = times[0] if kind != "dense" else 0.0
    lens = wl.inp.seq_lens.cpu().tolist()
    total_b, attn_b, summ_b = algorithmic_bytes(sh, lens, kind, wl.S.element_size(),
                                                4 if wl.S.dtype == torch.uint8 else 0)
    per_step_s = ms_step / 1e3
    attn_gbs = attn_b / (t_att * 1e-3) / 1e9
    return {
        "value": value, "ms_per_step": ms_step, "warmup_steps_run": n_warm,
        "host_enqueue_us_per_step": host_us,
        "kernels_ms": ({"sparse_decode_attn": t_att} if kind == "dense" else
                       {"decode_select_blocks": t_sel, "sparse_decode_attn": t_att}),
        "kernels_note": "mean of a second pass of the same steps with an event around each call "
                        "(the selection call is its scoring and ranking launches)",
        "roofline": {"bound": "hbm", "achieved": attn_gbs, "peak": peak, "unit": "GB/s",
                     "frac": attn_gbs / peak,
                     "traffic": stored_traffic("sparse_decode_attn", args.workload, sh.batch),
                     "kernel": "sparse_decode_attn", "peak_source": peak_kind,
                     "bytes_per_launch": attn_b},
        "step_hbm": {"bytes_per_step": total_b, "gbs": total_b / per_step_s / 1e9,
                     "frac": total_b / per_step_s / 1e9 / peak,
                     "kernel_sum_ms": t_sel + t_att},
        "select_hbm": (None if kind == "dense" else
                       {"bytes_per_launch": summ_b,
                        "gbs": summ_b / (t_sel * 1e-3) / 1e9 if t_sel > 0 else None}),
        "gpu_launches": wl.launches_per_step * args.steps,
        "config": {"workload": sh.name, "batch_per_gpu": sh.batch, "num_q_heads": sh.num_q_heads,
                   "num_kv_heads": sh.num_kv_heads, "head_dim": sh.head_dim,
                   "capacity": sh.capacity, "block_size": sh.block_size,
                   "seq_lens": ([sh.min_len, sh.max_len] if sh.min_len != sh.max_len
                                else sh.max_len),
                   "k_blocks": sh.k_blocks if kind != "dense" else "all",
                   "summaries": {torch.bfloat16: "bf16", torch.uint8: "fp8 e4m3 + fp32 "
                                 "scale per block"}.get(wl.S.dtype, "f32"),
                   "l2": "inputs larger than L2: K/V cache %.1f GB, %.0f MB read per step, %d "
                         "rotating query sets" % (2 * wl.inp.K.numel() * 2 / 1e9, total_b / 1e6,
                                                  wl.nq),
                   "step": ("dense attention" if kind == "dense" else
                            "ksa_decode_step: last-block summary refresh + scoring + top-k "
                            "(2 launches) + sparse attention (1 launch)")},
    }


def run_block(args, dist, dev, kind):
    wl = BlockWorkload(args.workload, args.batch, dev, args.summaries)
    peak, peak_kind = measured_peak()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    res = measure_block(wl, args, dist, peak, peak_kind, clocks)
    res["clocks"] = clocks.stop()
    if not args.no_e2e:
        res["e2e"] = run_block_e2e(args, dist, wl)
    if kind != "dense":
        try:
            res["prefill"] = time_prefill(wl.ksa, wl.inp, wl.shape, wl.S, wl.stream, peak)
        except Exception as e:  # a side figure: never lose the step's line for it
            res["prefill"] = {"error": str(e)[:200]}
    return res


EXTRA_WORKLOADS = ("qwen3-0.6b", "sweep-L32768-B1024")


def run_extra(args, dist, dev):
    """The other block workloads the line carries, each timed like the main one."""
    peak, peak_kind = measured_peak()
    out = {}
    for name in EXTRA_WORKLOADS:
        if name == args.workload:
            continue
        try:
            wl = BlockWorkload(name, 0, dev, args.summaries)
            r = measure_block(wl, args, dist, peak, peak_kind)
            out[name] = {"workload": wl.shape.name, "value": r["value"], "unit": UNIT,
                         "ms_per_step": r["ms_per_step"],
                         "host_enqueue_us_per_step": r["host_enqueue_us_per_step"],
                         "step_hbm": r["step_hbm"], "roofline_frac": r["roofline"]["frac"],
                         "kernels_ms": r["kernels_ms"], "gpu_launches": r["gpu_launches"]}
            del wl
        except torch.cuda.OutOfMemoryError as e:  # never lose the main line for a side figure
            out[name] = {"error": str(e)[:200]}
        torch.cuda.empty_cache()
    return out


def prefill_bytes(shape, seq_lens, summary_bytes: int = 4, summary_extra: int = 0) -> int:
    """The prefill's summary build (every block of every row): one read of the keys and one
    write of the block means (summary_extra: bytes per block besides the values)."""
    bs, Hkv, D = shape.block_size, shape.num_kv_heads, shape.head_dim
    return sum(Hkv * int(L) * D * 2 +
               Hkv * (-(-int(L) // bs)) * (D * summary_bytes + summary_extra)
               for L in seq_lens)


def time_prefill(ksa, inp, shape, S, stream, peak, reps: int = 5):
    """ksa_build_block_summaries (mode ALL) over the whole cache, timed alone with CUDA events
    (the cache is larger than L2, so the repetitions read from HBM)."""
    fp8 = S.dtype == torch.uint8
    S2 = ksa.alloc_summaries(*S.shape, "fp8" if fp8 else S.dtype, S.device)
    ksa.ksa_build_block_summaries(inp.K, inp.seq_lens, shape.block_size, summaries=S2,
                                  stream=stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        ksa.ksa_build_block_summaries(inp.K, inp.seq_lens, shape.block_size, summaries=S2,
                                      stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    b = prefill_bytes(shape, inp.seq_lens.cpu().tolist(), S.element_size(), 4 if fp8 else 0)
    return {"kernel": "block_summaries (mode ALL)", "ms": ms, "bytes": b,
            "gbs": b / (ms * 1e-3) / 1e9, "frac": b / (ms * 1e-3) / 1e9 / peak}


def run_block_e2e(args, dist, wl: BlockWorkload):
    """The same step through the public API with host buffers.  Per step: the new query and
    the new token's K/V rows go host->device from pinned memory, ksa_append_kv writes the
    rows into their cache slot (token L_b - 1: the lengths stay fixed, so every step is the
    same workload), then ksa_decode_step, and the output comes back device->host.  Every
    step's copies are inside the timed region.  Two forms: serial (every copy on the compute
    stream, in step order), and pipelined (as a serving loop runs it: the uploads on one copy
    stream and the downloads on another, with double buffers and events, so a step's copies
    overlap the neighbouring steps' kernels; the value reported)."""
    import block_top_sparse_ksa_b200 as ksa
    sh = wl.shape
    B, Hq, Hkv, D = sh.batch, sh.num_q_heads, sh.num_kv_heads, sh.head_dim
    dev = wl.qs.device
    nq = wl.nq
    h_q = wl.qs.cpu().pin_memory()
    h_kv = torch.randn((nq, 2, B, Hkv, D), dtype=torch.float32).to(torch.bfloat16).pin_memory()
    h_out = [torch.empty((B, Hq, D), dtype=torch.float32).pin_memory() for _ in range(2)]
    d_q = [torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    d_kv = [torch.empty((2, B, Hkv, D), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    d_out = [torch.empty((B, Hq, D), dtype=torch.float32, device=dev) for _ in range(2)]
    stream = wl.stream
    lens = wl.inp.seq_lens

    def compute(i, q, kv, out):
        ksa.ksa_append_kv(kv[0], kv[1], wl.inp.K, wl.inp.V, lens, stream=stream)
        if wl.kind == "dense":
            ksa.ksa_sparse_decode_attn(q, wl.inp.K, wl.inp.V, lens, out=out,
                                       workspace=wl.ws_att, stream=stream)
        else:
            ksa.ksa_decode_step(q, wl.inp.K, wl.inp.V, wl.S, lens, sh.block_size, sh.k_blocks,
                                block_idx=wl.idx, num_sel=wl.cnt, out=out,
                                workspace=wl.ws_step, stream=stream)

    def serial_step(i):
        d_q[0].copy_(h_q[i % nq], non_blocking=True)
        d_kv[0].copy_(h_kv[i % nq], non_blocking=True)
        compute(i, d_q[0], d_kv[0], d_out[0])
        h_out[0].copy_(d_out[0], non_blocking=True)

    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]  # whether buffer set s has been through a step yet
    last = [None]

    def piped_step(i):
        s = i & 1
        with torch.cuda.stream(up):
            if used[s]:
                up.wait_event(ev_comp[s])  # step i - 2 has read d_q[s], d_kv[s]
            d_q[s].copy_(h_q[i % nq], non_blocking=True)
            d_kv[s].copy_(h_kv[i % nq], non_blocking=True)
            ev_up[s].record(up)
        stream.wait_event(ev_up[s])
        if used[s]:
            stream.wait_event(ev_down[s])  # step i - 2's output has left d_out[s]
        compute(i, d_q[s], d_kv[s], d_out[s])
        ev_comp[s].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev_comp[s])
            h_out[s].copy_(d_out[s], non_blocking=True)
            ev_down[s].record(down)
        used[s] = True
        last[0] = s

    def join():
        stream.wait_event(ev_down[last[0]])

    warm_up(serial_step, args.warmup, 0.0)
    ms_ser, host_ser = timed_steps(serial_step, args.steps, dist, stream)
    value_ser, ms_step_ser = weak_scaling(dist, B, ms_ser, args.steps)
    warm_up(piped_step, args.warmup, 0.0)
    ms, host_us = timed_steps(piped_step, args.steps, dist, stream, side=(up, down), join=join)
    value, ms_step = weak_scaling(dist, B, ms, args.steps)
    torch.cuda.synchronize()
    ref = d_out[last[0]].cpu()
    assert torch.equal(h_out[last[0]], ref), "the last step's download differs from its output"
    h2d = (B * Hq * D + 2 * B * Hkv * D) * 2
    d2h = B * Hq * D * 4
    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms_step,
            "host_enqueue_us_per_step": host_us,
            "gpu_launches": (wl.launches_per_step + 1) * args.steps,  # + the append
            "serial": {"value": value_ser, "ms_per_step": ms_step_ser,
                       "host_enqueue_us_per_step": host_ser},
            "note": "per step: q and the new token's K/V rows host->device (pinned), "
                    "ksa_append_kv, ksa_decode_step, out device->host; value: uploads and "
                    "downloads on two copy streams with double buffers, overlapping the "
                    "neighbouring steps' kernels; serial: every copy on the compute stream"}


def run_unified(args, dist, dev):
    import block_top_sparse_ksa_b200 as ksa
    from block_top_sparse_ksa_b200 import synth
    _, sh = resolve_workload(args.workload, args.batch)
    inp = synth.lessismore_inputs(device=dev, shape=sh)
    B, Hq, Hkv, D, T = sh.batch, sh.num_q_heads, sh.num_kv_heads, sh.head_dim, sh.capacity
    ws = torch.empty((ksa.ksa_unified_select_workspace(B, Hq, Hkv, D, T, sh.per_head_topk,
                                                       sh.token_budget),),
                     dtype=torch.uint8, device=dev)
    tok = torch.empty((B, sh.token_budget), dtype=torch.int32, device=dev)
    cnt = torch.empty((B,), dtype=torch.int32, device=dev)
    outs = [torch.empty((B, Hq, D), dtype=torch.float32, device=dev) for _ in inp.layers]
    ws_att = torch.zeros((ksa.ksa_sparse_decode_attn_workspace(B, Hq, Hkv, D, T,
                                                               sh.token_budget, 1),),
                         dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def select(i):
        ksa.ksa_unified_select(inp.q_sel, inp.K_sel, inp.seq_lens, sh.per_head_topk,
                               sh.token_budget, sh.recent_tokens, tok, cnt, ws, stream=stream)

    def attend(i):
        for li, (q, K, V) in enumerate(inp.layers):
            ksa.ksa_sparse_decode_attn(q, K, V, inp.seq_lens, tok, cnt, tokens_per_idx=1,
                                       idx_shared=True, out=outs[li], workspace=ws_att,
                                       stream=stream)

    def step(i):
        select(i)
        attend(i)

    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    n_warm = warm_up(step, args.warmup, args.min_warmup_s)
    clocks.mark()
    ms, host_us = timed_steps(step, args.steps, dist, stream)
    clocks.mark()
    clk = clocks.stop()
    value, ms_step = weak_scaling(dist, B, ms, args.steps)
    t_sel, t_att3 = kernel_pass([select, attend], max(20, min(args.steps, 200)), stream)
    t_att = t_att3 / len(inp.layers)
    per = ms_step / 1e3
    sel_b = B * Hkv * sh.seq_len * D * 2 + B * Hq * D * 2
    att_b = B * Hkv * sh.token_budget * D * 2 * 2 + B * Hq * D * 6
    peak, peak_kind = measured_peak()
    return {
        "ms_per_step": ms_step, "value": value, "warmup_steps_run": n_warm,
        "host_enqueue_us_per_step": host_us,
        "kernels_ms": {"unified_select": t_sel, "sparse_decode_attn_per_layer": t_att},
        "kernels_note": "mean of a second pass of the same steps with an event around the "
                        "selection call and around the three attention calls",
        "roofline": {"bound": "hbm", "achieved": att_b / (t_att * 1e-3) / 1e9, "peak": peak,
                     "unit": "GB/s", "frac": att_b / (t_att * 1e-3) / 1e9 / peak,
                     "traffic": stored_traffic("sparse_decode_attn", args.workload, sh.batch),
                     "kernel": "sparse_decode_attn (token list)", "peak_source": peak_kind,
                     "bytes_per_launch": att_b},
        "select_hbm": {"bytes_per_launch": sel_b, "gbs": sel_b / (t_sel * 1e-3) / 1e9},
        "step_hbm": {"bytes_per_step": sel_b + 3 * att_b,
                     "gbs": (sel_b + 3 * att_b) / per / 1e9,
                     "frac": (sel_b + 3 * att_b) / per / 1e9 / peak,
                     "kernel_sum_ms": t_sel + t_att3},
        # selection: scores, picks, (vote counting when the picks keep the row's keys in
        # registers: capacity <= 24576), shared set; then one attention launch per layer
        # selection: scores, per-head picks, then the shared set straight from the pick bit
        # sets (register picks, < 64 heads), or votes + set; rows over 24576 tokens: scores,
        # picks with votes, set
        "gpu_launches": ((3 if T > 24576 or (Hq < 64 and -(-T // 32) <= 1024) else 4)
                         + len(inp.layers)) * args.steps, "clocks": clk,
        "config": {"workload": sh.name, "batch_per_gpu": B, "num_q_heads": Hq,
                   "num_kv_heads": Hkv, "head_dim": D, "context": sh.seq_len,
                   "per_head_topk": sh.per_head_topk, "token_budget": sh.token_budget,
                   "recent_tokens": sh.recent_tokens, "sparse_layers": sh.sparse_layers,
                   "l2": "inputs larger than L2 (4 x 1.3 GB K/V per layer)",
                   "step": "unified_select + 3 x sparse_decode_attn (one query = one sequence's "
                           "selection layer + 3 sparse layers)"},
    }


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)


def oracle_block_sample(shape, kind, n_rows, device):
    """Host copies of n_rows rows of the workload, summaries by the oracle (untimed prefill)."""
    from block_top_sparse_ksa_b200 import synth
    from oracle import oracle as O
    small = synth.dataclasses.replace(shape, batch=n_rows)
    inp = make_block_inputs(small, device)
    qs = query_sets(small, 4, device)
    o = O.get()
    lens = inp.seq_lens.cpu().numpy()
    K, V = synth.bits(inp.K), synth.bits(inp.V)
    qb = [synth.bits(qs[i]) for i in range(qs.shape[0])]
    S = None if kind == "dense" else o.block_summaries(K, lens, shape.block_size)
    return o, qb, K, V, S, lens


def oracle_step_units(o, shape, kind, q, K, V, S, lens, rows):
    """One oracle decode step over the given rows: scores, top-k, attention."""
    bs, k = shape.block_size, shape.k_blocks
    sel = np.asarray(rows)
    qv, Kv, Vv, Lv = q[sel], K[sel], V[sel], lens[sel]
    if kind == "dense":
        o.attention(qv, Kv, Vv, Lv)
        return
    s = o.block_scores(qv, S[sel], Lv, bs)
    n, hkv = s.shape[0], s.shape[1]
    idx = np.full((n, hkv, k), -1, np.int32)
    cnt = np.zeros((n, hkv), np.int32)
    for b in range(n):
        nb = -(-int(Lv[b]) // bs)
        for g in range(hkv):
            got = o.topk(s[b, g, :nb], k)
            idx[b, g, :len(got)] = got
            cnt[b, g] = len(got)
    o.attention(qv, Kv, Vv, Lv, idx, cnt, bs)


def oracle_runner(shape, kind, n_rows, device):
    """(oracle, step(i, rows), what a step computes) on a host sample of n_rows rows of the
    workload.  A LessIsMore step is the unified selection followed by attention over the
    shared set in each sparse layer, as on the GPU."""
    if kind != "unified":
        o, qb, K, V, S, lens = oracle_block_sample(shape, kind, n_rows, device)

        def step(i, rows):
            oracle_step_units(o, shape, kind, qb[i % len(qb)], K, V, S, lens, rows)
        return o, step, ("oracle block scores + top-k + attention (summaries precomputed, as "
                         "the GPU prefill)")
    from block_top_sparse_ksa_b200 import synth
    from oracle import oracle as O
    inp = synth.lessismore_inputs(device=device, shape=synth.dataclasses.replace(shape,
                                                                                 batch=n_rows))
    o = O.get()
    lens = inp.seq_lens.cpu().numpy()
    q_sel, K_sel = synth.bits(inp.q_sel), synth.bits(inp.K_sel)
    layers = [tuple(synth.bits(t) for t in layer) for layer in inp.layers]

    def step(i, rows):
        sel = np.asarray(rows)
        tok, cnt = o.unified_select(q_sel[sel], K_sel[sel], lens[sel], shape.per_head_topk,
                                    shape.token_budget, shape.recent_tokens)
        for q, K, V in layers:
            o.attention(q[sel], K[sel], V[sel], lens[sel], tok, cnt, 1, True)
    return o, step, (f"oracle unified selection + attention over the shared set in "
                     f"{len(layers)} sparse layers")


def cpu_baseline(args, dev, kind, budget_s):
    _, shape = resolve_workload(args.workload, args.batch)
    n_rows = 1 if kind == "unified" else min(8, shape.batch)
    o, step, what = oracle_runner(shape, kind, n_rows, dev)
    o.set_threads(os.cpu_count() or 1)
    rows_done = 0
    t0 = time.perf_counter()
    i = 0
    while True:
        step(i, list(range(n_rows)))
        rows_done += n_rows
        i += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": rows_done / el, "unit": UNIT, "cores": o.max_threads(), "kind": "oracle",
            "sample": f"{n_rows} rows of {shape.name}, {i} steps of {what}, {el:.1f} s"}


def run_reference(args, dist):
    """The oracle as the reference arm: same workload/metric, host cores."""
    if dist.rank != 0:
        return
    kind, shape = resolve_workload(args.workload, args.batch)
    dev = torch.device("cuda", dist.local) if torch.cuda.is_available() else torch.device("cpu")
    n_rows = min(8, shape.batch)
    o, step, what = oracle_runner(shape, kind, n_rows, dev)
    o.set_threads(os.cpu_count() or 1)
    # size one step so that warmup + steps take about two minutes
    t0 = time.perf_counter()
    step(0, [0])
    t_row = max(time.perf_counter() - t0, 1e-4)
    per_step = min(n_rows, max(1, int(120.0 / (args.steps + args.warmup) / t_row)))
    rows = list(range(per_step))
    for i in range(args.warmup):
        step(i, rows)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i, rows)
    el = time.perf_counter() - t0
    value = per_step * args.steps / el
    sample = f"{per_step} of {shape.batch} rows of {shape.name} per step ({what}, fp64)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": shape.name, "batch_per_gpu": shape.batch,
                   "sample_rows_per_step": per_step},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": o.max_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse_args()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)  # rank 0 only; no process group is needed
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    dist.init("nccl")
    import block_top_sparse_ksa_b200 as ksa
    ksa.lib()  # fails loudly if libksa.so is missing
    kind, _ = resolve_workload(args.workload)
    try:
        if kind == "unified":
            res = run_unified(args, dist, dev)
        else:
            res = run_block(args, dist, dev, kind)
        line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": dist.world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic (seeded; no dataset or weights)",
                "config": dict(res["config"], parallelism=f"dp{dist.world} (batch-sharded "
                               "replicas, no data-path collective)"),
                "roofline": res["roofline"], "kernels_ms": res["kernels_ms"],
                "step_hbm": res["step_hbm"],
                "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
                "warmup_steps_run": res["warmup_steps_run"],
                "host_enqueue_us_per_step": res["host_enqueue_us_per_step"],
                "kernels_note": res["kernels_note"]}
        if res.get("select_hbm") is not None:
            line["select_hbm"] = res["select_hbm"]
        if "e2e" in res:
            line["e2e"] = res["e2e"]
        if "prefill" in res:
            line["prefill"] = res["prefill"]
        if kind != "unified" and not args.no_extra and args.batch == 0:
            line["extra_workloads"] = run_extra(args, dist, dev)
        if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args, dev, kind, args.cpu_seconds)
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
