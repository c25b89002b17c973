"""bench.py's host-side bookkeeping on the CPU: the algorithmic byte model behind the roofline
figures (checked against byte counts worked out by hand for the named workloads), workload
resolution, and the conditions under which a stored DRAM traffic record is reported."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_bytes_qwen3_0_6b_step():
    _, sh = bench.resolve_workload("qwen3-0.6b")
    lens = [16384] * 64
    total, attn, summ = bench.algorithmic_bytes(sh, lens, "block")
    # 64 rows x 8 kv-heads x 512 blocks x 128 dims x 4 bytes of fp32 summaries
    assert summ == 134_217_728
    # K and V of 32 blocks x 32 tokens x 128 dims x 2 bytes, per (row, kv-head); q bf16 + out fp32
    assert attn == 64 * 8 * (32 * 32 * 128 * 2 * 2) + 64 * 16 * 128 * (2 + 4) == 269_221_888
    assert total == 403_439_616
    total16, attn16, summ16 = bench.algorithmic_bytes(sh, lens, "block", summary_bytes=2)
    assert summ16 == 67_108_864 and attn16 == attn and total16 == total - 67_108_864
    # fp8: one byte per value plus a 4-byte scale per block
    _, _, summ8 = bench.algorithmic_bytes(sh, lens, "block", summary_bytes=1, summary_extra=4)
    assert summ8 == 64 * 8 * 512 * (128 + 4)


def test_bytes_short_rows_and_dense():
    _, sh = bench.resolve_workload("qwen3-8b")  # bs 16, k 128, Hkv 8, Hq 32, D 128
    # a row of 1000 tokens has 63 blocks <= k: no scoring, all 1000 tokens read
    total, attn, summ = bench.algorithmic_bytes(sh, [1000], "block")
    assert summ == 0
    assert attn == 8 * 1000 * 128 * 4 + 32 * 128 * 6
    # a row of 20000 tokens: 1250 blocks scored, 128 x 16 tokens read
    total, attn, summ = bench.algorithmic_bytes(sh, [20000], "block")
    assert summ == 8 * 1250 * 128 * 4
    assert attn == 8 * 2048 * 128 * 4 + 32 * 128 * 6
    _, dsh = bench.resolve_workload("dense-L32768")
    total, attn, summ = bench.algorithmic_bytes(dsh, [32768, 100], "dense")
    assert summ == 0 and total == attn
    assert attn == 8 * (32768 + 100) * 128 * 4 + 2 * 32 * 128 * 6


def test_workload_names_and_batch_override():
    kind, sh = bench.resolve_workload("sweep-L32768-B1024")
    assert kind == "block" and sh.capacity == 32768 and sh.k_blocks * sh.block_size == 1024
    kind, sh = bench.resolve_workload("qwen3-0.6b", 32)
    assert kind == "block" and sh.batch == 32
    assert bench.resolve_workload("lessismore")[0] == "unified"
    with pytest.raises(SystemExit):
        bench.resolve_workload("no-such-workload")


def test_stored_traffic_needs_same_batch_and_sources(tmp_path, monkeypatch):
    a, b = tmp_path / "kernel.cuh", tmp_path / "launch.cu"
    a.write_bytes(b"// body v1\n")
    b.write_bytes(b"// launch v1\n")
    (tmp_path / "profiles").mkdir()
    digest = hashlib.sha256(b"// body v1\n// launch v1\n").hexdigest()[:16]
    rec = {"k": {"w": {"sources": ["kernel.cuh", "launch.cu"], "batch": 64,
                       "dram_bytes_per_launch": 123.0, "sources_sha256_16": digest}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.stored_traffic("k", "w", 64) == 123.0
    assert bench.stored_traffic("k", "w", 32) is None      # another batch
    assert bench.stored_traffic("k", "other", 64) is None  # no record
    b.write_bytes(b"// launch v2\n")
    assert bench.stored_traffic("k", "w", 64) is None      # the launcher changed since
    b.write_bytes(b"// launch v1\n")
    assert bench.stored_traffic("k", "w", 64) == 123.0
    a.write_bytes(b"// body v2\n")
    assert bench.stored_traffic("k", "w", 64) is None      # the kernel body changed since


def test_committed_traffic_record():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        ent = json.load(f)["sparse_decode_attn"]["qwen3-8b"]
    for p in ent["sources"]:
        assert os.path.exists(os.path.join(ROOT, p))
    assert len(ent["sources_sha256_16"]) == 16 and ent["batch"] == 32
    # one launch's algorithmic bytes at batch 32: 32 * 8 rows of 128 blocks of 16 tokens
    # (K and V, 2 bytes each, D 128), plus q (bf16) and the fp32 output of 32 * 32 heads
    algo = 32 * 8 * 128 * 16 * 128 * 2 * 2 + 32 * 32 * 128 * (2 + 4)
    assert algo == 269_221_888
    # the capture agrees with the algorithmic bytes to within 3%: no wasted re-reads
    assert abs(ent["dram_bytes_per_launch"] / algo - 1) < 0.03


@pytest.mark.parametrize("name", ["tiny", "lessismore"])
def test_oracle_runner_steps_on_the_host(name):
    """The oracle leg (cpu_baseline, --impl reference) runs a step of either workload kind on
    a small host sample."""
    from block_top_sparse_ksa_b200 import synth
    import torch
    kind, shape = bench.resolve_workload(name)
    if kind == "unified":
        shape = synth.dataclasses.replace(shape, num_q_heads=8, num_kv_heads=2, capacity=400,
                                          seq_len=400, per_head_topk=80, token_budget=80,
                                          recent_tokens=20)
    o, step, what = bench.oracle_runner(shape, kind, 1, torch.device("cpu"))
    step(0, [0])
    step(1, [0])
    assert "oracle" in what


def test_prefill_bytes():
    _, sh = bench.resolve_workload("qwen3-0.6b")
    # keys read: 64 rows x 8 kv-heads x 16384 tokens x 128 x 2 bytes; means written: 512 blocks
    assert bench.prefill_bytes(sh, [16384] * 64) == 2_147_483_648 + 134_217_728
    assert bench.prefill_bytes(sh, [16384] * 64, 2) == 2_147_483_648 + 67_108_864
    assert bench.prefill_bytes(sh, [33]) == 8 * 33 * 128 * 2 + 8 * 2 * 128 * 4
