"""The bench's algorithmic work counts (the roofline numerators), checked against
closed forms; host logic only."""
from __future__ import annotations

import dataclasses
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def test_full_prefill_counts_match_the_closed_forms():
    w = dataclasses.replace(synth.WORKLOADS["prefill_n1m_decode64"], n=4096, decode_steps=0)
    a = bench.algorithmic(w)
    nb = w.n // w.r
    # sum_i floor(i / r) over [0, n) = r * nb * (nb - 1) / 2 = 2 nb (nb - 1) at r = 4
    assert a["index_flops"] == 2 * nb * (nb - 1) * w.idx_heads * w.idx_dim * 2
    assert a["prefill_tokens"] == w.n
    # every query attends r * min(k_B, i // r) + i % r + 1 tokens
    tokens = sum(w.r * min(w.k_blocks, i // w.r) + i % w.r + 1 for i in range(w.n))
    assert a["attn_gather_bytes"] == tokens * w.kv_heads * w.head_dim * 4
    assert a["compress_bytes"] == nb * w.r * w.idx_dim * 2 + nb * w.idx_dim * 2


def test_chunked_prefill_counts_only_the_chunk():
    full = dataclasses.replace(synth.WORKLOADS["prefill_n1m_decode64"], n=8192, decode_steps=0)
    chunk = dataclasses.replace(full, q_begin=8192 - 1024)
    head = dataclasses.replace(full, n=8192 - 1024)
    a, b, c = bench.algorithmic(full), bench.algorithmic(chunk), bench.algorithmic(head)
    # The chunk's work is the full prefill's minus the prefix's (queries are independent).
    for k in ("index_flops", "attn_gather_bytes", "attn_flops", "prefill_tokens", "compress_bytes"):
        assert b[k] == a[k] - c[k], k
    assert b["prefill_tokens"] == 1024
    assert synth.WORKLOADS["prefill_chunk8k_n1m"].n - synth.WORKLOADS["prefill_chunk8k_n1m"].q_begin == 8192


def test_fp8_caches_count_code_rows_and_scales():
    w = dataclasses.replace(synth.WORKLOADS["prefill_n1m_decode64"], n=4096, decode_steps=0)
    a, b = bench.algorithmic(w), bench.algorithmic(w, "fp8")
    rows = a["attn_gather_bytes"] // (w.head_dim * 2)  # gathered (token, kv head, K or V) rows
    assert b["attn_gather_bytes"] == rows * (w.head_dim + 4)
    assert b["quantize_bytes"] == w.n * w.kv_heads * 2 * (w.head_dim * 3 + 4) and a["quantize_bytes"] == 0
    assert b["index_flops"] == a["index_flops"] and b["attn_flops"] == a["attn_flops"]


def test_training_counts_match_the_closed_forms():
    w = dataclasses.replace(synth.WORKLOADS["train_n32k"], n=2048)
    a = bench.algorithmic(w)
    n, r, d, H, hk = w.n, w.r, w.head_dim, w.q_heads, w.kv_heads
    tokens = sum(r * min(w.k_blocks, i // r) + i % r + 1 for i in range(n))
    # the five products of the gradient over the forward's token sets
    assert a["bwd_flops"] == 5 * tokens * H * d * 2
    # the forward's gather, an fp32 dK and dV row per gathered (token, kv head), q / dout / out read, dq written
    assert a["bwd_bytes"] == tokens * hk * (d * 4 + d * 8) + n * H * d * (6 + 4)
    # the target: logits over tokens <= i (log-sum-exp), then over the visible blocks' tokens
    assert a["target_flops"] == sum(i + 1 + r * (i // r) for i in range(n)) * H * d * 2
    ld = (n - 1) // r
    assert a["scores_bytes"] == n * (ld * 4 + w.idx_heads * w.idx_dim * 2)
    assert a["kl_bytes"] == sum(i // r for i in range(n)) * 8 + n * ld * 4 + n * 4
    # a workload without training counts none of it
    b = bench.algorithmic(dataclasses.replace(w, train=False))
    assert b["bwd_bytes"] == b["bwd_flops"] == b["target_flops"] == b["scores_bytes"] == b["kl_bytes"] == 0


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host) prints one JSON line
    with the contract's keys, the reference marker, a cpu_baseline that
    describes the run and an e2e object with zero copied bytes."""
    import json
    import subprocess

    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_prefill_n256", "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, check=True).stdout.strip().splitlines()
    d = json.loads(out[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config"):
        assert k in d, k
    assert d["impl"] == "reference" and d["config"]["workload"] == "tiny_prefill_n256"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["cpu_baseline"]["value"] == d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_host_prefill_chunk_plan():
    """QSALayer.chunk_plan (prefill_from_host): chunks sum to nq, none above the
    chunk size, ramping up and back down at the ends (host logic only)."""
    from block_sparse_long_02_b200.layer import QSALayer

    for nq, chunk, first in [(1 << 20, 131072, 8192), (6007, 2048, 512), (6007, 2048, 2048), (100, 100, 100),
                             (7, 4, 4), (131072, 131072, 8192), (1 << 20, 131072, 131072)]:
        plan = QSALayer.chunk_plan(nq, chunk, first)
        assert sum(plan) == nq and all(0 < m <= chunk for m in plan), (nq, chunk, first, plan)
        k = 0
        while k + 1 < len(plan) and plan[k] < chunk and plan[k + 1] == 2 * plan[k]:
            k += 1
        assert plan[:k] == plan[::-1][:k]  # the ramp down mirrors the ramp up
    assert QSALayer.chunk_plan(1 << 20, 131072, 8192)[:5] == [8192, 16384, 32768, 65536, 131072]
    assert QSALayer.chunk_plan(1 << 20, 131072, 8192)[-4:] == [65536, 32768, 16384, 8192]


def test_traffic_figures_follow_the_kernel_sources():
    """roofline.traffic comes from profiles/dram_traffic.txt only while the
    stage's kernel sources hash to what the figure was measured on."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        workload, stage, nbytes, sha = line.split()
        want = float(nbytes) if sha == bench.stage_source_sha1(stage) else None
        assert bench.traffic_for(workload, stage) == want, line
    assert bench.traffic_for("decode_b8_n256k", "attention") is None  # never measured
