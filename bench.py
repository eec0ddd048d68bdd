#!/usr/bin/env python
"""QSA layer benchmark: prefill + decode tokens/s at 1M context on B200.

One step = one pass of the whole hot path over the workload
"prefill_n1m_decode64": key pooling, fused indexer score + top-k_B selection
and sparse attention for all 1,048,576 prefill positions of one sequence, then
64 decode steps (append, score, select, attend, pool). Inputs are synthetic
(seeded), resident in HBM before timing; they are far larger than L2 (q 8.6 GB,
K/V 2.1 GB), and decode steps run back to back as in real decoding.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]

Prints one JSON line (rank 0). With N > 1 (torchrun), every rank runs an
independent replica (the layer has no cross-GPU exchange); time is the max
over ranks and value counts the tokens of all ranks. On one GPU the default run
also measures the metric's other workloads (32K and 8 x 256K decode, 128K
prefill) and reports them under "configs", each with its stage rooflines and
the oracle timed beside it (--no-configs skips them).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "QSA layer prefill & decode tokens/s at 256K/1M ctx; % of HBM/tensor roofline"
DEFAULT_WORKLOAD = "prefill_n1m_decode64"


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def algorithmic(w, kv="bf16"):
    """Per-step algorithmic work (the units the roofline divides by). kv="fp8":
    the prefill attention gathers 128-byte E4M3 code rows plus a 4-byte scale
    per row, and the step quantizes the prefill's K/V rows (2 bytes read, 1
    written per value, 4 bytes per row scale)."""
    r, kB, n, q0 = w.r, w.k_blocks, w.n, w.q_begin
    i = np.arange(q0, n, dtype=np.int64)
    vis = i // r
    pairs = int(vis.sum()) if w.prefill else 0
    tok = (r * np.minimum(kB, vis) + i % r + 1) if w.prefill else np.zeros(0, np.int64)
    sum_t = int(tok.sum())
    d = w.head_dim
    nb = n // r - q0 // r  # blocks pooled by the prefill
    out = {
        "compress_bytes": (nb * r * w.idx_dim * 2 + nb * w.idx_dim * 2) if w.prefill else 0,
        "index_flops": pairs * w.idx_heads * w.idx_dim * 2,
        "attn_gather_bytes": sum_t * w.kv_heads * (d * 2 * 2 if kv == "bf16" else (d + 4) * 2),
        "quantize_bytes": (((n - q0) * w.kv_heads * 2 * (d * 3 + 4))
                           + ((n // r - q0 // r) * (w.idx_dim * 3 + 4) if w.decode_steps else 0))
                          if (w.prefill and kv == "fp8") else 0,
        "attn_flops": sum_t * w.q_heads * d * 4,
        "prefill_tokens": (n - q0) if w.prefill else 0,
    }
    dec = 0
    dec_tok = 0
    for s in range(w.decode_steps):
        p = w.n + s
        nb = p // r
        t = r * min(kB, nb) + p % r + 1
        if kv == "fp8":  # code rows plus 4-byte scales
            dec += nb * (w.idx_dim + 4) + t * w.kv_heads * (d + 4) * 2
        else:
            dec += nb * w.idx_dim * 2 + t * w.kv_heads * d * 2 * 2
        dec_tok += 1
    out["decode_bytes"] = dec * w.batch
    out["decode_gather_bytes"] = sum(
        (r * min(kB, (w.n + s) // r) + (w.n + s) % r + 1) * w.kv_heads * d * 2 * 2 for s in range(w.decode_steps)
    ) * w.batch
    out["decode_tokens"] = dec_tok * w.batch
    out["prefill_tokens"] *= w.batch
    # Training kernels (zero unless the workload trains).
    nq = n - q0
    ld = (n - 1) // r
    train = bool(getattr(w, "train", False)) and w.prefill
    # backward: the forward's gather again, every (token, kv head) row's dK and
    # dV added once per query that holds it (fp32), q / dout / out read, dq written.
    out["bwd_bytes"] = (sum_t * w.kv_heads * (d * 2 * 2 + d * 4 * 2) + nq * w.q_heads * d * (2 * 3 + 4)) if train else 0
    out["bwd_flops"] = sum_t * w.q_heads * d * 2 * 5 if train else 0  # S, dP, dQ, dK, dV products
    # target: every head's logits over tokens <= i (log-sum-exp), then over the
    # visible blocks' tokens (probabilities).
    out["target_flops"] = int((i + 1 + r * vis).sum()) * w.q_heads * d * 2 if train else 0
    out["scores_bytes"] = nq * (ld * 4 + w.idx_heads * w.idx_dim * 2) if train else 0
    out["kl_bytes"] = (pairs * 4 * 2 + nq * ld * 4 + nq * 4) if train else 0  # target + scores read, dscores written
    for k in ("compress_bytes", "index_flops", "attn_gather_bytes", "attn_flops", "quantize_bytes", "bwd_bytes",
              "bwd_flops", "target_flops", "scores_bytes", "kl_bytes"):
        out[k] *= w.batch
    return out


class ClockSampler:
    """nvidia-smi samples during the timed region (clocks and throttle reasons)."""

    Q = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id=None):
        self.bus_id = bus_id if isinstance(bus_id, int) else None  # PCI bus number of our GPU
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except FileNotFoundError:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        try:
            return self._stop()
        except Exception as e:  # the sampler must never abort a measurement
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"sampler error: {e}"]}

    def _stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) >= 10:
                rows.append(f)

        def bus(f):
            try:
                return int(f[1].split(":")[1], 16)
            except (IndexError, ValueError):
                return None

        mine = [f for f in rows if self.bus_id is not None and bus(f) == self.bus_id]
        if mine:
            rows = mine
        elif len({f[0] for f in rows}) > 1:
            rows = [f for f in rows if f[0] == rows[0][0]]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(f[2]) for f in rows if f[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for f in rows:
            for nm, v in zip(names, f[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(rows[0][3]) if rows[0][3].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(float(f[4]) for f in rows if f[4].replace(".", "").isdigit())}


def host_copy_gbs(dev, stream) -> float:
    """Pinned host -> HBM copy rate (256 MB copies), the host link's reference."""
    hb = torch.empty(256 << 20, dtype=torch.uint8, pin_memory=True)
    db = torch.empty(hb.shape, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(2):
            db.copy_(hb, non_blocking=True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            db.copy_(hb, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    return 5 * hb.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9


# The sources that define each stage's kernels (their code and launch shape).
STAGE_SOURCES = {
    "attention": ("attention.cu", "attend.cuh", "common.cuh"),
    "topk": ("indexer_tc.cu", "topk.cu", "select.cuh", "common.cuh"),
}


def stage_source_sha1(stage: str) -> str:
    src = os.path.join(ROOT, "block_sparse_long_02_b200", "csrc")
    h = hashlib.sha1()
    for name in STAGE_SOURCES[stage]:
        h.update(open(os.path.join(src, name), "rb").read())
    return h.hexdigest()[:12]


def traffic_for(workload: str, stage: str):
    """DRAM bytes per launch of a stage of a workload from the committed ncu
    summary, or None when there is none or it was taken on a different version
    of the stage's kernel sources."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p) or stage not in STAGE_SOURCES:
        return None
    for ln in open(p):
        f = ln.split("#")[0].split()
        if len(f) == 4 and f[0] == workload and f[1] == stage:
            return float(f[2]) if stage_source_sha1(stage) == f[3] else None
    return None


# ----------------------------------------------------------------------------- replicas
def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (the job's time is its slowest replica's)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(tokens_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


# ----------------------------------------------------------------------------- CUDA arm
class Bench:
    def __init__(self, w, device, stage="all", kv="bf16", offload=0):
        import block_sparse_long_02_b200 as qsa
        from block_sparse_long_02_b200.layer import QSALayer

        self.qsa, self.w, self.dev = qsa, w, device
        self.stage = stage
        self.kv = kv
        self.offload = offload  # hot-cache blocks per sequence (0: K/V caches in HBM)
        cfg = qsa.Config.of(w)
        self.cfg = cfg
        B, n, S = w.batch, w.n, w.decode_steps
        cap = -(-(n + S) // w.r) * w.r
        # stage "topk" (profiling): only what key pooling and the indexer need.
        kv_cap = 1 if stage == "topk" else cap
        self.L = L = QSALayer(cfg, B, cap, device=device, kv_cap=kv_cap)
        bf = torch.bfloat16
        if stage != "topk":
            w.device_fill("k", L.k_cache.view(B, cap, -1), rows=(0, n))
            w.device_fill("v", L.v_cache.view(B, cap, -1), rows=(0, n))
        w.device_fill("idx_k", L.idx_k_cache, rows=(0, n))
        self.pre = None
        if w.prefill:
            q0, nq = w.q_begin, n - w.q_begin
            q = torch.empty(B, nq if stage != "topk" else 1, cfg.q_heads, cfg.head_dim, dtype=bf, device=device)
            iq = torch.empty(B, nq, cfg.idx_heads, cfg.idx_dim, dtype=bf, device=device)
            for s in range(B):  # rows [q0, n) of each sequence
                for name, t in (("q", q), ("idx_q", iq)):
                    if name == "q" and stage == "topk":
                        continue
                    L_ = w.row_len(name)
                    synth.fill_device(w.seed(s), synth.TENSOR_IDS[name], q0 * L_, nq * L_, t[s].data_ptr())
            self.pre = {"q": q, "idx_q": iq,
                        "out": torch.empty_like(q),
                        "sel": torch.empty(B, nq, cfg.k_blocks, dtype=torch.int32, device=device),
                        "nsel": torch.empty(B, nq, dtype=torch.int32, device=device)}
            if q0:
                L.compress(0, q0 // w.r)  # the existing cache's pooled keys
            if w.train:
                # Training step: the forward's LSE, a seeded upstream gradient, the
                # gradients, and the stage-1 target / scores / loss rows.
                dout = torch.empty_like(q)
                for s in range(B):
                    L_ = w.row_len("dout")
                    synth.fill_device(w.seed(s), synth.TENSOR_IDS["dout"], q0 * L_, nq * L_, dout[s].data_ptr())
                ld = (n - 1) // w.r
                f32 = torch.float32
                self.pre.update({
                    "lse": torch.empty(B, nq, cfg.q_heads, dtype=f32, device=device), "dout": dout,
                    "dq": torch.empty(B, nq, cfg.q_heads, cfg.head_dim, dtype=f32, device=device),
                    "dk": torch.empty(B, cap, cfg.kv_heads, cfg.head_dim, dtype=f32, device=device),
                    "dv": torch.empty(B, cap, cfg.kv_heads, cfg.head_dim, dtype=f32, device=device),
                    "ld": ld, "target": torch.empty(B, nq, ld, dtype=f32, device=device),
                    "scores": torch.empty(B, nq, ld, dtype=f32, device=device),
                    "dscores": torch.empty(B, nq, ld, dtype=f32, device=device),
                    "kl": torch.empty(B, nq, dtype=f32, device=device)})
                L.workspace(qsa.OP_INDEX_SCORES, nq)
                L.workspace(qsa.OP_DISTILL_TARGET, nq)
        else:
            L.compress(0, n // w.r)
        self.dec = []
        if S:
            tmp = {}
            for name in ("q", "k", "v", "idx_q", "idx_k"):
                t = torch.empty(B, S, w.row_len(name), dtype=bf, device=device)
                for s in range(B):
                    synth.fill_device(w.seed(s), synth.TENSOR_IDS[name], n * w.row_len(name),
                                      S * w.row_len(name), t[s].data_ptr())
                tmp[name] = t
            # Needle rows of decode positions are raw indexer keys of earlier blocks
            # (already in the cache); the decode tokens themselves carry no needles.
            for st in range(S):
                self.dec.append({
                    "pos": torch.full((B,), n + st, dtype=torch.int64, device=device),
                    "q": tmp["q"][:, st].contiguous().view(B, cfg.q_heads, cfg.head_dim),
                    "k": tmp["k"][:, st].contiguous().view(B, cfg.kv_heads, cfg.head_dim),
                    "v": tmp["v"][:, st].contiguous().view(B, cfg.kv_heads, cfg.head_dim),
                    "idx_q": tmp["idx_q"][:, st].contiguous().view(B, cfg.idx_heads, cfg.idx_dim),
                    "idx_k": tmp["idx_k"][:, st].contiguous(),
                    "out": torch.empty(B, cfg.q_heads, cfg.head_dim, dtype=bf, device=device),
                })
        # Workspaces allocated before timing.
        if w.prefill:
            L.workspace(qsa.OP_TOPK_BLOCKS, n - w.q_begin)
        if S:
            L.workspace(qsa.OP_DECODE_STEP)
        if kv == "fp8":
            # The caches already present before the timed step are held in fp8.
            cached = w.q_begin if w.prefill else n
            if cached:
                L.quantize_kv(0, cached)
                L.quantize_pooled(0, cached // w.r)
        if offload:
            if w.prefill:
                raise SystemExit("--offload applies to the decode-only workloads")
            L.offload_kv(offload)
        self.dec_graph, self.dec_graphs_1, self.graph_kernels = None, [], 0
        self.graph_launches = 0  # kernels launched by graph replays so far
        torch.cuda.synchronize()

    def capture(self):
        """The decode steps as CUDA graphs (after an eager warm-up step): one
        graph for the back-to-back steps and one per step for the cold pass.
        Replays launch the same kernels as the eager calls."""
        if not self.dec or self.dec_graph is not None:
            return
        qsa = self.qsa
        n0 = qsa.qsa_launch_count()
        q8, off = self.kv == "fp8", bool(self.offload)
        self.dec_graph = self.L.capture_decode(self.dec, q8, off)
        self.graph_kernels = qsa.qsa_launch_count() - n0
        self.dec_graphs_1 = [self.L.capture_decode([d], q8, off) for d in self.dec]
        torch.cuda.synchronize()

    def step(self, mark=None, prefill=True):
        w, L = self.w, self.L
        if self.stage == "topk":
            from block_sparse_long_02_b200 import OP_TOPK_BLOCKS, qsa_topk_blocks

            p = self.pre
            nq = w.n - w.q_begin
            L.compress(w.q_begin // w.r, w.n // w.r)
            if mark:
                mark("compress")
            qsa_topk_blocks(self.cfg, w.batch, p["idx_q"], w.q_begin, nq, L.pooled, L.cap, None, 0, p["sel"],
                            p["nsel"], L.workspace(OP_TOPK_BLOCKS, nq))
            if mark:
                mark("topk")
            return
        if self.pre is not None and prefill:
            p = self.pre
            if self.kv == "fp8":
                # The prefill's new K/V rows to E4M3 codes (the caches' other rows
                # were quantized in set-up), then the prefill on the fp8 caches.
                L.quantize_kv(w.q_begin, w.n)
                if mark:
                    mark("quantize")
                L.prefill_q8(p["q"], p["idx_q"], w.q_begin, w.n - w.q_begin, p["out"], p["sel"], p["nsel"],
                             mark=mark)
                if self.dec:  # the decode score stream reads fp8 pooled keys
                    L.quantize_pooled(w.q_begin // w.r, w.n // w.r)
                    if mark:
                        mark("quantize")
            else:
                L.prefill(p["q"], p["idx_q"], w.q_begin, w.n - w.q_begin, p["out"], p["sel"], p["nsel"],
                          lse=p.get("lse"), mark=mark)
            if w.train:
                self.train_step(mark)
        if self.dec_graph is not None:
            self.dec_graph.replay()
            self.graph_launches += self.graph_kernels
        else:
            dstep = (L.decode_step_q8 if self.kv == "fp8" else
                     L.decode_step_offload if self.offload else L.decode_step)
            for d in self.dec:
                dstep(d["pos"], d["q"], d["k"], d["v"], d["idx_q"], d["idx_k"], d["out"])
        if mark and self.dec:
            mark("decode")

    def train_step(self, mark=None):
        """The training kernels after the forward: the sparse-attention gradient
        (dk, dv accumulate, so they are cleared first), the stage-1 target, the
        materialised indexer scores and the KL loss with its gradient."""
        qsa, w, L, p, cfg = self.qsa, self.w, self.L, self.pre, self.cfg
        q0, nq, B = w.q_begin, w.n - w.q_begin, w.batch
        p["dk"].zero_()
        p["dv"].zero_()
        qsa.qsa_sparse_attention_backward(cfg, B, p["q"], q0, nq, L.k_cache, L.v_cache, L.cap, p["sel"], p["nsel"],
                                          p["out"], p["lse"], p["dout"], p["dq"], p["dk"], p["dv"])
        if mark:
            mark("backward")
        qsa.qsa_distill_target(cfg, B, p["q"], q0, nq, L.k_cache, L.cap, p["target"], p["ld"],
                               L.workspace(qsa.OP_DISTILL_TARGET, nq))
        if mark:
            mark("target")
        qsa.qsa_index_scores(cfg, B, p["idx_q"], q0, nq, L.pooled, L.cap, p["scores"], p["ld"],
                             L.workspace(qsa.OP_INDEX_SCORES, nq))
        if mark:
            mark("scores")
        qsa.qsa_distill_kl(cfg, B, q0, nq, p["target"], p["scores"], p["ld"], p["kl"], p["dscores"])
        if mark:
            mark("kl")

    # -- end to end: host buffers in, host result out -----------------------------------
    def e2e(self, steps, warmup):
        w, L, B, n = self.w, self.L, self.w.batch, self.w.n
        host_in, host_out = [], []

        def pin_like(t):
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            h.copy_(t)
            return h

        if self.pre is not None:
            for dst in (self.pre["q"], self.pre["idx_q"]) + ((self.pre["dout"],) if w.train else ()):
                host_in.append((pin_like(dst), dst))
            for src in (self.pre["out"],) + ((self.pre["kl"], self.pre["dq"], self.pre["dk"], self.pre["dv"])
                                             if w.train else ()):
                host_out.append((pin_like(src), src))
        for c in (L.k_cache, L.v_cache, L.idx_k_cache):
            for s in range(B):
                # the step's new rows (a chunked prefill's earlier rows are cache state)
                dst = c[s, w.q_begin if w.prefill else 0:n]
                host_in.append((pin_like(dst), dst))
        for d in self.dec:
            for nm in ("q", "k", "v", "idx_q", "idx_k"):
                host_in.append((pin_like(d[nm]), d[nm]))
            host_out.append((pin_like(d["out"]), d["out"]))
        h2d = sum(h.numel() * h.element_size() for h, _ in host_in)
        d2h = sum(h.numel() * h.element_size() for h, _ in host_out)
        stream = torch.cuda.current_stream()
        # A bf16 inference prefill streams its inputs and output through
        # QSALayer.prefill_from_host (transfers overlapped with the compute,
        # chunk by chunk); the decode steps' small inputs and outputs move
        # around them. The same bytes move either way.
        piped = self.pre is not None and not w.train and self.kv == "bf16" and not self.offload
        if piped:
            q0 = w.q_begin
            hq, hiq, hout = host_in[0][0], host_in[1][0], host_out[0][0]
            hk = pin_like(L.k_cache[:, q0:n])
            hv = pin_like(L.v_cache[:, q0:n])
            hik = pin_like(L.idx_k_cache[:, q0:n])
            dec_in = host_in[2 + 3 * B:]
            dec_out = host_out[1:]

        def one():
            if piped:
                L.prefill_from_host(hq, hiq, hk, hv, hik, w.q_begin, n - w.q_begin, hout)
                for h, dv in dec_in:
                    dv.copy_(h, non_blocking=True)
                self.step(prefill=False)
                for h, dv in dec_out:
                    h.copy_(dv, non_blocking=True)
                return
            for h, dv in host_in:
                dv.copy_(h, non_blocking=True)
            self.step()
            for h, dv in host_out:
                h.copy_(dv, non_blocking=True)

        for _ in range(warmup):
            one()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            one()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps, h2d, d2h


def run_cuda(args, w, rank, world):
    dev = torch.device("cuda", torch.cuda.current_device())
    b = Bench(w, dev, stage=args.stage, kv=args.kv, offload=args.offload)
    qsa = b.qsa
    qsa.qsa_set_attention_kernel(qsa.ATTENTION_TCGEN05 if args.attention == "tcgen05" else qsa.ATTENTION_WARP)
    qsa.qsa_set_decode_kernel(qsa.DECODE_THREE_KERNELS if args.decode == "three" else qsa.DECODE_STEP_KERNEL)
    for k in range(args.warmup):
        b.step()
        if k == 0 and not args.no_graph:
            b.capture()  # decode steps replayed from CUDA graphs from here on
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    bus = getattr(torch.cuda.get_device_properties(dev), "pci_bus_id", None)
    clocks = ClockSampler(bus)
    clocks.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    marks = []

    def mark(name):
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        marks.append((name, e))

    launches0 = qsa.qsa_launch_count() + b.graph_launches
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        mark("start")
        b.step(mark)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    launches = qsa.qsa_launch_count() + b.graph_launches - launches0
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / args.steps
    stage_ms = {}
    prev = None
    for name, e in marks:
        if name != "start" and prev is not None:
            stage_ms[name] = stage_ms.get(name, 0.0) + prev.elapsed_time(e) / args.steps
        prev = e
    ms = max_over_ranks(ms, world, dev)

    alg = algorithmic(w, args.kv)
    pk = peaks()
    tokens = alg["prefill_tokens"] + alg["decode_tokens"]
    stages = {}
    defs = {"compress": ("hbm", alg["compress_bytes"]), "topk": ("tensor", alg["index_flops"]),
            "quantize": ("hbm", alg["quantize_bytes"]),
            "attention": ("hbm", alg["attn_gather_bytes"]), "decode": ("hbm", alg["decode_bytes"]),
            "backward": ("hbm", alg["bwd_bytes"]), "target": ("tensor", alg["target_flops"]),
            "scores": ("hbm", alg["scores_bytes"]), "kl": ("hbm", alg["kl_bytes"])}
    for name, t in stage_ms.items():
        bound, amount = defs[name]
        if bound == "hbm":
            ach = amount / (t * 1e-3) / 1e9
            peak = pk["hbm_gbs"]
            unit = "GB/s"
        else:
            ach = amount / (t * 1e-3) / 1e12
            peak = pk["bf16_tflops_sustained"]
            unit = "TFLOP/s"
        stages[name] = {"ms": round(t, 4), "bound": bound, "achieved": round(ach, 2), "unit": unit,
                        "frac": round(ach / peak, 4)}
    if "attention" in stages:
        stages["attention"]["tensor_tflops"] = round(alg["attn_flops"] / (stage_ms["attention"] * 1e-3) / 1e12, 2)
    if "backward" in stages:
        stages["backward"]["tensor_tflops"] = round(alg["bwd_flops"] / (stage_ms["backward"] * 1e-3) / 1e12, 2)
    dom = max(stage_ms, key=stage_ms.get)
    if b.dec and args.stage == "all":
        # Cold decode: the same steps again (re-writing the same cache rows), each
        # after a 256 MB write that evicts L2; only the decode calls are timed.
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        evs = []
        for k, d in enumerate(b.dec):
            flush.fill_(len(evs) & 0xFF)
            if b.offload:
                b.L.hot_tags.fill_(-1)  # every selected block misses: read over the host link
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            if b.dec_graphs_1:
                b.dec_graphs_1[k].replay()
            else:
                (b.L.decode_step_q8 if b.kv == "fp8" else b.L.decode_step)(
                    d["pos"], d["q"], d["k"], d["v"], d["idx_q"], d["idx_k"], d["out"])
            a1.record(stream)
            evs.append((a0, a1))
        torch.cuda.synchronize()
        cold = sum(x.elapsed_time(y) for x, y in evs)
        del flush
        ach = alg["decode_bytes"] / (cold * 1e-3) / 1e9
        stages["decode_cold"] = {"ms": round(cold, 4), "bound": "hbm", "achieved": round(ach, 2), "unit": "GB/s",
                                 "frac": round(ach / pk["hbm_gbs"], 4),
                                 "note": "each step after a 256 MB L2-evicting write"}
        if b.offload:
            host = alg["decode_gather_bytes"] / (cold * 1e-3) / 1e9
            stages["decode_cold"]["note"] += ("; hot cache emptied before each step, so every selected block and the "
                                              "tail are read from host memory by the attention (host_gbs counts "
                                              "these bytes), and the install kernel reads the blocks once more")
            stages["decode_cold"]["host_gbs"] = round(host, 2)
            stages["decode_cold"]["host_copy_gbs"] = round(host_copy_gbs(dev, stream), 2)
    ds = stages[dom]
    roofline = {"bound": ds["bound"], "achieved": ds["achieved"],
                "peak": pk["hbm_gbs"] if ds["bound"] == "hbm" else pk["bf16_tflops_sustained"],
                "unit": ds["unit"], "frac": ds["frac"], "traffic": traffic_for(w.name + ("" if args.kv == "bf16" else "+fp8"), dom), "kernel": dom,
                "peak_source": pk["source"] + (" (sustained bf16)" if ds["bound"] == "tensor" else " (copy)")}

    res = {
        "metric": METRIC, "value": round(job_value(tokens, ms, world), 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if args.kv == "bf16" else "bf16 (K/V caches fp8 E4M3)",
        "data": "synthetic: seeded counter-based N(0,1) bf16 inputs with planted needle blocks",
        "config": {"workload": w.name, "n": w.n, "q_begin": w.q_begin, "batch": w.batch,
                   "decode_steps": w.decode_steps, "r": w.r,
                   "K": w.K, "k_B": w.k_blocks, "indexer": f"{w.idx_heads}x{w.idx_dim} MQA",
                   "core": f"GQA {w.q_heads}q/{w.kv_heads}kv d={w.head_dim}",
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": (f"inputs larger than L2 (K/V cache {2 * w.batch * w.total * w.kv_heads * w.head_dim * 2 / 1e9:.1f} GB"
                          f" gathered, q {w.batch * (w.n - w.q_begin) * w.q_heads * w.head_dim * 2 / 1e9:.2f} GB);"
                          " decode steps back to back"),
                   "decode_launch": "eager calls" if b.dec_graph is None else "CUDA graph replay of the steps",
                   "kv_location": ("HBM" if not args.offload else
                                   f"pinned host memory, {args.offload} hot blocks per sequence in HBM"),
                   "kv_cache": ("bf16" if args.kv == "bf16" else
                                "fp8 E4M3 codes + one fp32 scale per row: core K/V, and pooled keys for decode"),
                   "attention_kernel": ("tcgen05 tiles in TMEM, TMA block gathers" if args.attention == "tcgen05"
                                        and args.kv == "bf16" else "warp-level mma.sync tiles, cp.async gathers"),
                   "decode_kernels": ("three per step: scores, selection, attention" if args.decode == "three"
                                      else "one persistent kernel per step")},
        "roofline": roofline, "stages": stages,
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if alg["prefill_tokens"] and "decode" in stage_ms:
        pre_ms = sum(stage_ms.get(k, 0.0) for k in ("compress", "topk", "attention"))
        res["prefill_tokens_per_s"] = round(alg["prefill_tokens"] / (pre_ms * 1e-3), 1)
        res["decode_tokens_per_s"] = round(alg["decode_tokens"] / (stage_ms["decode"] * 1e-3), 1)
    if not args.no_e2e:
        e_ms, h2d, d2h = b.e2e(max(5, args.steps), 1)
        e_ms = max_over_ranks(e_ms, world, dev)
        res["e2e"] = {"value": round(job_value(tokens, e_ms, world), 2), "unit": "tokens/s",
                      "ms_per_step": round(e_ms, 3), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}
    return res


# ----------------------------------------------------------------------------- oracle (CPU)
class OracleTimer:
    """Times the oracle (single-threaded C) on a bounded sample of the workload and
    extrapolates one whole step: key pooling timed on `blocks` blocks, prefill
    rows on `rows` positions stratified over [0, n) (fit t(i) = a + b*floor(i/r)),
    and `dec` decode positions."""

    def __init__(self, w):
        import oracle

        self.w = w
        self.o = oracle.Oracle.for_workload(w)
        n = w.n
        self.idx_k = w.host_full("idx_k", 0, n + w.decode_steps)
        t = time.perf_counter()
        self.pooled = self.o.compress(self.idx_k, (n + w.decode_steps) // w.r)
        self.t_compress_full = time.perf_counter() - t

    def _row(self, i):
        w, o = self.w, self.o
        train = w.train and i < w.n
        iq = w.host_rows("idx_q", 0, [i]).reshape(w.idx_heads, w.idx_dim)
        qr = w.host_rows("q", 0, [i]).reshape(w.q_heads, w.head_dim)
        t = time.perf_counter()
        res = o.row(i, iq, self.pooled, want_scores=train)
        t_sel = time.perf_counter() - t
        toks = o.token_set(res["sel"], i)
        kc = w.host_rows("k", 0, toks)
        vc = w.host_rows("v", 0, toks)
        t = time.perf_counter()
        o.attention(qr, kc, vc, np.arange(toks.size, dtype=np.int64))
        t_att = time.perf_counter() - t
        if not train:
            return t_sel + t_att
        # The training kernels' work for this row: the attention gradient, the
        # stage-1 target over tokens <= i, and the KL with its gradient.
        g = w.host_rows("dout", 0, [i]).reshape(w.q_heads, w.head_dim)
        k_all = w.host_rows("k", 0, np.arange(i + 1))
        t = time.perf_counter()
        o.attention_backward(qr, kc, vc, np.arange(toks.size, dtype=np.int64), g)
        tgt = o.distill_target(i, qr, k_all)
        o.distill_kl(tgt, res["scores"])
        return t_sel + t_att + time.perf_counter() - t

    def sample(self, rows, dec, blocks):
        w = self.w
        n, r = w.n, w.r
        total = 0.0
        parts = {}
        if w.prefill:
            q0 = w.q_begin
            nb = n // r - q0 // r
            b = min(blocks, nb)
            t = time.perf_counter()
            self.o.compress(self.idx_k, b)
            tc = (time.perf_counter() - t) * nb / max(b, 1)
            pos = sorted(set([q0 + int((k + 0.5) * (n - q0) / rows) for k in range(rows)] + [n - 1]))
            ts = np.array([self._row(i) for i in pos])
            x = np.array([i // r for i in pos], dtype=np.float64)
            A = np.stack([np.ones_like(x), x], 1)
            if len(set(x.tolist())) < 2:  # (a chunk inside one block range: constant work)
                a, bcoef = float(ts.mean()), 0.0
            else:
                (a, bcoef), *_ = np.linalg.lstsq(A, ts, rcond=None)
            pairs = float((np.arange(q0, n) // r).sum())
            tp = (n - q0) * a + bcoef * pairs
            resid = float(np.sqrt(np.mean((A @ np.array([a, bcoef]) - ts) ** 2)))
            parts.update(compress_s=tc, prefill_rows_s=tp, fit={"a_s": a, "b_s": bcoef, "rms_resid_s": resid,
                                                                 "rows": len(pos)})
            total += tc + tp
        if w.decode_steps:
            ps = [n + int(k * w.decode_steps / dec) for k in range(dec)]
            td = np.mean([self._row(p) for p in ps])
            parts["decode_s_per_step"] = td
            total += td * w.decode_steps
        return total * w.batch, parts


def host_cpu():
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return model, os.cpu_count()


class one_core:
    """Pins the calling process to one CPU (the oracle is single-threaded) and
    restores the previous affinity on exit."""

    def __enter__(self):
        self.prev = os.sched_getaffinity(0)
        os.sched_setaffinity(0, {min(self.prev)})
        return self

    def __exit__(self, *exc):
        os.sched_setaffinity(0, self.prev)


def cpu_baseline(w, rows=64, dec=2, blocks=65536):
    if w.train:
        rows = 16  # each row also runs the dense stage-1 target over tokens <= i
    with one_core():
        ot = OracleTimer(w)
        t, parts = ot.sample(rows, dec, blocks)
    tokens = ((w.n - w.q_begin) if w.prefill else 0) * w.batch + w.decode_steps * w.batch
    model, ncpu = host_cpu()
    return {"value": round(tokens / t, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "cpu_model": model, "host_cores": ncpu,
            "sample": (f"{parts.get('fit', {}).get('rows', 0)} prefill rows stratified over [q_begin,n)"
                       + (" (each also running the attention gradient, the stage-1 target and the KL)"
                          if w.train else "")
                       + f" fitted by t(i)=a+b*floor(i/r) and extrapolated over all n; key pooling timed on "
                       f"{blocks} blocks and scaled"
                       + (f"; {dec} decode positions, scaled to {w.decode_steps} steps" if w.decode_steps else "")),
            "extrapolated_step_s": round(t, 3), "parts": {k: (round(v, 4) if isinstance(v, float) else v)
                                                        for k, v in parts.items()}}


# The other workloads of the metric, measured in the same run as the headline
# (one GPU): tokens/s, the stage rooflines and the oracle beside each.
OTHER_CONFIGS = (("decode_b1_n32k", 50), ("prefill_n128k", 3), ("decode_b8_n256k", 50))


def run_configs(args):
    import copy

    out = {}
    for name, steps in OTHER_CONFIGS:
        a = copy.copy(args)
        a.workload, a.steps, a.warmup, a.no_e2e, a.n = name, steps, 3, True, None
        w = synth.WORKLOADS[name]
        r = run_cuda(a, w, 0, 1)
        torch.cuda.empty_cache()
        ent = {k: r[k] for k in ("value", "unit", "ms_per_step", "steps", "roofline", "stages", "gpu_launches",
                                 "clocks", "config")}
        for k in ("prefill_tokens_per_s", "decode_tokens_per_s"):
            if k in r:
                ent[k] = r[k]
        if not args.no_cpu_baseline:
            ent["cpu_baseline"] = cpu_baseline(w, rows=32)
        out[name] = ent
    return out


def run_reference(args, w):
    times = []
    with one_core():
        ot = OracleTimer(w)
        for k in range(args.warmup + args.steps):
            t, parts = ot.sample(rows=6, dec=1, blocks=8192)
            if k >= args.warmup:
                times.append(t)
    model, ncpu = host_cpu()
    t = float(np.mean(times))
    tokens = ((w.n - w.q_begin) if w.prefill else 0) * w.batch + w.decode_steps * w.batch
    v = tokens / t
    return {"metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(t * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "impl": "reference",
            "data": "synthetic: seeded counter-based N(0,1) bf16 inputs with planted needle blocks",
            "config": {"workload": w.name, "n": w.n, "batch": w.batch, "decode_steps": w.decode_steps,
                       "r": w.r, "K": w.K},
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "cpu_model": model, "host_cores": ncpu,
                             "sample": "per step: 6 stratified prefill rows (fit t(i)=a+b*floor(i/r)), key "
                                       "pooling on 8192 blocks, 1 decode position; extrapolated to the step"},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="decode steps as eager calls, not CUDA graph replays")
    ap.add_argument("--offload", type=int, default=0, metavar="SLOTS",
                    help="decode with the K/V caches in pinned host memory and SLOTS hot blocks per sequence in HBM")
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16",
                    help="core K/V cache format of the prefill attention (fp8: E4M3 codes, per-row scales)")
    ap.add_argument("--stage", choices=["all", "topk"], default="all",
                    help="topk: time only key pooling + the fused indexer (for profiling)")
    ap.add_argument("--n", type=int, default=None, help="override the workload's sequence length")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads that the default run also measures (32K and 8x256K decode, "
                         "128K prefill)")
    ap.add_argument("--decode", choices=["step", "three"], default="three",
                    help="decode step as three kernels (default) or as one persistent kernel")
    ap.add_argument("--attention", choices=["warp", "tcgen05"], default="warp",
                    help="sparse-attention kernel on bf16 caches: warp-level tiles (default) or tcgen05 tiles in TMEM "
                         "fed by TMA block gathers")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.n is not None:
        import dataclasses

        w = dataclasses.replace(w, n=args.n, name=f"{w.name}@n={args.n}",
                                n_needles_prefill=min(w.n_needles_prefill, args.n // 4096))
    if args.stage == "topk":
        args.no_e2e = True
        args.no_cpu_baseline = True

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return
    if world > 1:
        import datetime

        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    res = run_cuda(args, w, rank, world)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(w)
        if world == 1 and args.workload == DEFAULT_WORKLOAD and args.stage == "all" and args.n is None \
                and not args.no_configs and not args.offload and args.kv == "bf16":
            res["configs"] = run_configs(args)
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
