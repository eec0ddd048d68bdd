"""QSALayer: the layer's buffers plus the call sequence of the C-ABI.

Holds the per-layer caches (core K/V, raw indexer keys, pooled indexer keys)
and the workspaces, all allocated once with torch, and issues the library
calls in the order the layer runs them:

  prefill(q, idx_q, q_begin, nq):   qsa_compress_keys -> qsa_topk_blocks (fused)
                                    -> qsa_sparse_attention
  prefill_from_host(...):           the same per chunk of positions, with the
                                    host <-> device copies of the inputs and the
                                    output overlapped on side streams
  decode_step(pos, q, k, v, idx_q, idx_k): qsa_decode_step

Every step of the computation runs in libqsa.so; this class only owns memory
and marshals arguments.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (OP_DECODE_STEP, OP_SPARSE_ATTENTION, OP_TOPK_BLOCKS, Config, qsa_compress_keys, qsa_decode_step,
               qsa_decode_step_offload, qsa_decode_step_q8, qsa_quantize_rows,
               qsa_sparse_attention, qsa_sparse_attention_q8, qsa_topk_blocks, qsa_workspace_size)


class QSALayer:
    def __init__(self, cfg: Config, batch: int, cap: int, device="cuda", rms_w: Optional[torch.Tensor] = None,
                 kv_cap: Optional[int] = None):
        self.cfg, self.batch, self.cap = cfg, batch, cap
        self.device = torch.device(device)
        bf = torch.bfloat16
        kv_cap = cap if kv_cap is None else kv_cap  # smaller only for indexer-only use
        self.k_cache = torch.zeros(batch, kv_cap, cfg.kv_heads, cfg.head_dim, dtype=bf, device=self.device)
        self.v_cache = torch.zeros_like(self.k_cache)
        self.idx_k_cache = torch.zeros(batch, cap, cfg.idx_dim, dtype=bf, device=self.device)
        self.pooled = torch.zeros(batch, cap // cfg.r, cfg.idx_dim, dtype=bf, device=self.device)
        self.rms_w = rms_w
        self._ws = {}

    def workspace(self, op: int, nq: int = 0) -> torch.Tensor:
        need = qsa_workspace_size(self.cfg, op, self.batch, self.cap, nq)
        ws = self._ws.get(op)
        if ws is None or ws.numel() < need:
            ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=self.device)
            self._ws[op] = ws
        return ws

    def compress(self, blk_begin: int, blk_end: int, stream=None) -> None:
        qsa_compress_keys(self.cfg, self.batch, self.idx_k_cache, self.cap, self.rms_w, blk_begin, blk_end,
                          self.pooled, stream)

    def prefill(self, q: torch.Tensor, idx_q: torch.Tensor, q_begin: int, nq: int,
                out: torch.Tensor, sel: torch.Tensor, nsel: torch.Tensor,
                lse: Optional[torch.Tensor] = None, stream=None, mark=None) -> None:
        """Queries [q_begin, q_begin + nq) of every sequence, whose keys and values
        (positions < q_begin + nq) are already in the caches. `mark(name)`, if
        given, is called after each stage (e.g. to record a CUDA event)."""
        r = self.cfg.r
        self.compress(q_begin // r, (q_begin + nq) // r, stream)
        if mark:
            mark("compress")
        ws = self.workspace(OP_TOPK_BLOCKS, nq)
        qsa_topk_blocks(self.cfg, self.batch, idx_q, q_begin, nq, self.pooled, self.cap, None, 0, sel, nsel,
                        ws, stream)
        if mark:
            mark("topk")
        qsa_sparse_attention(self.cfg, self.batch, q, q_begin, nq, self.k_cache, self.v_cache, self.cap, sel,
                             nsel, out, lse, self.workspace(OP_SPARSE_ATTENTION), stream)
        if mark:
            mark("attention")

    def prefill_from_host(self, host_q: torch.Tensor, host_idx_q: torch.Tensor, host_k: torch.Tensor,
                          host_v: torch.Tensor, host_idx_k: torch.Tensor, q_begin: int, nq: int,
                          host_out: torch.Tensor, chunk: int = 131072, first: int = 8192) -> None:
        """prefill of positions [q_begin, q_begin + nq) whose inputs and output
        live in pinned host memory: host_q [batch][nq][q_heads][128], host_idx_q
        [batch][nq][4][128], the new cache rows host_k, host_v
        [batch][nq][kv_heads][128] and host_idx_k [batch][nq][128], and host_out
        [batch][nq][q_heads][128] (rows before q_begin are already in the
        caches). The positions go in chunks: chunk j's rows move to the device
        on one stream while chunk j - 1 computes on the current stream, and its
        output returns on a third stream while chunk j + 1 computes. The chunks
        grow from `first` positions, doubling, to `chunk` and shrink the same way
        at the end, so that only a small first transfer and a small last output
        copy are not overlapped. Each chunk is the prefill call on a
        double-buffered staging area, so the outputs equal prefill's bit for bit.
        Returns when the work is queued; host_out is complete once the current
        stream has synchronised, and the host tensors must stay alive and
        unchanged until then."""
        B, r = self.batch, self.cfg.r
        chunk = max(r, min(chunk, nq) // r * r)
        plan = self.chunk_plan(nq, chunk, max(r, min(first, chunk) // r * r))
        dev = self.device
        bf = torch.bfloat16
        cs = torch.cuda.current_stream(dev)
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        stage = [{"q": torch.empty(B, chunk, *host_q.shape[2:], dtype=bf, device=dev),
                  "idx_q": torch.empty(B, chunk, *host_idx_q.shape[2:], dtype=bf, device=dev),
                  "out": torch.empty(B, chunk, *host_out.shape[2:], dtype=bf, device=dev),
                  "sel": torch.empty(B, chunk, self.cfg.k_blocks, dtype=torch.int32, device=dev),
                  "nsel": torch.empty(B, chunk, dtype=torch.int32, device=dev)} for _ in range(2)]
        for st in stage:  # the staging area is written on the side streams
            for t in st.values():
                t.record_stream(h2d)
                t.record_stream(d2h)
        computed, drained = [None, None], [None, None]  # per staging set: last compute / output copy
        cs_ready = torch.cuda.Event()
        cs_ready.record(cs)
        h2d.wait_event(cs_ready)  # the caches and staging exist before the first copy
        a = 0
        for j, m in enumerate(plan):
            st = stage[j % 2]
            with torch.cuda.stream(h2d):
                if computed[j % 2] is not None:  # chunk j - 2 has read this set
                    h2d.wait_event(computed[j % 2])
                p0 = q_begin + a
                for s in range(B):
                    self.k_cache[s, p0:p0 + m].copy_(host_k[s, a:a + m], non_blocking=True)
                    self.v_cache[s, p0:p0 + m].copy_(host_v[s, a:a + m], non_blocking=True)
                    self.idx_k_cache[s, p0:p0 + m].copy_(host_idx_k[s, a:a + m], non_blocking=True)
                    st["q"][s, :m].copy_(host_q[s, a:a + m], non_blocking=True)
                    st["idx_q"][s, :m].copy_(host_idx_q[s, a:a + m], non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(h2d)
            cs.wait_event(arrived)
            if drained[j % 2] is not None:  # chunk j - 2's output has left this set
                cs.wait_event(drained[j % 2])
            q_in = st["q"] if m == chunk else st["q"][:, :m].contiguous()
            iq_in = st["idx_q"] if m == chunk else st["idx_q"][:, :m].contiguous()
            out = st["out"] if m == chunk else torch.empty(B, m, *host_out.shape[2:], dtype=bf, device=dev)
            sel = st["sel"] if m == chunk else torch.empty(B, m, self.cfg.k_blocks, dtype=torch.int32, device=dev)
            nsel = st["nsel"] if m == chunk else torch.empty(B, m, dtype=torch.int32, device=dev)
            self.prefill(q_in, iq_in, p0, m, out, sel, nsel)
            done = torch.cuda.Event()
            done.record(cs)
            computed[j % 2] = done
            with torch.cuda.stream(d2h):
                d2h.wait_event(done)
                out.record_stream(d2h)
                for s in range(B):
                    host_out[s, a:a + m].copy_(out[s], non_blocking=True)
                left = torch.cuda.Event()
                left.record(d2h)
            drained[j % 2] = left
            a += m
        # The current stream waits for the last output copies.
        for ev in drained:
            if ev is not None:
                cs.wait_event(ev)

    @staticmethod
    def chunk_plan(nq: int, chunk: int, first: int) -> list:
        """Chunk sizes of prefill_from_host: first, 2 first, ... below chunk at
        both ends (while they fit twice), chunk-sized ones between, and the
        remainder as one more middle chunk; they sum to nq."""
        ramp, c = [], first
        while c < chunk and 2 * (sum(ramp) + c) <= nq:
            ramp.append(c)
            c *= 2
        middle = nq - 2 * sum(ramp)
        mids = [chunk] * (middle // chunk) + ([middle % chunk] if middle % chunk else [])
        return ramp + mids + ramp[::-1]

    def prefill_varlen(self, q: torch.Tensor, idx_q: torch.Tensor, q_begin, nq, out: torch.Tensor,
                       sel: torch.Tensor, nsel: torch.Tensor, lse: Optional[torch.Tensor] = None,
                       stream=None) -> None:
        """Prefill of a different query range per sequence in one call each:
        queries [q_begin[s], q_begin[s] + nq[s]) of sequence s (host lists),
        packed one sequence after another in q ([total][q_heads][128]), idx_q,
        out, sel, nsel and lse. Their keys and values are already in the caches."""
        from . import qsa_sparse_attention_varlen, qsa_topk_blocks_varlen

        r = self.cfg.r
        for s, (b, m) in enumerate(zip(q_begin, nq)):
            if m:
                qsa_compress_keys(self.cfg, 1, self.idx_k_cache[s:s + 1], self.cap, self.rms_w, b // r,
                                  (b + m) // r, self.pooled[s:s + 1], stream)
        ws = self.workspace_for(OP_TOPK_BLOCKS, 1, max(nq))
        qsa_topk_blocks_varlen(self.cfg, idx_q, q_begin, nq, self.pooled, self.cap, sel, nsel, ws, stream)
        qsa_sparse_attention_varlen(self.cfg, q, q_begin, nq, self.k_cache, self.v_cache, self.cap, sel, nsel, out,
                                    lse, self.workspace(OP_SPARSE_ATTENTION), stream)

    def workspace_for(self, op: int, batch: int, nq: int) -> torch.Tensor:
        """A workspace of `op` for `batch` sequences and nq queries (kept per op
        and size class; grown as needed)."""
        need = qsa_workspace_size(self.cfg, op, batch, self.cap, nq)
        key = (op, batch)
        ws = self._ws.get(key)
        if ws is None or ws.numel() < need:
            ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=self.device)
            self._ws[key] = ws
        return ws

    # ------------------------------------------------ fp8 (E4M3) core K/V caches
    def quantize_kv(self, begin: int, end: int, stream=None) -> None:
        """FP8 copies of the core K/V cache rows [begin, end) of every sequence
        (allocated on first use: codes [batch][cap][kv_heads][head_dim] uint8,
        scales [batch][cap][kv_heads] fp32), read by prefill_q8."""
        if getattr(self, "k8", None) is None:
            shape = self.k_cache.shape
            self.k8 = torch.zeros(shape, dtype=torch.uint8, device=self.device)
            self.v8 = torch.zeros_like(self.k8)
            self.ks = torch.zeros(shape[:3], dtype=torch.float32, device=self.device)
            self.vs = torch.zeros_like(self.ks)
        h, d = self.cfg.kv_heads, self.cfg.head_dim
        for s in range(self.batch):
            for src, codes, scales in ((self.k_cache, self.k8, self.ks), (self.v_cache, self.v8, self.vs)):
                qsa_quantize_rows(src[s, begin:end], (end - begin) * h, d, codes[s, begin:end], scales[s, begin:end],
                                  stream)

    def quantize_pooled(self, blk_begin: int, blk_end: int, stream=None) -> None:
        """FP8 copies of the pooled keys of blocks [blk_begin, blk_end) of every
        sequence (codes [batch][cap/r][128] uint8, scales [batch][cap/r] fp32),
        read by decode_step_q8's score stream."""
        if getattr(self, "pooled8", None) is None:
            self.pooled8 = torch.zeros(self.pooled.shape, dtype=torch.uint8, device=self.device)
            self.pscale = torch.zeros(self.pooled.shape[:2], dtype=torch.float32, device=self.device)
        for s in range(self.batch):
            qsa_quantize_rows(self.pooled[s, blk_begin:blk_end], blk_end - blk_begin, self.cfg.idx_dim,
                              self.pooled8[s, blk_begin:blk_end], self.pscale[s, blk_begin:blk_end], stream)

    def decode_step_q8(self, pos: torch.Tensor, q, k, v, idx_q, idx_k, out, sel_out=None, nsel_out=None,
                       stream=None) -> None:
        """decode_step on the fp8 caches (quantize_kv and quantize_pooled must
        cover the cached positions and blocks)."""
        ws = self.workspace(OP_DECODE_STEP)
        qsa_decode_step_q8(self.cfg, self.batch, pos, q, k, v, idx_q, idx_k, self.k8, self.ks, self.v8, self.vs,
                           self.idx_k_cache, self.pooled, self.pooled8, self.pscale, self.cap, self.rms_w, out,
                           sel_out, nsel_out, ws, stream)

    # ------------------------------------------------ host-offloaded K/V caches
    def offload_kv(self, hot_blocks: int) -> None:
        """Moves the core K/V caches to pinned host memory (copying their
        contents) and puts an HBM cache of hot_blocks blocks per sequence
        (plus the tail slot) in front of them, initially empty;
        decode_step_offload uses them."""
        self.host_k = torch.empty(self.k_cache.shape, dtype=self.k_cache.dtype, pin_memory=True)
        self.host_v = torch.empty_like(self.host_k, pin_memory=True)
        self.host_k.copy_(self.k_cache)
        self.host_v.copy_(self.v_cache)
        c = self.cfg
        self.hot_blocks = hot_blocks
        self.hot_k = torch.zeros(self.batch, hot_blocks + 1, c.r, c.kv_heads, c.head_dim, dtype=torch.bfloat16,
                                 device=self.device)
        self.hot_v = torch.zeros_like(self.hot_k)
        self.hot_tags = torch.full((self.batch, hot_blocks + 1), -1, dtype=torch.int32, device=self.device)

    def decode_step_offload(self, pos: torch.Tensor, q, k, v, idx_q, idx_k, out, sel_out=None, nsel_out=None,
                            stream=None) -> None:
        ws = self.workspace(OP_DECODE_STEP)
        qsa_decode_step_offload(self.cfg, self.batch, pos, q, k, v, idx_q, idx_k, self.host_k, self.host_v,
                                self.hot_k, self.hot_v, self.hot_tags, self.hot_blocks, self.idx_k_cache, self.pooled,
                                self.cap, self.rms_w, out, sel_out, nsel_out, ws, stream)

    def prefill_q8(self, q: torch.Tensor, idx_q: torch.Tensor, q_begin: int, nq: int, out: torch.Tensor,
                   sel: torch.Tensor, nsel: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None,
                   mark=None) -> None:
        """As prefill, with the sparse attention reading the fp8 K/V caches
        (quantize_kv must cover positions < q_begin + nq)."""
        r = self.cfg.r
        self.compress(q_begin // r, (q_begin + nq) // r, stream)
        if mark:
            mark("compress")
        ws = self.workspace(OP_TOPK_BLOCKS, nq)
        qsa_topk_blocks(self.cfg, self.batch, idx_q, q_begin, nq, self.pooled, self.cap, None, 0, sel, nsel,
                        ws, stream)
        if mark:
            mark("topk")
        qsa_sparse_attention_q8(self.cfg, self.batch, q, q_begin, nq, self.k8, self.ks, self.v8, self.vs, self.cap,
                                sel, nsel, out, lse, None, stream)
        if mark:
            mark("attention")

    def decode_step(self, pos: torch.Tensor, q, k, v, idx_q, idx_k, out, sel_out=None, nsel_out=None,
                    stream=None) -> None:
        ws = self.workspace(OP_DECODE_STEP)
        qsa_decode_step(self.cfg, self.batch, pos, q, k, v, idx_q, idx_k, self.k_cache, self.v_cache,
                        self.idx_k_cache, self.pooled, self.cap, self.rms_w, out, sel_out, nsel_out, ws,
                        stream)

    def capture_decode(self, steps, q8: bool = False, offload: bool = False) -> "torch.cuda.CUDAGraph":
        """Captures the decode steps `steps` (a list of dicts with the
        decode_step arguments pos, q, k, v, idx_q, idx_k, out) into one CUDA
        graph, run by `graph.replay()`: one launch for the whole sequence of
        steps, with the kernels' programmatic dependencies kept as graph edges.
        The graph holds the tensors' addresses: refill the same tensors
        between replays. The workspace is allocated (and warmed) first, so
        nothing is allocated during capture."""
        self.workspace(OP_DECODE_STEP)
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side, capture_error_mode="thread_local"):
            step = self.decode_step_q8 if q8 else (self.decode_step_offload if offload else self.decode_step)
            for d in steps:
                step(d["pos"], d["q"], d["k"], d["v"], d["idx_q"], d["idx_k"], d["out"])
        torch.cuda.current_stream(self.device).wait_stream(side)
        return graph
