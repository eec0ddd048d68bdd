"""QSA layer oracle (Python face of ``oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``; never by the product path. It is a plain,
slow, single-threaded statement of the layer (pool -> RMSNorm -> partial RoPE ->
ReLU-sum indexer score -> top-k_B blocks -> expand + tail -> attention), written
from the "QSA (Qwen Sparse Attention)" concept page, section "Key math / How it
works", and the "Qwen Sparse Attention" gallery page, section "How block
selection works"; plus the training pieces of the concept page's "Native
trainability" section (the gradient of the sparse attention, the stage-1
block-max-pooled dense target and its KL loss). Every function is pinned by
``tests/test_oracle_pins.py``; none is "parity unpinned".

Arrays are numpy: bf16 values travel as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

GCC_FLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False, src: str = _SRC, out: str = _SO) -> str:
    """Compile oracle.c (plain C, single-threaded, strict IEEE fp64)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", out, src, "-lm"])
    return out


class Cfg(ctypes.Structure):
    _fields_ = [("r", ctypes.c_int32), ("K", ctypes.c_int32),
                ("idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
                ("rope_dims", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("rms_eps", ctypes.c_double),
                ("q_heads", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("sm_scale", ctypes.c_double)]


def _p(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


class Oracle:
    """The oracle for one layer configuration (shapes of a ``synth.Workload``)."""

    def __init__(self, r=4, K=2048, idx_heads=4, idx_dim=128, rope_dims=64, rope_base=10000.0,
                 rms_eps=1e-6, q_heads=32, kv_heads=4, head_dim=128, sm_scale=0.0,
                 lib_path: Optional[str] = None):
        path = lib_path or build()
        self.lib = ctypes.CDLL(path)
        self.cfg = Cfg(r, K, idx_heads, idx_dim, rope_dims, rope_base, rms_eps, q_heads, kv_heads,
                       head_dim, sm_scale)
        self._c = ctypes.byref(self.cfg)
        L = self.lib
        vp = ctypes.c_void_p
        L.qsa_oracle_k_blocks.restype = ctypes.c_int64
        L.qsa_oracle_k_blocks.argtypes = [vp]
        L.qsa_oracle_rope.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int64, vp]
        L.qsa_oracle_pool_block.argtypes = [vp, vp, vp, ctypes.c_int64, vp, vp, vp, vp]
        L.qsa_oracle_compress.argtypes = [vp, vp, ctypes.c_int64, vp, vp]
        L.qsa_oracle_rotate_query.argtypes = [vp, vp, ctypes.c_int64, vp]
        L.qsa_oracle_scores.argtypes = [vp, vp, vp, ctypes.c_int64, vp]
        L.qsa_oracle_select.restype = ctypes.c_int64
        L.qsa_oracle_select.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp]
        L.qsa_oracle_token_set.restype = ctypes.c_int64
        L.qsa_oracle_token_set.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int64, vp]
        L.qsa_oracle_attention.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int64, vp, vp]
        L.qsa_oracle_row.restype = ctypes.c_int64
        L.qsa_oracle_row.argtypes = [vp, ctypes.c_int64, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.qsa_oracle_decode_step.restype = ctypes.c_int64
        L.qsa_oracle_decode_step.argtypes = [vp, ctypes.c_int64] + [vp] * 13
        L.qsa_oracle_e4m3_value.restype = ctypes.c_double
        L.qsa_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.qsa_oracle_e4m3_encode.restype = ctypes.c_uint8
        L.qsa_oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.qsa_oracle_quant_rows.argtypes = [vp, ctypes.c_int64, ctypes.c_int, vp, vp]
        L.qsa_oracle_attention_q8.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_int64, vp, vp]
        L.qsa_oracle_scores_q8.argtypes = [vp, vp, vp, vp, ctypes.c_int64, vp]
        L.qsa_oracle_attention_f64.argtypes = [vp, vp, vp, vp, ctypes.c_int64, vp, vp]
        L.qsa_oracle_attention_backward_f64.argtypes = [vp, vp, vp, vp, ctypes.c_int64, vp, vp, vp, vp]
        L.qsa_oracle_attention_backward.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int64, vp, vp, vp, vp]
        L.qsa_oracle_distill_target.argtypes = [vp, ctypes.c_int64, vp, vp, vp]
        L.qsa_oracle_distill_kl.restype = ctypes.c_double
        L.qsa_oracle_distill_kl.argtypes = [vp, vp, ctypes.c_int64, vp]
        L.qsa_oracle_round_bf16.argtypes = [vp, ctypes.c_int64, vp]

    @classmethod
    def for_workload(cls, w, **kw) -> "Oracle":
        return cls(r=w.r, K=w.K, idx_heads=w.idx_heads, idx_dim=w.idx_dim, rope_dims=w.rope_dims,
                   rope_base=w.rope_base, rms_eps=w.rms_eps, q_heads=w.q_heads,
                   kv_heads=w.kv_heads, head_dim=w.head_dim, **kw)

    # ------------------------------------------------------------------ steps
    @property
    def k_blocks(self) -> int:
        return int(self.lib.qsa_oracle_k_blocks(self._c))

    def round_bf16(self, x) -> np.ndarray:
        """The storage rounding (fp64 -> bf16 bits, nearest even)."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty(x.shape, dtype=np.uint16)
        self.lib.qsa_oracle_round_bf16(_p(x), x.size, _p(out))
        return out

    def rope(self, x: np.ndarray, pos: int) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty_like(x)
        c = self.cfg
        self.lib.qsa_oracle_rope(_p(x), x.size, c.rope_dims, c.rope_base, pos, _p(out))
        return out

    def pool_block(self, keys: np.ndarray, pos: int, w: Optional[np.ndarray] = None) -> dict:
        keys = _u16(keys)
        d = self.cfg.idx_dim
        kbar, knorm, krot = (np.empty(d) for _ in range(3))
        out = np.empty(d, dtype=np.uint16)
        w = None if w is None else np.ascontiguousarray(w, dtype=np.float32)
        self.lib.qsa_oracle_pool_block(self._c, _p(keys), _p(w), pos, _p(kbar), _p(knorm),
                                       _p(krot), _p(out))
        return {"kbar": kbar, "knorm": knorm, "krot": krot, "out": out}

    def compress(self, idx_k: np.ndarray, n_blocks: int, w: Optional[np.ndarray] = None) -> np.ndarray:
        idx_k = _u16(idx_k)
        assert idx_k.size >= n_blocks * self.cfg.r * self.cfg.idx_dim
        out = np.empty((n_blocks, self.cfg.idx_dim), dtype=np.uint16)
        w = None if w is None else np.ascontiguousarray(w, dtype=np.float32)
        self.lib.qsa_oracle_compress(self._c, _p(idx_k), n_blocks, _p(w), _p(out))
        return out

    def rotate_query(self, q: np.ndarray, pos: int) -> np.ndarray:
        q = _u16(q)
        out = np.empty((self.cfg.idx_heads, self.cfg.idx_dim), dtype=np.uint16)
        self.lib.qsa_oracle_rotate_query(self._c, _p(q), pos, _p(out))
        return out

    def scores(self, qrot: np.ndarray, pooled: np.ndarray, n_vis: int) -> np.ndarray:
        qrot, pooled = _u16(qrot), _u16(pooled)
        assert pooled.size >= n_vis * self.cfg.idx_dim
        out = np.empty(n_vis, dtype=np.float32)
        self.lib.qsa_oracle_scores(self._c, _p(qrot), _p(pooled), n_vis, _p(out))
        return out

    def select(self, scores: np.ndarray, k_b: Optional[int] = None) -> np.ndarray:
        scores = np.ascontiguousarray(scores, dtype=np.float32)
        k_b = self.k_blocks if k_b is None else k_b
        sel = np.empty(max(min(k_b, scores.size), 1), dtype=np.int32)
        m = self.lib.qsa_oracle_select(_p(scores), scores.size, k_b, _p(sel))
        return sel[:m].copy()

    def token_set(self, sel: np.ndarray, i: int) -> np.ndarray:
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        out = np.empty(sel.size * self.cfg.r + self.cfg.r, dtype=np.int64)
        n = self.lib.qsa_oracle_token_set(self._c, _p(sel), sel.size, i, _p(out))
        return out[:n].copy()

    def attention(self, q: np.ndarray, kc: np.ndarray, vc: np.ndarray, tokens: np.ndarray):
        q, kc, vc = _u16(q), _u16(kc), _u16(vc)
        tokens = np.ascontiguousarray(tokens, dtype=np.int64)
        c = self.cfg
        out = np.empty((c.q_heads, c.head_dim))
        lse = np.empty(c.q_heads)
        self.lib.qsa_oracle_attention(self._c, _p(q), _p(kc), _p(vc), _p(tokens), tokens.size,
                                      _p(out), _p(lse))
        return out, lse

    def row(self, i: int, idx_q_row: np.ndarray, pooled: np.ndarray, q_row=None, kc=None, vc=None,
            want_scores: bool = True) -> dict:
        """a3'..a7 for query position i. Attention is skipped when q_row is None."""
        c = self.cfg
        n_vis = i // c.r
        assert pooled.size >= n_vis * c.idx_dim
        # Padded with a sentinel: a row that scores more blocks than are visible is
        # reported, not a buffer overrun.
        scores = np.full(n_vis + c.r + 1, -7.0, dtype=np.float32) if want_scores else None
        sel = np.empty(max(self.k_blocks, 1), dtype=np.int32)
        out = lse = None
        if q_row is not None:
            out = np.empty((c.q_heads, c.head_dim))
            lse = np.empty(c.q_heads)
            q_row, kc, vc = _u16(q_row), _u16(kc), _u16(vc)
        m = self.lib.qsa_oracle_row(self._c, i, _p(_u16(idx_q_row)), _p(_u16(pooled)), _p(q_row),
                                    _p(kc), _p(vc), _p(scores), _p(sel), _p(out), _p(lse))
        res = {"sel": sel[:m].copy(), "nsel": int(m), "out": out, "lse": lse}
        if want_scores:
            assert (scores[n_vis:] == -7.0).all(), "scored blocks beyond floor(i/r)"
            res["scores"] = scores[:n_vis].copy()
        return res

    def decode_step(self, p: int, q_new, k_new, v_new, idx_q_new, idx_k_new, kc, vc, idx_k_cache,
                    pooled, w: Optional[np.ndarray] = None) -> dict:
        """a8 + a3'..a7 for the token at position p; updates the caches in place."""
        c = self.cfg
        for a in (kc, vc, idx_k_cache, pooled):
            assert a.flags.c_contiguous and a.dtype == np.uint16
        sel = np.empty(max(self.k_blocks, 1), dtype=np.int32)
        out = np.empty((c.q_heads, c.head_dim))
        lse = np.empty(c.q_heads)
        w = None if w is None else np.ascontiguousarray(w, dtype=np.float32)
        m = self.lib.qsa_oracle_decode_step(
            self._c, p, _p(_u16(q_new)), _p(_u16(k_new)), _p(_u16(v_new)), _p(_u16(idx_q_new)),
            _p(_u16(idx_k_new)), _p(kc), _p(vc), _p(idx_k_cache), _p(pooled), _p(w), _p(sel),
            _p(out), _p(lse))
        return {"sel": sel[:m].copy(), "nsel": int(m), "out": out, "lse": lse}

    # ------------------------------------------------ low-precision (fp8) caches
    def e4m3_value(self, code: int) -> float:
        return float(self.lib.qsa_oracle_e4m3_value(int(code) & 0xFF))

    def e4m3_encode(self, y: float) -> int:
        return int(self.lib.qsa_oracle_e4m3_encode(float(y)))

    def quant_rows(self, x: np.ndarray):
        """bf16 rows [..., dim] -> (E4M3 codes uint8 [..., dim], fp32 scales [...])."""
        x = _u16(x)
        dim = x.shape[-1]
        rows = x.size // dim
        codes = np.empty(x.shape, dtype=np.uint8)
        scales = np.empty(x.shape[:-1], dtype=np.float32)
        self.lib.qsa_oracle_quant_rows(_p(x), rows, dim, _p(codes), _p(scales))
        return codes, scales

    def dequant(self, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
        """E4M3(code) * scale in fp64, [..., dim]."""
        table = np.array([self.e4m3_value(c) for c in range(256)])
        return table[codes] * scales.astype(np.float64)[..., None]

    def attention_q8(self, q, kc, ks, vc, vs, tokens):
        q = _u16(q)
        kc, vc = (np.ascontiguousarray(a, dtype=np.uint8) for a in (kc, vc))
        ks, vs = (np.ascontiguousarray(a, dtype=np.float32) for a in (ks, vs))
        tokens = np.ascontiguousarray(tokens, dtype=np.int64)
        c = self.cfg
        out = np.empty((c.q_heads, c.head_dim))
        lse = np.empty(c.q_heads)
        self.lib.qsa_oracle_attention_q8(self._c, _p(q), _p(kc), _p(ks), _p(vc), _p(vs), _p(tokens), tokens.size,
                                         _p(out), _p(lse))
        return out, lse

    def scores_q8(self, qrot, pooled_codes, pooled_scales, n_vis: int) -> np.ndarray:
        qrot = _u16(qrot)
        pc = np.ascontiguousarray(pooled_codes, dtype=np.uint8)
        ps = np.ascontiguousarray(pooled_scales, dtype=np.float32)
        assert pc.size >= n_vis * self.cfg.idx_dim and ps.size >= n_vis
        out = np.empty(n_vis, dtype=np.float32)
        self.lib.qsa_oracle_scores_q8(self._c, _p(qrot), _p(pc), _p(ps), n_vis, _p(out))
        return out

    # ------------------------------------------------------------ training (f3)
    def attention_f64(self, q, kt, vt):
        """Sparse attention on fp64 operands: q [q_heads][d], kt, vt [ntok][kv_heads][d]
        (the listed tokens' rows in order) -> (out [q_heads][d], lse [q_heads])."""
        c = self.cfg
        q, kt, vt = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, kt, vt))
        ntok = kt.size // (c.kv_heads * c.head_dim)
        out = np.empty((c.q_heads, c.head_dim))
        lse = np.empty(c.q_heads)
        self.lib.qsa_oracle_attention_f64(self._c, _p(q), _p(kt), _p(vt), ntok, _p(out), _p(lse))
        return out, lse

    def attention_backward_f64(self, q, kt, vt, dout):
        """Gradient of attention_f64 for the upstream gradient dout [q_heads][d]:
        (dq [q_heads][d], dk [ntok][kv_heads][d], dv [ntok][kv_heads][d])."""
        c = self.cfg
        q, kt, vt, dout = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, kt, vt, dout))
        ntok = kt.size // (c.kv_heads * c.head_dim)
        dq = np.empty((c.q_heads, c.head_dim))
        dk = np.empty((ntok, c.kv_heads, c.head_dim))
        dv = np.empty((ntok, c.kv_heads, c.head_dim))
        self.lib.qsa_oracle_attention_backward_f64(self._c, _p(q), _p(kt), _p(vt), ntok, _p(dout), _p(dq),
                                                   _p(dk), _p(dv))
        return dq, dk, dv

    def attention_backward(self, q, kc, vc, tokens, dout):
        """The gradient on bf16 operands (as ``attention`` takes them); dk, dv hold
        one row per listed token."""
        c = self.cfg
        q, kc, vc, dout = _u16(q), _u16(kc), _u16(vc), _u16(dout)
        tokens = np.ascontiguousarray(tokens, dtype=np.int64)
        dq = np.empty((c.q_heads, c.head_dim))
        dk = np.empty((tokens.size, c.kv_heads, c.head_dim))
        dv = np.empty((tokens.size, c.kv_heads, c.head_dim))
        self.lib.qsa_oracle_attention_backward(self._c, _p(q), _p(kc), _p(vc), _p(tokens), tokens.size,
                                               _p(dout), _p(dq), _p(dk), _p(dv))
        return dq, dk, dv

    def distill_target(self, i: int, q, kc) -> np.ndarray:
        """Stage-1 target of query i over its floor(i/r) visible blocks (fp64)."""
        c = self.cfg
        n_vis = i // c.r
        q, kc = _u16(q), _u16(kc)
        assert kc.size >= (i + 1) * c.kv_heads * c.head_dim
        # Padded with a sentinel: writing past the visible blocks is reported.
        t = np.full(n_vis + c.r + 1, -7.0)
        self.lib.qsa_oracle_distill_target(self._c, i, _p(q), _p(kc), _p(t))
        assert (t[n_vis:] == -7.0).all(), "target written beyond floor(i/r)"
        return t[:n_vis].copy()

    def distill_kl(self, t, scores):
        """(KL(t || softmax(scores)), d KL / d scores) over the given blocks."""
        t = np.ascontiguousarray(t, dtype=np.float64)
        s = np.ascontiguousarray(scores, dtype=np.float32)
        ds = np.empty(t.size)
        kl = self.lib.qsa_oracle_distill_kl(_p(t), _p(s), t.size, _p(ds))
        return float(kl), ds
