"""Python binding of libqsa.so, the B200 (sm_100a) hot path of the QSA layer.

Thin argument marshalling over the C-ABI of ``include/qsa.h``: every function
below has the C entry point's name, takes torch tensors (device memory) and
passes their pointers plus the current CUDA stream. All computation happens in
the library's CUDA kernels; there is no fallback. The library is loaded on the
first call, which raises if it has not been built (``python -m
block_sparse_long_02_b200.build``).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqsa.so")

QSA_OK = 0
STATUS_NAMES = {0: "QSA_OK", 1: "QSA_ERR_INVALID_ARG", 2: "QSA_ERR_UNSUPPORTED", 3: "QSA_ERR_WORKSPACE",
                4: "QSA_ERR_CAPACITY", 5: "QSA_ERR_CUDA", 6: "QSA_ERR_TIMEOUT", 7: "QSA_ERR_DEVICE_CHECK"}
OP_INDEX_SCORES, OP_TOPK_BLOCKS, OP_SPARSE_ATTENTION, OP_DECODE_STEP, OP_DISTILL_TARGET = 0, 1, 2, 3, 4

EXPORTS = ["qsa_workspace_size", "qsa_compress_keys", "qsa_index_scores", "qsa_topk_blocks",
           "qsa_sparse_attention", "qsa_decode_step", "qsa_workspace_status", "qsa_last_error",
           "qsa_launch_count", "qsa_decode_step_noalloc", "qsa_set_fault_injection", "qsa_quantize_rows",
           "qsa_sparse_attention_q8", "qsa_decode_step_q8", "qsa_decode_step_offload",
           "qsa_sparse_attention_backward", "qsa_distill_target", "qsa_distill_kl", "qsa_set_attention_kernel",
           "qsa_index_scores_varlen", "qsa_topk_blocks_varlen", "qsa_sparse_attention_varlen",
           "qsa_set_decode_kernel"]


class QSAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class qsa_config(ctypes.Structure):
    _fields_ = [("r", ctypes.c_int32), ("K", ctypes.c_int32), ("idx_heads", ctypes.c_int32),
                ("idx_dim", ctypes.c_int32), ("rope_dims", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("rms_eps", ctypes.c_double), ("q_heads", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("sm_scale", ctypes.c_double)]


@dataclasses.dataclass
class Config:
    """The layer as the pages state it (r = 4, K = 2048, 4 x 128 indexer, ...)."""

    r: int = 4
    K: int = 2048
    idx_heads: int = 4
    idx_dim: int = 128
    rope_dims: int = 64
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    q_heads: int = 32
    kv_heads: int = 4
    head_dim: int = 128
    sm_scale: float = 0.0

    @property
    def k_blocks(self) -> int:
        return -(-self.K // self.r)

    def c(self) -> qsa_config:
        return qsa_config(self.r, self.K, self.idx_heads, self.idx_dim, self.rope_dims, self.rope_base,
                          self.rms_eps, self.q_heads, self.kv_heads, self.head_dim, self.sm_scale)

    @classmethod
    def of(cls, w) -> "Config":
        """From any object with the same attribute names (e.g. a synth.Workload)."""
        return cls(**{f.name: getattr(w, f.name) for f in dataclasses.fields(cls) if hasattr(w, f.name)})


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_CFG = ctypes.POINTER(qsa_config)
_SIGS = {
    "qsa_workspace_size": [_CFG, _i32, _i32, _i64, _i64, ctypes.POINTER(_sz)],
    "qsa_compress_keys": [_CFG, _i32, _vp, _i64, _vp, _i64, _i64, _vp, _vp],
    "qsa_index_scores": [_CFG, _i32, _vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _sz, _vp],
    "qsa_topk_blocks": [_CFG, _i32, _vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _vp, _vp, _sz, _vp],
    "qsa_sparse_attention": [_CFG, _i32, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "qsa_decode_step": [_CFG, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp,
                        _vp, _vp, _sz, _vp],
    "qsa_workspace_status": [_vp, _vp, ctypes.POINTER(_i32)],
    "qsa_sparse_attention_backward": [_CFG, _i32, _vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _vp, _vp, _vp],
    "qsa_distill_target": [_CFG, _i32, _vp, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _sz, _vp],
    "qsa_distill_kl": [_CFG, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp],
    "qsa_quantize_rows": [_vp, _i64, _i32, _vp, _vp, _vp],
    "qsa_decode_step_q8": [_CFG, _i32] + [_vp] * 14 + [_i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "qsa_decode_step_offload": [_CFG, _i32] + [_vp] * 11 + [_i64, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz,
                                                           _vp],
    "qsa_sparse_attention_q8": [_CFG, _i32, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp,
                                _sz, _vp],
    "qsa_index_scores_varlen": [_CFG, _i32, _vp, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _sz, _vp],
    "qsa_topk_blocks_varlen": [_CFG, _i32, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _sz, _vp],
    "qsa_sparse_attention_varlen": [_CFG, _i32, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "qsa_decode_step_noalloc": [_CFG, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp,
                                _vp, _vp, _vp],
}
_lib_handle = None


def lib() -> ctypes.CDLL:
    """The loaded libqsa.so (loaded on first use). Raises if it was not built:
    there is no other implementation to fall back to."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_long_02_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(h, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        h.qsa_last_error.restype = ctypes.c_char_p
        h.qsa_last_error.argtypes = []
        h.qsa_launch_count.restype = ctypes.c_uint64
        h.qsa_launch_count.argtypes = []
        h.qsa_set_fault_injection.restype = ctypes.c_int
        h.qsa_set_fault_injection.argtypes = [ctypes.c_int32, ctypes.c_double]
        h.qsa_set_attention_kernel.restype = ctypes.c_int
        h.qsa_set_attention_kernel.argtypes = [ctypes.c_int32]
        h.qsa_set_decode_kernel.restype = ctypes.c_int
        h.qsa_set_decode_kernel.argtypes = [ctypes.c_int32]
        _lib_handle = h
    return _lib_handle


def _check(status: int) -> None:
    if status != QSA_OK:
        raise QSAError(status, lib().qsa_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to libqsa must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libqsa must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t: torch.Tensor):
    """Address of a pinned host tensor (the library checks that it is mapped
    into the device address space)."""
    if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
        raise ValueError("host caches must be contiguous pinned CPU tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def qsa_workspace_size(cfg: Config, op: int, batch: int, cap: int, nq: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().qsa_workspace_size(ctypes.byref(cfg.c()), op, batch, cap, nq, ctypes.byref(out)))
    return out.value


def workspace(cfg: Config, op: int, batch: int, cap: int, nq: int = 0, device=None) -> torch.Tensor:
    """A zero-initialised workspace of the size qsa_workspace_size reports."""
    n = qsa_workspace_size(cfg, op, batch, cap, nq)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def qsa_compress_keys(cfg: Config, batch: int, idx_k: torch.Tensor, cap: int, rms_w, blk_begin: int,
                      blk_end: int, pooled: torch.Tensor, stream=None) -> None:
    _check(lib().qsa_compress_keys(ctypes.byref(cfg.c()), batch, _ptr(idx_k), cap, _ptr(rms_w), blk_begin,
                                  blk_end, _ptr(pooled), _stream(stream)))


def qsa_index_scores(cfg: Config, batch: int, idx_q: torch.Tensor, q_begin: int, nq: int,
                     pooled: torch.Tensor, cap: int, scores: torch.Tensor, ld: int, ws: torch.Tensor,
                     stream=None) -> None:
    _check(lib().qsa_index_scores(ctypes.byref(cfg.c()), batch, _ptr(idx_q), q_begin, nq, _ptr(pooled), cap,
                                 _ptr(scores), ld, _ptr(ws), ws.numel(), _stream(stream)))


def qsa_topk_blocks(cfg: Config, batch: int, idx_q, q_begin: int, nq: int, pooled, cap: int,
                    scores: Optional[torch.Tensor], ld: int, sel: torch.Tensor, nsel: torch.Tensor,
                    ws: Optional[torch.Tensor], stream=None) -> None:
    _check(lib().qsa_topk_blocks(ctypes.byref(cfg.c()), batch, _ptr(idx_q), q_begin, nq, _ptr(pooled), cap,
                                _ptr(scores), ld, _ptr(sel), _ptr(nsel), _ptr(ws),
                                0 if ws is None else ws.numel(), _stream(stream)))


def qsa_sparse_attention(cfg: Config, batch: int, q: torch.Tensor, q_begin: int, nq: int,
                         k_cache: torch.Tensor, v_cache: torch.Tensor, cap: int, sel: torch.Tensor,
                         nsel: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                         ws: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().qsa_sparse_attention(ctypes.byref(cfg.c()), batch, _ptr(q), q_begin, nq, _ptr(k_cache),
                                     _ptr(v_cache), cap, _ptr(sel), _ptr(nsel), _ptr(out), _ptr(lse),
                                     _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def _host_i64(values) -> ctypes.Array:
    return (ctypes.c_int64 * len(values))(*[int(v) for v in values])


def qsa_index_scores_varlen(cfg: Config, idx_q: torch.Tensor, q_begin, nq, pooled: torch.Tensor, cap: int,
                            scores: torch.Tensor, ld: int, ws: torch.Tensor, stream=None) -> None:
    """Per-sequence query ranges (q_begin[s], nq[s]: host lists), queries packed."""
    _check(lib().qsa_index_scores_varlen(ctypes.byref(cfg.c()), len(nq), _ptr(idx_q), _host_i64(q_begin),
                                         _host_i64(nq), _ptr(pooled), cap, _ptr(scores), ld, _ptr(ws), ws.numel(),
                                         _stream(stream)))


def qsa_topk_blocks_varlen(cfg: Config, idx_q: torch.Tensor, q_begin, nq, pooled: torch.Tensor, cap: int,
                           sel: torch.Tensor, nsel: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check(lib().qsa_topk_blocks_varlen(ctypes.byref(cfg.c()), len(nq), _ptr(idx_q), _host_i64(q_begin),
                                        _host_i64(nq), _ptr(pooled), cap, _ptr(sel), _ptr(nsel), _ptr(ws),
                                        ws.numel(), _stream(stream)))


def qsa_sparse_attention_varlen(cfg: Config, q: torch.Tensor, q_begin, nq, k_cache: torch.Tensor,
                                v_cache: torch.Tensor, cap: int, sel: torch.Tensor, nsel: torch.Tensor,
                                out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                                ws: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().qsa_sparse_attention_varlen(ctypes.byref(cfg.c()), len(nq), _ptr(q), _host_i64(q_begin),
                                             _host_i64(nq), _ptr(k_cache), _ptr(v_cache), cap, _ptr(sel),
                                             _ptr(nsel), _ptr(out), _ptr(lse), _ptr(ws),
                                             0 if ws is None else ws.numel(), _stream(stream)))


def qsa_sparse_attention_backward(cfg: Config, batch: int, q: torch.Tensor, q_begin: int, nq: int,
                                  k_cache: torch.Tensor, v_cache: torch.Tensor, cap: int, sel: torch.Tensor,
                                  nsel: torch.Tensor, out: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor,
                                  dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor, stream=None) -> None:
    """Gradient of qsa_sparse_attention: dq written, dk and dv added to (see include/qsa.h)."""
    _check(lib().qsa_sparse_attention_backward(ctypes.byref(cfg.c()), batch, _ptr(q), q_begin, nq, _ptr(k_cache),
                                              _ptr(v_cache), cap, _ptr(sel), _ptr(nsel), _ptr(out), _ptr(lse),
                                              _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream)))


def qsa_distill_target(cfg: Config, batch: int, q: torch.Tensor, q_begin: int, nq: int, k_cache: torch.Tensor,
                       cap: int, target: torch.Tensor, ld: int, ws: torch.Tensor, stream=None) -> None:
    """Stage-1 distillation target (see include/qsa.h)."""
    _check(lib().qsa_distill_target(ctypes.byref(cfg.c()), batch, _ptr(q), q_begin, nq, _ptr(k_cache), cap,
                                   _ptr(target), ld, _ptr(ws), ws.numel(), _stream(stream)))


def qsa_distill_kl(cfg: Config, batch: int, q_begin: int, nq: int, target: torch.Tensor, scores: torch.Tensor,
                   ld: int, kl: torch.Tensor, dscores: Optional[torch.Tensor] = None, stream=None) -> None:
    """KL(target || softmax(scores)) per query and its gradient (see include/qsa.h)."""
    _check(lib().qsa_distill_kl(ctypes.byref(cfg.c()), batch, q_begin, nq, _ptr(target), _ptr(scores), ld,
                               _ptr(kl), _ptr(dscores), _stream(stream)))


def qsa_quantize_rows(x: torch.Tensor, rows: int, dim: int, codes: torch.Tensor, scales: torch.Tensor,
                      stream=None) -> None:
    """FP8 E4M3 rows with one fp32 scale per row (see include/qsa.h)."""
    _check(lib().qsa_quantize_rows(_ptr(x), rows, dim, _ptr(codes), _ptr(scales), _stream(stream)))


def qsa_sparse_attention_q8(cfg: Config, batch: int, q: torch.Tensor, q_begin: int, nq: int,
                            k_codes: torch.Tensor, k_scales: torch.Tensor, v_codes: torch.Tensor,
                            v_scales: torch.Tensor, cap: int, sel: torch.Tensor, nsel: torch.Tensor,
                            out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                            ws: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().qsa_sparse_attention_q8(ctypes.byref(cfg.c()), batch, _ptr(q), q_begin, nq, _ptr(k_codes),
                                        _ptr(k_scales), _ptr(v_codes), _ptr(v_scales), cap, _ptr(sel), _ptr(nsel),
                                        _ptr(out), _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel(),
                                        _stream(stream)))


def qsa_decode_step_q8(cfg: Config, batch: int, pos, q, k, v, idx_q, idx_k, k_codes, k_scales, v_codes, v_scales,
                       idx_k_cache, pooled, pooled_codes, pooled_scales, cap: int, rms_w, out, sel_out=None,
                       nsel_out=None, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().qsa_decode_step_q8(ctypes.byref(cfg.c()), batch, _ptr(pos), _ptr(q), _ptr(k), _ptr(v), _ptr(idx_q),
                                   _ptr(idx_k), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales),
                                   _ptr(idx_k_cache), _ptr(pooled), _ptr(pooled_codes), _ptr(pooled_scales), cap,
                                   _ptr(rms_w), _ptr(out), _ptr(sel_out), _ptr(nsel_out), _ptr(ws),
                                   0 if ws is None else ws.numel(), _stream(stream)))


def qsa_decode_step_offload(cfg: Config, batch: int, pos, q, k, v, idx_q, idx_k, host_k_cache, host_v_cache,
                            hot_k, hot_v, hot_tags, hot_blocks: int, idx_k_cache, pooled, cap: int, rms_w, out,
                            sel_out=None, nsel_out=None, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().qsa_decode_step_offload(ctypes.byref(cfg.c()), batch, _ptr(pos), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(idx_q), _ptr(idx_k), _host_ptr(host_k_cache), _host_ptr(host_v_cache),
                                        _ptr(hot_k),
                                        _ptr(hot_v), _ptr(hot_tags), hot_blocks, _ptr(idx_k_cache), _ptr(pooled), cap,
                                        _ptr(rms_w), _ptr(out), _ptr(sel_out), _ptr(nsel_out), _ptr(ws),
                                        0 if ws is None else ws.numel(), _stream(stream)))


def qsa_decode_step(cfg: Config, batch: int, pos: torch.Tensor, q, k, v, idx_q, idx_k, k_cache, v_cache,
                    idx_k_cache, pooled, cap: int, rms_w, out, sel_out=None, nsel_out=None,
                    ws: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().qsa_decode_step(ctypes.byref(cfg.c()), batch, _ptr(pos), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(idx_q), _ptr(idx_k), _ptr(k_cache), _ptr(v_cache), _ptr(idx_k_cache),
                                _ptr(pooled), cap, _ptr(rms_w), _ptr(out), _ptr(sel_out), _ptr(nsel_out),
                                _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def qsa_decode_step_noalloc(cfg: Config, batch: int, pos: torch.Tensor, q, k, v, idx_q, idx_k, k_cache,
                            v_cache, idx_k_cache, pooled, cap: int, rms_w, out, sel_out=None, nsel_out=None,
                            stream=None) -> None:
    """qsa_decode_step for callers that cannot allocate: no workspace argument;
    the library's fixed 16 MiB device scratch is used instead (see qsa.h)."""
    _check(lib().qsa_decode_step_noalloc(ctypes.byref(cfg.c()), batch, _ptr(pos), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(idx_q), _ptr(idx_k), _ptr(k_cache), _ptr(v_cache),
                                         _ptr(idx_k_cache), _ptr(pooled), cap, _ptr(rms_w), _ptr(out),
                                         _ptr(sel_out), _ptr(nsel_out), _stream(stream)))


def qsa_workspace_status(ws: torch.Tensor, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(lib().qsa_workspace_status(_ptr(ws), _stream(stream), ctypes.byref(out)))
    return out.value


def qsa_last_error() -> str:
    return lib().qsa_last_error().decode()


def qsa_launch_count() -> int:
    """Kernel launches issued by libqsa.so so far in this process."""
    return int(lib().qsa_launch_count())


ATTENTION_WARP, ATTENTION_TCGEN05 = 0, 1


def qsa_set_attention_kernel(kernel: int) -> None:
    """Kernel of qsa_sparse_attention on bf16 caches: ATTENTION_WARP (default)
    or ATTENTION_TCGEN05 (see qsa.h)."""
    _check(lib().qsa_set_attention_kernel(int(kernel)))


DECODE_STEP_KERNEL, DECODE_THREE_KERNELS = 0, 1


def qsa_set_decode_kernel(kernel: int) -> None:
    """Kernels of a decode step: DECODE_STEP_KERNEL (one persistent kernel) or
    DECODE_THREE_KERNELS (the default; see qsa.h)."""
    _check(lib().qsa_set_decode_kernel(int(kernel)))


def qsa_set_fault_injection(mode: int, wait_seconds: float = 0.0) -> None:
    """Tests of the failure path only (see include/qsa.h): mode 1 makes the fused
    top-k's bounded wait run out after wait_seconds; mode 0 restores normal use."""
    _check(lib().qsa_set_fault_injection(int(mode), float(wait_seconds)))
