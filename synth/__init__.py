"""Seeded synthetic QSA workloads: the one module both the oracle and the CUDA path use.

It draws inputs and plants needles; it holds none of the layer's arithmetic (no
pooling, normalisation, rotation, scoring, selection or attention). The
generator itself is defined in ``gen_host.c`` and mirrored bit for bit on the
GPU by ``gen_device.cu``.

Logical tensors of one sequence (row-major; ``T`` = total positions drawn):

=========  ======================  =========
name       logical shape           tensor id
=========  ======================  =========
idx_q      [T][idx_heads][idx_dim]  1
idx_k      [T][idx_dim]             2
q          [T][q_heads][head_dim]   3
k          [T][kv_heads][head_dim]  4
v          [T][kv_heads][head_dim]  5
=========  ======================  =========

Sequence ``s`` of a batch uses seed ``base_seed + s * 2**32``.

Needles (input construction, stated as a reading of "keys are the query
direction x4"): for a needle block ``b`` probed by position ``p``, let ``u`` be
the unit vector of sum_h idx_q[p][h][64:128]. All ``r`` raw indexer keys of the
block become ``[0]*64 + 32*u`` (4x a unit-variance vector along ``u``), rounded
to bf16. Dims 64..127 are the ones partial RoPE leaves untouched, so the
needle's score against its probe does not depend on the two positions.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "libsynth_host.so")
_DEV_SO = os.path.join(_HERE, "libsynth_device.so")

TENSOR_IDS = {"idx_q": 1, "idx_k": 2, "q": 3, "k": 4, "v": 5, "dout": 6}  # dout: an upstream gradient of out


# ----------------------------------------------------------------------------- build / load
def build(force: bool = False) -> None:
    """Compile the host generator (gcc) and the device generator (nvcc, sm_100a)."""
    src_h = os.path.join(_HERE, "gen_host.c")
    if force or not os.path.exists(_HOST_SO) or os.path.getmtime(_HOST_SO) < os.path.getmtime(src_h):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _HOST_SO, src_h])
    src_d = os.path.join(_HERE, "gen_device.cu")
    if force or not os.path.exists(_DEV_SO) or os.path.getmtime(_DEV_SO) < os.path.getmtime(src_d):
        subprocess.check_call(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
                               "-shared", "-Xcompiler", "-fPIC", "-o", _DEV_SO, src_d])


_host_lib = None
_dev_lib = None


def _host():
    global _host_lib
    if _host_lib is None:
        if not os.path.exists(_HOST_SO):
            build()
        lib = ctypes.CDLL(_HOST_SO)
        lib.synth_fill_host.argtypes = [ctypes.c_uint64] * 4 + [ctypes.c_void_p]
        lib.synth_fill_host.restype = None
        lib.synth_fill_rows_host.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p,
                                             ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_fill_rows_host.restype = None
        _host_lib = lib
    return _host_lib


def _dev():
    global _dev_lib
    if _dev_lib is None:
        if not os.path.exists(_DEV_SO):
            build()
        lib = ctypes.CDLL(_DEV_SO)
        lib.synth_fill_device.argtypes = [ctypes.c_uint64] * 4 + [ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_fill_device.restype = ctypes.c_int
        _dev_lib = lib
    return _dev_lib


# ----------------------------------------------------------------------------- bf16 helpers
def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


# ----------------------------------------------------------------------------- raw draws
def fill_host(seed: int, tensor_id: int, e0: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.uint16)
    if count:
        _host().synth_fill_host(seed & (2**64 - 1), tensor_id, e0, count, out.ctypes.data)
    return out


def fill_rows_host(seed: int, tensor_id: int, rows: Sequence[int], row_len: int) -> np.ndarray:
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((rows.size, row_len), dtype=np.uint16)
    if rows.size:
        _host().synth_fill_rows_host(seed & (2**64 - 1), tensor_id, rows.ctypes.data, rows.size,
                                     row_len, out.ctypes.data)
    return out


def fill_device(seed: int, tensor_id: int, e0: int, count: int, ptr: int, stream: int = 0) -> None:
    rc = _dev().synth_fill_device(seed & (2**64 - 1), tensor_id, e0, count, ctypes.c_void_p(ptr),
                                  ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_device failed with cudaError {rc}")


# ----------------------------------------------------------------------------- workloads
@dataclasses.dataclass
class Workload:
    """One synthetic QSA workload (shapes follow the layer as the pages state it)."""

    name: str
    n: int                      # prefill length, or tokens already cached before decoding
    batch: int = 1
    decode_steps: int = 0       # new tokens decoded after the first n positions
    prefill: bool = True        # every position in [q_begin, n) is a query
    q_begin: int = 0            # positions before it form an existing cache (chunked prefill)
    r: int = 4
    K: int = 2048
    idx_heads: int = 4
    idx_dim: int = 128
    q_heads: int = 32
    kv_heads: int = 4
    head_dim: int = 128
    rope_dims: int = 64
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    base_seed: int = 0
    n_needles_prefill: int = 0  # per sequence, probes drawn among prefill positions
    n_needles_decode: int = 0   # per sequence; probes are decode positions (cycled)
    train: bool = False         # the prefill also runs the training kernels (upstream gradient "dout")

    @property
    def k_blocks(self) -> int:
        return -(-self.K // self.r)

    @property
    def total(self) -> int:
        return self.n + self.decode_steps

    def seed(self, seq: int) -> int:
        return (self.base_seed + (seq << 32)) & (2**64 - 1)

    def row_len(self, name: str) -> int:
        return {"idx_q": self.idx_heads * self.idx_dim, "idx_k": self.idx_dim,
                "q": self.q_heads * self.head_dim, "k": self.kv_heads * self.head_dim,
                "v": self.kv_heads * self.head_dim, "dout": self.q_heads * self.head_dim}[name]

    # -- needles ---------------------------------------------------------------
    def needles(self, seq: int) -> List[Tuple[int, int]]:
        """(block, probe position) pairs of sequence ``seq``; blocks are disjoint."""
        rng = np.random.Generator(np.random.PCG64(self.seed(seq) ^ 0x4E454544))
        out: List[Tuple[int, int]] = []
        used = set()
        n_blocks = self.n // self.r
        for j in range(self.n_needles_decode):
            probe = self.n + (j % max(self.decode_steps, 1))
            while True:
                b = int(rng.integers(0, n_blocks))
                if b not in used:
                    break
            used.add(b)
            out.append((b, probe))
        for _ in range(self.n_needles_prefill):
            while True:
                b = int(rng.integers(0, n_blocks - 1))
                if b not in used:
                    break
            used.add(b)
            probe = int(rng.integers(self.r * (b + 1), self.n))
            out.append((b, probe))
        return out

    def needle_rows(self, seq: int) -> Dict[int, np.ndarray]:
        """Raw idx_k rows (bf16 bits) that the needles replace, keyed by position."""
        rows: Dict[int, np.ndarray] = {}
        nd = self.needles(seq)
        if not nd:
            return rows
        probes = sorted({p for _, p in nd})
        qrows = fill_rows_host(self.seed(seq), TENSOR_IDS["idx_q"], probes, self.row_len("idx_q"))
        qf = bf16_bits_to_f32(qrows).astype(np.float64).reshape(len(probes), self.idx_heads, self.idx_dim)
        direction = {}
        half = self.idx_dim - self.rope_dims
        for k, p in enumerate(probes):
            u = qf[k, :, self.rope_dims:].sum(axis=0)
            u = u / np.linalg.norm(u)
            row = np.zeros(self.idx_dim, dtype=np.float32)
            row[self.rope_dims:] = (4.0 * np.sqrt(half) * u).astype(np.float32)
            direction[p] = f32_to_bf16_bits(row)
        for b, p in nd:
            for t in range(self.r * b, self.r * b + self.r):
                rows[t] = direction[p]
        return rows

    # -- host tensors ----------------------------------------------------------
    def host_rows(self, name: str, seq: int, rows: Sequence[int]) -> np.ndarray:
        """bf16 bits [len(rows)][row_len] of a logical tensor, needles applied."""
        out = fill_rows_host(self.seed(seq), TENSOR_IDS[name], rows, self.row_len(name))
        if name == "idx_k":
            nr = self.needle_rows(seq)
            for k, t in enumerate(np.asarray(rows, dtype=np.int64).tolist()):
                if t in nr:
                    out[k] = nr[t]
        return out

    def host_full(self, name: str, seq: int, T: Optional[int] = None) -> np.ndarray:
        T = self.total if T is None else T
        L = self.row_len(name)
        out = fill_host(self.seed(seq), TENSOR_IDS[name], 0, T * L).reshape(T, L)
        if name == "idx_k":
            for t, row in self.needle_rows(seq).items():
                if t < T:
                    out[t] = row
        return out

    # -- device tensors --------------------------------------------------------
    def device_fill(self, name: str, tensor, rows: Tuple[int, int] = None, stream: int = 0) -> None:
        """Fill ``tensor`` ([batch][cap][row_len] bf16 on a CUDA device) with logical
        rows [r0, r1) of every sequence (default [0, total)), needles applied."""
        import torch  # plumbing only

        r0, r1 = rows if rows is not None else (0, self.total)
        L = self.row_len(name)
        t = tensor.view(tensor.shape[0], -1, L) if tensor.dim() != 3 or tensor.shape[-1] != L else tensor
        assert t.is_contiguous() and t.dtype == torch.bfloat16
        # Rows are absolute: the tensor must hold rows [0, r1) of each sequence.
        if not 0 <= r0 <= r1 <= t.shape[1]:
            raise ValueError(f"rows [{r0}, {r1}) outside a tensor of {t.shape[1]} rows")
        for s in range(t.shape[0]):
            dst = t[s, r0:r1]
            fill_device(self.seed(s), TENSOR_IDS[name], r0 * L, (r1 - r0) * L, dst.data_ptr(), stream)
            if name == "idx_k":
                nr = self.needle_rows(s)
                sel = sorted(p for p in nr if r0 <= p < r1)
                if sel:
                    vals = torch.from_numpy(np.stack([nr[p] for p in sel]).view(np.int16))
                    idx = torch.tensor([p - r0 for p in sel], dtype=torch.long)
                    dst.view(torch.int16)[idx.to(dst.device)] = vals.to(dst.device)


def _w(**kw) -> Workload:
    return Workload(**kw)


# The workloads the layer is measured on (contexts of 32K, ~261K and 1M tokens).
WORKLOADS: Dict[str, Workload] = {
    "tiny_prefill_n256": _w(name="tiny_prefill_n256", n=256, K=32, q_heads=4, kv_heads=1,
                            base_seed=0x51534101),
    "decode_b1_n32k": _w(name="decode_b1_n32k", n=32768, decode_steps=1, prefill=False,
                         base_seed=0x51534102, n_needles_decode=16),
    "prefill_n128k": _w(name="prefill_n128k", n=131072, base_seed=0x51534103, n_needles_prefill=64),
    "decode_b8_n256k": _w(name="decode_b8_n256k", n=262144, batch=8, decode_steps=1, prefill=False,
                          base_seed=0x51534104, n_needles_decode=32),
    "prefill_n1m_decode64": _w(name="prefill_n1m_decode64", n=1048576, decode_steps=64,
                               base_seed=0x51534105, n_needles_prefill=64, n_needles_decode=64),
    # Chunked prefill against an existing cache: the last 8192 positions of a 1M context.
    "prefill_chunk8k_n1m": _w(name="prefill_chunk8k_n1m", n=1048576, q_begin=1048576 - 8192,
                              base_seed=0x51534106),
    # One training step of the layer on a 32K sequence: the prefill forward, the
    # sparse-attention gradient and the stage-1 distillation target and loss.
    "train_n32k": _w(name="train_n32k", n=32768, base_seed=0x51534107, train=True),
}
