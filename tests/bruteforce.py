"""Dense brute-force restatement of the QSA layer for tiny inputs (test-only).

It is deliberately formulated differently from the oracle, so that agreement
between the two pins the oracle:
  - RoPE as complex multiplication z_j * exp(i * pos * theta_j), with the pair
    (x_j, x_{j+half}) read as z_j = x_j + i x_{j+half} (textbook RoFormer form);
  - pooling/normalisation as numpy reductions over the whole key tensor;
  - scores as one einsum over all (query, head, block) triples;
  - selection with numpy's lexsort;
  - attention as a dense [n x n] softmax under a boolean mask built from the
    selection and the tail, instead of a gather of the token set.
Only small n (a few hundred) is meant to run here.
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


_BF16_TABLE = None


def _bf16_table():
    """Every non-negative bf16 pattern 0x0000 .. 0x7F80 (+inf) and its value,
    increasing. The value used for +inf is 2^128, the grid point one step
    past the largest finite bf16, so that rounding to it means overflow."""
    global _BF16_TABLE
    if _BF16_TABLE is None:
        pat = np.arange(0x7F81, dtype=np.uint32)
        val = (pat << np.uint32(16)).view(np.float32).astype(np.float64)
        val[-1] = 2.0 ** 128
        _BF16_TABLE = (pat.astype(np.uint16), val)
    return _BF16_TABLE


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 to bf16 bits as the nearest bf16 value, ties to the even
    pattern: a search over the table of all bf16 values (no bit tricks)."""
    x = np.asarray(x, dtype=np.float64)
    pat, val = _bf16_table()
    a = np.abs(x).ravel()
    hi = np.clip(np.searchsorted(val, a, side="left"), 0, val.size - 1)
    lo = np.clip(hi - 1, 0, None)
    mid = val[lo] + val[hi]          # exact: two 8-bit significands
    twice = 2.0 * a                  # exact
    pick = np.where(twice < mid, lo, np.where(twice > mid, hi, np.where(pat[lo] % 2 == 0, lo, hi)))
    pick = np.where(val[hi] == a, hi, pick)
    out = pat[pick].astype(np.uint16)
    out = np.where(np.signbit(x.ravel()), out | np.uint16(0x8000), out).astype(np.uint16)
    return out.reshape(x.shape)


def rope_complex(x: np.ndarray, pos: np.ndarray, rope_dims: int, base: float) -> np.ndarray:
    """x: [..., dim] fp64, pos broadcastable to x.shape[:-1]."""
    half = rope_dims // 2
    theta = base ** (-2.0 * np.arange(half) / rope_dims)
    z = x[..., :half] + 1j * x[..., half:rope_dims]
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * theta)
    out = x.copy()
    out[..., :half] = z.real
    out[..., half:rope_dims] = z.imag
    return out


def layer(w, idx_q, idx_k, q, k, v, K=None, rms_w=None):
    """Whole prefill of one sequence. Arrays are bf16 bits shaped
    idx_q [n][Hi][Di], idx_k [n][Di], q [n][Hq][d], k/v [n][Hkv][d]."""
    n = idx_k.shape[0]
    r = w.r
    K = w.K if K is None else K
    kB = -(-K // r)
    nb = n // r
    kf = bf16_to_f64(idx_k)
    kbar = kf[: nb * r].reshape(nb, r, -1).mean(axis=1)
    knorm = kbar / np.sqrt((kbar**2).mean(axis=-1, keepdims=True) + w.rms_eps)
    if rms_w is not None:
        knorm = knorm * np.asarray(rms_w, dtype=np.float64)
    khat_bits = f64_to_bf16(rope_complex(knorm, r * np.arange(nb), w.rope_dims, w.rope_base))
    qrot_bits = f64_to_bf16(rope_complex(bf16_to_f64(idx_q), np.arange(n)[:, None], w.rope_dims,
                                         w.rope_base))
    dots = np.einsum("ihd,bd->ihb", bf16_to_f64(qrot_bits), bf16_to_f64(khat_bits))
    scores = np.maximum(dots, 0.0).sum(axis=1).astype(np.float32)  # [n][nb]
    block_sel = np.zeros((n, nb), dtype=bool)
    for i in range(n):
        c = i // r
        if c == 0:
            continue
        s = scores[i, :c]
        order = np.lexsort((np.arange(c), -s.astype(np.float64)))
        block_sel[i, order[:kB]] = True
    t = np.arange(n)
    tok_block = t // r
    mask = block_sel[:, tok_block] | ((tok_block[None, :] == (t // r)[:, None]) & (t[None, :] <= t[:, None]))
    qf, kf2, vf = bf16_to_f64(q), bf16_to_f64(k), bf16_to_f64(v)
    g = q.shape[1] // k.shape[1]
    kx = np.repeat(kf2, g, axis=1)
    vx = np.repeat(vf, g, axis=1)
    logits = np.einsum("ihd,thd->iht", qf, kx) / np.sqrt(q.shape[2])
    logits = np.where(mask[:, None, :], logits, -np.inf)
    m = logits.max(axis=-1, keepdims=True)
    p = np.exp(logits - m)
    z = p.sum(axis=-1, keepdims=True)
    out = np.einsum("iht,thd->ihd", p / z, vx)
    lse = (m + np.log(z))[..., 0]
    return {"pooled": khat_bits, "qrot": qrot_bits, "scores": scores, "block_sel": block_sel,
            "mask": mask, "out": out, "lse": lse}
