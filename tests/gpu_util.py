"""Shared helpers of the GPU parity tests: inputs from synth on both sides, the
oracle on the host, the CUDA path through the C-ABI binding, and the parity
rules (written out here once, used by every test)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

# Parity rules.
SCORE_RTOL = 1e-3        # indexer scores: relative
SCORE_COND_ATOL = 1e-5   # ... plus this times sum_h sum_j |q_j^h k_bj| (fp32 accumulation scale)
ATTN_ATOL = 2e-2         # attention output vs the fp64 oracle on the same selection (max-abs)
LSE_ATOL = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32(b: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(b)


def dev_full(w, name: str, cap: int, T: int = None) -> torch.Tensor:
    """[batch][cap][row_len] bf16 with logical rows [0, T) drawn on the device."""
    T = min(cap, w.total) if T is None else T
    t = torch.zeros(w.batch, cap, w.row_len(name), dtype=torch.bfloat16, device="cuda")
    w.device_fill(name, t, rows=(0, T))
    return t


def score_tol(qrot_bits: np.ndarray, pooled_bits: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per-block tolerance of an indexer score row."""
    qa = np.abs(f32(qrot_bits).astype(np.float64))          # [4][128]
    ka = np.abs(f32(pooled_bits[: ref.size]).astype(np.float64))  # [n][128]
    cond = (ka @ qa.T).sum(axis=1)
    return SCORE_RTOL * np.abs(ref.astype(np.float64)) + SCORE_COND_ATOL * cond


def check_scores(got: np.ndarray, ref: np.ndarray, tol: np.ndarray, what=""):
    d = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    bad = np.nonzero(d > tol)[0]
    assert bad.size == 0, f"{what}: {bad.size} scores out of tolerance, first {bad[:5]}, d={d[bad[:5]]}, tol={tol[bad[:5]]}"


def check_selection(got_row: np.ndarray, got_n: int, ref_scores: np.ndarray, tol: np.ndarray, kB: int,
                    what=""):
    """Selected block sets must be equal as sets, except for swaps between blocks
    whose reference scores lie within tolerance of the k-th reference score."""
    n_vis = ref_scores.size
    m = min(kB, n_vis)
    assert got_n == m, f"{what}: nsel {got_n} != {m}"
    sel = got_row[:m]
    assert (got_row[m:] == -1).all(), f"{what}: padding"
    assert np.all(np.diff(sel) > 0), f"{what}: not strictly ascending"
    if m == 0:
        return
    assert sel.min() >= 0 and sel.max() < n_vis, f"{what}: out of range"
    order = np.lexsort((np.arange(n_vis), -ref_scores.astype(np.float64)))
    ref = set(order[:m].tolist())
    diff = set(sel.tolist()) ^ ref
    if not diff:
        return
    k = order[m - 1]
    kth = float(ref_scores[k])
    for b in diff:
        lim = tol[b] + tol[k]
        assert abs(float(ref_scores[b]) - kth) <= lim, \
            f"{what}: block {b} score {ref_scores[b]} vs k-th {kth} (tol {lim})"


def check_attention(got: np.ndarray, ref: np.ndarray, what=""):
    d = np.abs(got.astype(np.float64) - ref)
    assert d.max() <= ATTN_ATOL, f"{what}: max abs {d.max()}"
