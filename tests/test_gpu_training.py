"""Training kernels (the concept page's "Native trainability" section) through
the C-ABI against the oracle, element by element on the same seeded inputs:
the sparse-attention gradient, the stage-1 distillation target and the KL loss
with its gradient. Sizes span several query tiles and key chunks with ragged
tails. Each stage takes the GPU's own previous-stage outputs (selection,
forward output and LSE, target), as the other parity tests do."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bits, dev_full

pytestmark = pytest.mark.gpu

# dq, dk, dv: max |GPU - oracle| over a tensor, relative to the tensor's largest
# reference magnitude. P and dS enter the tile products as bf16 (relative
# rounding 2^-9 per term) and D comes from the bf16 forward output, so a few
# 2^-9 is the expected scale; 1e-2 leaves room for the sums over tokens.
GRAD_RTOL = 1e-2
# Target: entries are fp32 products of fp32 exponentials of fp32 logits (bf16
# inputs, exact products); relative error ~1e-5.
TARGET_RTOL, TARGET_ATOL = 2e-3, 1e-7


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_02_b200 as m

    return m


def _oracle(cfg):
    return oracle.Oracle(r=cfg.r, K=cfg.K, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads, rope_dims=cfg.rope_dims,
                         rope_base=cfg.rope_base, rms_eps=cfg.rms_eps)


def _forward(qsa, w, cfg, cap):
    """Prefill on the GPU: caches, selection, forward output and LSE."""
    from block_sparse_long_02_b200.layer import QSALayer

    L = QSALayer(cfg, w.batch, cap)
    w.device_fill("k", L.k_cache.view(w.batch, cap, -1), rows=(0, w.n))
    w.device_fill("v", L.v_cache.view(w.batch, cap, -1), rows=(0, w.n))
    w.device_fill("idx_k", L.idx_k_cache, rows=(0, w.n))
    nq = w.n
    q = dev_full(w, "q", cap, nq)[:, :nq].contiguous().view(w.batch, nq, cfg.q_heads, 128)
    iq = dev_full(w, "idx_q", cap, nq)[:, :nq].contiguous().view(w.batch, nq, 4, 128)
    out = torch.empty(w.batch, nq, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(w.batch, nq, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(w.batch, nq, dtype=torch.int32, device="cuda")
    lse = torch.empty(w.batch, nq, cfg.q_heads, dtype=torch.float32, device="cuda")
    L.prefill(q, iq, 0, nq, out, sel, nsel, lse)
    torch.cuda.synchronize()
    return L, q, out, sel, nsel, lse


@pytest.mark.parametrize("n,K,q_heads,kv_heads,batch", [(1003, 256, 32, 4, 1), (517, 128, 16, 1, 2),
                                                         (389, 64, 8, 8, 1)])
def test_attention_backward_matches_oracle(qsa, n, K, q_heads, kv_heads, batch):
    """dq of every query and the accumulated dk, dv of every token against the
    oracle's gradient on the GPU's own selection, forward output and LSE."""
    w = synth.Workload(name="bwd", n=n, K=K, q_heads=q_heads, kv_heads=kv_heads, batch=batch,
                       base_seed=0xB0 + n)
    cfg = qsa.Config.of(w)
    cap = n + 5
    L, q, out, sel, nsel, lse = _forward(qsa, w, cfg, cap)
    dout = dev_full(w, "dout", cap, n)[:, :n].contiguous()
    dq = torch.full((batch, n, q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
    dk = torch.zeros(batch, cap, kv_heads, 128, dtype=torch.float32, device="cuda")
    dv = torch.zeros_like(dk)
    qsa.qsa_sparse_attention_backward(cfg, batch, q, 0, n, L.k_cache, L.v_cache, cap, sel, nsel, out, lse, dout,
                                      dq, dk, dv)
    torch.cuda.synchronize()
    o = _oracle(cfg)
    dq_g, dk_g, dv_g = dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()
    sel_h, nsel_h = sel.cpu().numpy(), nsel.cpu().numpy()
    for s in range(batch):
        qh = w.host_full("q", s, n).reshape(n, q_heads, 128)
        kh = w.host_full("k", s, n)
        vh = w.host_full("v", s, n)
        gh = w.host_full("dout", s, n).reshape(n, q_heads, 128)
        dq_r = np.empty((n, q_heads, 128))
        dk_r = np.zeros((n, kv_heads, 128))
        dv_r = np.zeros((n, kv_heads, 128))
        for i in range(n):
            toks = o.token_set(sel_h[s, i, :nsel_h[s, i]], i)
            a, b, c = o.attention_backward(qh[i], kh, vh, toks, gh[i])
            dq_r[i] = a
            np.add.at(dk_r, toks, b)
            np.add.at(dv_r, toks, c)
        for name, got, ref in (("dq", dq_g[s], dq_r), ("dk", dk_g[s, :n], dk_r), ("dv", dv_g[s, :n], dv_r)):
            err = np.abs(got - ref).max() / np.abs(ref).max()
            assert err <= GRAD_RTOL, f"s{s} {name}: max error {err:.2e} of the largest magnitude"
        assert not dk_g[s, n:].any() and not dv_g[s, n:].any()  # rows past the queries stay zero


def _target_case(qsa, w, cfg, cap, q_begin, nq):
    kc = dev_full(w, "k", cap, q_begin + nq).view(w.batch, cap, cfg.kv_heads, 128)
    q = dev_full(w, "q", cap, q_begin + nq)[:, q_begin:q_begin + nq].contiguous()
    ld = (q_begin + nq - 1) // cfg.r + 3
    target = torch.full((w.batch, nq, ld), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(qsa.qsa_workspace_size(cfg, qsa.OP_DISTILL_TARGET, w.batch, cap, nq), dtype=torch.uint8,
                     device="cuda")
    qsa.qsa_distill_target(cfg, w.batch, q, q_begin, nq, kc, cap, target, ld, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_workspace_status(ws) == 0
    return target.cpu().numpy(), ld


@pytest.mark.parametrize("n,q_begin,r,q_heads,kv_heads,batch",
                         [(700, 0, 4, 32, 4, 2), (611, 250, 4, 32, 4, 1), (300, 0, 1, 8, 8, 1),
                          (530, 0, 16, 16, 1, 1), (401, 0, 2, 16, 8, 1), (333, 0, 8, 16, 4, 1),
                          (290, 0, 4, 32, 2, 1)])
def test_distill_target_matches_oracle(qsa, n, q_begin, r, q_heads, kv_heads, batch):
    """Every entry of every row: the oracle's block-max-pooled, head-averaged
    dense distribution over the visible blocks; zeros from floor(i/r) to ld."""
    w = synth.Workload(name="tgt", n=n, K=64, r=r, q_heads=q_heads, kv_heads=kv_heads, batch=batch,
                       base_seed=0xD1 + n)
    cfg = qsa.Config.of(w)
    cap = n + 7
    nq = n - q_begin
    got, ld = _target_case(qsa, w, cfg, cap, q_begin, nq)
    o = _oracle(cfg)
    for s in range(batch):
        qh = w.host_full("q", s, n).reshape(n, q_heads, 128)
        kh = w.host_full("k", s, n)
        for j in range(nq):
            i = q_begin + j
            nv = i // r
            ref = o.distill_target(i, qh[i], kh)
            row = got[s, j]
            assert np.isfinite(row).all(), (s, i)
            assert not row[nv:].any(), (s, i)
            d = np.abs(row[:nv] - ref)
            assert (d <= TARGET_RTOL * ref + TARGET_ATOL).all(), (s, i, d.max())


def test_distill_kl_matches_oracle(qsa):
    """KL and its gradient per row, from the GPU's target and the GPU's indexer
    scores (qsa_index_scores), against the oracle on the same two rows."""
    w = synth.Workload(name="kl", n=900, K=64, q_heads=32, kv_heads=4, batch=2, base_seed=0xE1)
    cfg = qsa.Config.of(w)
    cap = 904
    q_begin, nq = 100, 800
    target, ld = _target_case(qsa, w, cfg, cap, q_begin, nq)
    from block_sparse_long_02_b200.layer import QSALayer

    L = QSALayer(cfg, w.batch, cap)
    w.device_fill("idx_k", L.idx_k_cache, rows=(0, w.n))
    L.compress(0, w.n // cfg.r)
    iq = dev_full(w, "idx_q", cap, w.n)[:, q_begin:q_begin + nq].contiguous()
    scores = torch.empty(w.batch, nq, ld, dtype=torch.float32, device="cuda")
    ws = L.workspace(qsa.OP_INDEX_SCORES, nq)
    qsa.qsa_index_scores(cfg, w.batch, iq, q_begin, nq, L.pooled, cap, scores, ld, ws)
    tgt_d = torch.tensor(target, device="cuda")
    kl = torch.full((w.batch, nq), float("nan"), dtype=torch.float32, device="cuda")
    ds = torch.full((w.batch, nq, ld), float("nan"), dtype=torch.float32, device="cuda")
    qsa.qsa_distill_kl(cfg, w.batch, q_begin, nq, tgt_d, scores, ld, kl, ds)
    torch.cuda.synchronize()
    o = _oracle(cfg)
    kl_g, ds_g, sc = kl.cpu().numpy(), ds.cpu().numpy(), scores.cpu().numpy()
    for s in range(w.batch):
        for j in range(nq):
            n = (q_begin + j) // cfg.r
            ref_kl, ref_ds = o.distill_kl(target[s, j, :n].astype(np.float64), sc[s, j, :n])
            assert abs(kl_g[s, j] - ref_kl) <= 1e-4 * (1.0 + abs(ref_kl)), (s, j, kl_g[s, j], ref_kl)
            scale = np.abs(ref_ds).max() if n else 0.0
            assert (np.abs(ds_g[s, j, :n] - ref_ds) <= 1e-4 * np.abs(ref_ds) + 1e-6 * scale + 1e-9).all(), (s, j)
            assert not ds_g[s, j, n:].any()


def test_distill_kl_is_zero_at_its_target(qsa):
    """Scores equal to log(target) + c give KL 0 and a zero gradient (the
    minimum), on every row with visible blocks."""
    w = synth.Workload(name="kl0", n=300, K=64, q_heads=32, kv_heads=4, batch=1, base_seed=0xE2)
    cfg = qsa.Config.of(w)
    target, ld = _target_case(qsa, w, cfg, 304, 0, 300)
    t = torch.tensor(target, device="cuda")
    scores = torch.where(t > 0, torch.log(t.clamp_min(1e-38)) + 5.0, torch.full_like(t, -1e4))
    kl = torch.empty(1, 300, dtype=torch.float32, device="cuda")
    ds = torch.empty(1, 300, ld, dtype=torch.float32, device="cuda")
    qsa.qsa_distill_kl(cfg, 1, 0, 300, t, scores, ld, kl, ds)
    torch.cuda.synchronize()
    assert kl.abs().max().item() < 1e-5 and ds.abs().max().item() < 1e-5


def test_target_forced_timeout_is_reported_and_the_context_survives(qsa):
    """Failure path of the tcgen05 target kernels, without a GPU fault: with
    fault injection their producers withhold every key tile, the MMA warps'
    bounded waits run out (0.1 s), each CTA records QSA_ERR_TIMEOUT in the
    workspace status, drains, frees its tensor memory and returns; the next
    call is normal and matches the oracle."""
    import time

    w = synth.Workload(name="tto", n=300, K=64, q_heads=32, kv_heads=4, batch=1, base_seed=0xE3)
    cfg = qsa.Config.of(w)
    cap, nq = 304, 300
    kc = dev_full(w, "k", cap, nq).view(1, cap, cfg.kv_heads, 128)
    q = dev_full(w, "q", cap, nq)[:, :nq].contiguous()
    ld = (nq - 1) // cfg.r
    target = torch.zeros(1, nq, ld, dtype=torch.float32, device="cuda")
    ws = torch.zeros(qsa.qsa_workspace_size(cfg, qsa.OP_DISTILL_TARGET, 1, cap, nq), dtype=torch.uint8,
                     device="cuda")
    qsa.qsa_set_fault_injection(2, 0.1)
    try:
        t0 = time.time()
        qsa.qsa_distill_target(cfg, 1, q, 0, nq, kc, cap, target, ld, ws)
        torch.cuda.synchronize()
        elapsed = time.time() - t0
    finally:
        qsa.qsa_set_fault_injection(0)
    assert qsa.qsa_workspace_status(ws) == 6  # QSA_ERR_TIMEOUT (read and cleared)
    assert elapsed >= 0.1
    qsa.qsa_distill_target(cfg, 1, q, 0, nq, kc, cap, target, ld, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_workspace_status(ws) == 0
    o = _oracle(cfg)
    qh = w.host_full("q", 0, nq).reshape(nq, cfg.q_heads, 128)
    kh = w.host_full("k", 0, nq)
    got = target.cpu().numpy()[0]
    for i in (5, 150, nq - 1):
        ref = o.distill_target(i, qh[i], kh)
        assert (np.abs(got[i, : i // cfg.r] - ref) <= TARGET_RTOL * ref + TARGET_ATOL).all(), i
