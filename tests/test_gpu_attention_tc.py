"""The sparse core attention on the fifth-generation tensor cores (tcgen05 tiles
fed by TMA block gathers; qsa_set_attention_kernel(1) for this module) against
the oracle, on the cases its design has to get right:
cache rows past the last query holding NaN (the tail's box reads them; they must
be masked and their values cleared), block sizes whose pieces pad or split a
tile, a logit maximum that only appears late in a query's tile stream (the
accumulator is rescaled in TMEM), GQA groups that are not a power of two (the
other kernel), and the failure path of its bounded waits."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import LSE_ATOL, bits, check_attention, dev_full

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC0


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_02_b200 as m

    m.qsa_set_attention_kernel(m.ATTENTION_TCGEN05)
    yield m
    m.qsa_set_attention_kernel(m.ATTENTION_WARP)


def _oracle(cfg):
    return oracle.Oracle(r=cfg.r, K=cfg.K, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads, rope_dims=cfg.rope_dims,
                         rope_base=cfg.rope_base, rms_eps=cfg.rms_eps)


def _layer(qsa, w, cap):
    from block_sparse_long_02_b200.layer import QSALayer

    cfg = qsa.Config.of(w)
    L = QSALayer(cfg, w.batch, cap)
    return cfg, L


def _attend_and_check(qsa, w, cfg, L, q_begin, nq, rows, seqs=(0,)):
    """Prefill [q_begin, q_begin + nq) through the layer (indexer, then the
    attention) and check the given rows' outputs and LSEs against the oracle
    on the GPU's own selection."""
    B = w.batch
    T = q_begin + nq
    iq = dev_full(w, "idx_q", L.cap, T)[:, q_begin:T].contiguous().view(B, nq, 4, 128)
    qq = dev_full(w, "q", L.cap, T)[:, q_begin:T].contiguous().view(B, nq, cfg.q_heads, 128)
    out = torch.empty(B, nq, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, nq, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(B, nq, dtype=torch.int32, device="cuda")
    lse = torch.empty(B, nq, cfg.q_heads, dtype=torch.float32, device="cuda")
    if q_begin // cfg.r:
        L.compress(0, q_begin // cfg.r)
    L.prefill(qq, iq, q_begin, nq, out, sel, nsel, lse)
    torch.cuda.synchronize()
    assert qsa.qsa_workspace_status(L.workspace(qsa.OP_SPARSE_ATTENTION)) == 0
    assert torch.isfinite(out.float()).all()
    o = _oracle(cfg)
    g_sel, g_n = sel.cpu().numpy(), nsel.cpu().numpy()
    g_out, g_lse = out.float().cpu().numpy(), lse.cpu().numpy()
    for s in seqs:
        q = w.host_full("q", s, T).reshape(T, cfg.q_heads, 128)
        k = w.host_full("k", s, T).reshape(T, cfg.kv_heads, 128)
        v = w.host_full("v", s, T).reshape(T, cfg.kv_heads, 128)
        for i in rows:
            j = i - q_begin
            toks = o.token_set(g_sel[s, j, : g_n[s, j]], i)
            ref, ref_lse = o.attention(q[i], k, v, toks)
            check_attention(g_out[s, j], ref, f"s{s} row {i}")
            assert np.abs(g_lse[s, j] - ref_lse).max() <= LSE_ATOL, (s, i)
    return out, sel, nsel


@pytest.mark.parametrize("r", [4, 3])
def test_nan_past_the_last_query_is_never_used(qsa, r):
    """The caches hold NaN from position T on (never written); the last
    queries' tails share a block with those rows, which the gather loads and
    must mask, values included."""
    T, q_begin = 1003, 600
    w = synth.Workload(name="t", n=T, batch=2, r=r, K=256, q_heads=32, kv_heads=4, base_seed=0xA7 + r)
    cap = T + 61
    cfg, L = _layer(qsa, w, cap)
    for name, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
        w.device_fill(name, c.view(w.batch, cap, -1), rows=(0, T))
    for c in (L.k_cache, L.v_cache):
        c.view(torch.int16)[:, T:] = NAN_BF16
    rows = list(range(T - 12, T)) + [q_begin, q_begin + 1, 777]
    _attend_and_check(qsa, w, cfg, L, q_begin, T - q_begin, rows, seqs=(0, 1))


@pytest.mark.parametrize("r,kv_heads", [(3, 4), (16, 4), (64, 4), (64, 8), (2, 1), (5, 2)])
def test_pieces_that_pad_or_split_a_tile(qsa, r, kv_heads):
    """Block sizes whose (tokens x kv heads) pieces leave padding rows in their
    tile slots (r = 3, 2, 5) or span a whole tile or two (r = 64)."""
    n = 1400
    w = synth.Workload(name="t", n=n, r=r, K=512, q_heads=8 * kv_heads, kv_heads=kv_heads,
                       base_seed=0xA9 + r + kv_heads)
    cfg, L = _layer(qsa, w, n)
    for name, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
        w.device_fill(name, c.view(1, n, -1), rows=(0, n))
    rows = list(range(0, 12)) + list(range(n - 9, n)) + [min(r * 40 + 1, n - 10), 999]
    _attend_and_check(qsa, w, cfg, L, 0, n, rows)


def test_late_maximum_rescales_the_accumulator(qsa):
    """A key that makes one head's logit far larger than every earlier one sits
    in the last selected block of a 65-tile query: the reference maxima are
    raised there and the TMEM accumulator columns rescaled."""
    n = 4096
    w = synth.Workload(name="t", n=n, K=2048, q_heads=32, kv_heads=4, base_seed=0xAB)
    cfg, L = _layer(qsa, w, n)
    for name, c in (("k", L.k_cache), ("v", L.v_cache)):
        w.device_fill(name, c.view(1, n, -1), rows=(0, n))
    q = dev_full(w, "q", n).view(1, n, 32, 128)
    i = n - 1
    kB = cfg.k_blocks  # 512 = every visible block of query n-1
    sel = torch.arange(kB, dtype=torch.int32, device="cuda").view(1, 1, kB).repeat(1, n, 1)
    nsel = torch.full((1, n), kB, dtype=torch.int32, device="cuda")
    nsel[0, : n - 4] = 0  # only the last few queries attend over blocks (the others: their tail)
    # Token 4*509+2, kv head 1: aligned with q head 9 of query n-1 (logit ~ 60 / sqrt(d) * |q|).
    qh = q[0, i, 9].float()
    L.k_cache[0, 4 * 509 + 2, 1] = (qh / qh.norm() * 60.0).to(torch.bfloat16)
    out = torch.empty(1, n, 32, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, n, 32, dtype=torch.float32, device="cuda")
    ws = L.workspace(qsa.OP_SPARSE_ATTENTION)
    qsa.qsa_sparse_attention(cfg, 1, q, 0, n, L.k_cache, L.v_cache, n, sel, nsel, out, lse, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_workspace_status(ws) == 0
    o = _oracle(cfg)
    kh = bits(L.k_cache)[0].reshape(n, 4, 128)
    vh = bits(L.v_cache)[0].reshape(n, 4, 128)
    qb = bits(q)[0]
    for row in (n - 4, n - 3, n - 1, 100, 7):
        m = int(nsel[0, row].item())
        toks = o.token_set(np.arange(m, dtype=np.int32), row)
        ref, ref_lse = o.attention(qb[row], kh, vh, toks)
        got = out[0, row].float().cpu().numpy()
        check_attention(got, ref, f"row {row}")
        assert np.abs(lse[0, row].cpu().numpy() - ref_lse).max() <= LSE_ATOL, row
    # the planted key dominates head 9's distribution
    assert lse[0, i, 9].item() > lse[0, i, 8].item() + 5.0


@pytest.mark.parametrize("q_heads,kv_heads", [(12, 4), (24, 8), (10, 2)])
def test_groups_that_are_not_powers_of_two(qsa, q_heads, kv_heads):
    n = 1201
    w = synth.Workload(name="t", n=n, K=256, q_heads=q_heads, kv_heads=kv_heads, base_seed=0xAC + q_heads)
    cfg, L = _layer(qsa, w, n)
    for name, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
        w.device_fill(name, c.view(1, n, -1), rows=(0, n))
    _attend_and_check(qsa, w, cfg, L, 0, n, list(range(0, 9)) + list(range(n - 9, n)))


def test_attention_forced_timeout_is_reported_and_the_context_survives(qsa):
    """Failure path of the tensor-core attention, without a GPU fault: fault
    injection mode 3 withholds the key tiles of each CTA's first group, the MMA
    warp's bounded wait runs out (0.25 s), the kernel records QSA_ERR_TIMEOUT in
    the workspace status, drains, frees its tensor memory and returns; the next
    call on the same context is normal and matches the oracle."""
    import time

    n = 2048 + 5
    w = synth.Workload(name="t", n=n, K=512, q_heads=32, kv_heads=4, base_seed=0xAD)
    cfg, L = _layer(qsa, w, n)
    for name, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
        w.device_fill(name, c.view(1, n, -1), rows=(0, n))
    L.compress(0, n // 4)
    iq = dev_full(w, "idx_q", n).view(1, n, 4, 128).contiguous()
    q = dev_full(w, "q", n).view(1, n, 32, 128).contiguous()
    sel = torch.empty(1, n, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(1, n, dtype=torch.int32, device="cuda")
    qsa.qsa_topk_blocks(cfg, 1, iq, 0, n, L.pooled, n, None, 0, sel, nsel, L.workspace(qsa.OP_TOPK_BLOCKS, n))
    out = torch.empty(1, n, 32, 128, dtype=torch.bfloat16, device="cuda")
    ws = L.workspace(qsa.OP_SPARSE_ATTENTION)
    torch.cuda.synchronize()
    assert qsa.qsa_workspace_status(ws) == 0
    qsa.qsa_set_fault_injection(3, 0.25)
    try:
        t0 = time.time()
        qsa.qsa_sparse_attention(cfg, 1, q, 0, n, L.k_cache, L.v_cache, n, sel, nsel, out, None, ws)
        torch.cuda.synchronize()
        elapsed = time.time() - t0
    finally:
        qsa.qsa_set_fault_injection(0)
    assert qsa.qsa_workspace_status(ws) == 6  # QSA_ERR_TIMEOUT (read and cleared)
    assert elapsed >= 0.2
    qsa.qsa_sparse_attention(cfg, 1, q, 0, n, L.k_cache, L.v_cache, n, sel, nsel, out, None, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_workspace_status(ws) == 0
    o = _oracle(cfg)
    qh = w.host_full("q", 0).reshape(n, 32, 128)
    k = w.host_full("k", 0).reshape(n, 4, 128)
    v = w.host_full("v", 0).reshape(n, 4, 128)
    g_sel, g_n, g_out = sel.cpu().numpy()[0], nsel.cpu().numpy()[0], out.float().cpu().numpy()[0]
    for i in (0, 5, 1000, n - 1):
        toks = o.token_set(g_sel[i, : g_n[i]], i)
        ref, _ = o.attention(qh[i], k, v, toks)
        check_attention(g_out[i], ref, f"row {i}")
