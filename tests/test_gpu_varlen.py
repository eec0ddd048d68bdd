"""Variable-length batched prefill (the *_varlen calls): three sequences with
different query ranges (a whole prompt, a chunk against an existing cache, a
short tail) in one call each, against the oracle row by row and against the
single-range calls bit for bit. Also the prefill from pinned host memory with
overlapped transfers (QSALayer.prefill_from_host) against the device prefill."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import LSE_ATOL, bits, check_attention, check_selection, dev_full, score_tol

pytestmark = pytest.mark.gpu

Q_BEGIN = [0, 700, 2000]
NQ = [1500, 901, 333]
CAP = 2400


@pytest.fixture(params=[0, 1], ids=["warp_tiles", "tcgen05_tiles"])
def qsa(request):
    import block_sparse_long_02_b200 as m

    m.qsa_set_attention_kernel(request.param)
    yield m
    m.qsa_set_attention_kernel(0)


def _packed(w, name, width):
    rows = []
    for s, (b, m) in enumerate(zip(Q_BEGIN, NQ)):
        rows.append(torch.from_numpy(np.ascontiguousarray(w.host_rows(name, s, list(range(b, b + m)))).view(np.int16)))
    return torch.cat(rows).view(torch.bfloat16).reshape(sum(NQ), width // 128, 128).cuda()


def test_varlen_prefill_matches_oracle_and_single_range_calls(qsa):
    from block_sparse_long_02_b200.layer import QSALayer

    w = synth.Workload(name="varlen", n=CAP, batch=3, K=512, q_heads=32, kv_heads=4, base_seed=0x7A1E)
    cfg = qsa.Config.of(w)
    L = QSALayer(cfg, w.batch, CAP)
    for name, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
        w.device_fill(name, c.view(w.batch, CAP, -1), rows=(0, CAP))
    total = sum(NQ)
    q = _packed(w, "q", w.row_len("q"))
    iq = _packed(w, "idx_q", w.row_len("idx_q"))
    out = torch.empty(total, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.full((total, cfg.k_blocks), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((total,), -7, dtype=torch.int32, device="cuda")
    lse = torch.empty(total, cfg.q_heads, dtype=torch.float32, device="cuda")
    # Earlier positions of the chunked sequences are cache state: pool them.
    for s, b in enumerate(Q_BEGIN):
        qsa.qsa_compress_keys(cfg, 1, L.idx_k_cache[s:s + 1], CAP, None, 0, b // cfg.r, L.pooled[s:s + 1])
    L.prefill_varlen(q, iq, Q_BEGIN, NQ, out, sel, nsel, lse)
    torch.cuda.synchronize()

    # The single-range calls on the same inputs give the same bits.
    off = 0
    ws_t = L.workspace_for(qsa.OP_TOPK_BLOCKS, 1, max(NQ))
    for s, (b, m) in enumerate(zip(Q_BEGIN, NQ)):
        sel1 = torch.empty(1, m, cfg.k_blocks, dtype=torch.int32, device="cuda")
        nsel1 = torch.empty(1, m, dtype=torch.int32, device="cuda")
        out1 = torch.empty(1, m, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
        qsa.qsa_topk_blocks(cfg, 1, iq[off:off + m].contiguous(), b, m, L.pooled[s:s + 1], CAP, None, 0, sel1,
                            nsel1, ws_t)
        qsa.qsa_sparse_attention(cfg, 1, q[off:off + m].contiguous(), b, m, L.k_cache[s:s + 1], L.v_cache[s:s + 1],
                                 CAP, sel1, nsel1, out1)
        torch.cuda.synchronize()
        assert torch.equal(sel1[0], sel[off:off + m]) and torch.equal(nsel1[0], nsel[off:off + m]), s
        assert torch.equal(out1[0], out[off:off + m]), s
        off += m

    # Row by row against the oracle (selection on the GPU's pooled keys,
    # attention and LSE on the GPU's selection).
    o = oracle.Oracle(r=cfg.r, K=cfg.K, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads)
    g_sel, g_n, g_out, g_lse = sel.cpu().numpy(), nsel.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy()
    pooled = bits(L.pooled)
    off = 0
    rng = np.random.default_rng(9)
    for s, (b, m) in enumerate(zip(Q_BEGIN, NQ)):
        T = b + m
        hq = w.host_full("q", s, T).reshape(T, cfg.q_heads, 128)
        hk = w.host_full("k", s, T).reshape(T, cfg.kv_heads, 128)
        hv = w.host_full("v", s, T).reshape(T, cfg.kv_heads, 128)
        hiq = w.host_full("idx_q", s, T).reshape(T, 4, 128)
        rows = sorted(set([b, b + 1, T - 1, T - 2] + rng.integers(b, T, 12).tolist()))
        for i in rows:
            j = off + i - b
            ref = o.row(i, hiq[i], pooled[s])
            tol = score_tol(o.rotate_query(hiq[i], i), pooled[s], ref["scores"])
            check_selection(g_sel[j], g_n[j], ref["scores"], tol, o.k_blocks, f"s{s} row {i}")
            toks = o.token_set(g_sel[j, : g_n[j]], i)
            ref_out, ref_lse = o.attention(hq[i], hk, hv, toks)
            check_attention(g_out[j], ref_out, f"s{s} row {i}")
            assert np.abs(g_lse[j] - ref_lse).max() <= LSE_ATOL, (s, i)
        # every row's count invariant
        i = np.arange(b, T)
        want = np.minimum(cfg.k_blocks, i // cfg.r)
        assert np.array_equal(g_n[off:off + m], want), s
        off += m


def test_varlen_errors_launch_nothing(qsa):
    cfg = qsa.Config()
    t = torch.zeros(1 << 12, dtype=torch.bfloat16, device="cuda")
    i32 = torch.zeros(1 << 12, dtype=torch.int32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    n0 = qsa.qsa_launch_count()
    with pytest.raises(qsa.QSAError) as e:  # a range past the capacity
        qsa.qsa_topk_blocks_varlen(cfg, t, [0, 10], [4, 60], t, 64, i32, i32, ws)
    assert e.value.status == 4
    with pytest.raises(qsa.QSAError) as e:  # a negative count
        qsa.qsa_sparse_attention_varlen(cfg, t, [0, 0], [4, -1], t, t, 64, i32, i32, t)
    assert e.value.status == 1
    assert qsa.qsa_launch_count() == n0


@pytest.mark.parametrize("q_begin,first", [(0, 2048), (1000, 2048), (0, 512), (1001, 512)])
def test_prefill_from_host_equals_prefill(q_begin, first):
    """QSALayer.prefill_from_host (inputs and output in pinned host memory,
    moved in chunks overlapped with the compute on side streams) gives the
    device prefill's outputs and caches bit for bit: equal chunks with a
    ragged last one, or chunks ramping 512 -> 2048 -> 512 with a ragged middle
    one; a batch of two; a start after an existing cache (at a block boundary
    or inside a block)."""
    import block_sparse_long_02_b200 as m
    from block_sparse_long_02_b200.layer import QSALayer

    n, B = 6007, 2
    w = synth.Workload(name="pfh", n=n, batch=B, K=512, q_heads=32, kv_heads=4, base_seed=0x7A2F)
    cfg = m.Config.of(w)
    nq = n - q_begin
    full = {nm: dev_full(w, nm, n, n) for nm in ("q", "k", "v", "idx_q", "idx_k")}

    def layer():
        L = QSALayer(cfg, B, n)
        if q_begin:
            for nm, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
                c.view(B, n, -1)[:, :q_begin] = full[nm][:, :q_begin]
            L.compress(0, q_begin // cfg.r)
        return L

    La, Lb = layer(), layer()
    for nm, c in (("k", La.k_cache), ("v", La.v_cache), ("idx_k", La.idx_k_cache)):
        c.view(B, n, -1)[:, q_begin:] = full[nm][:, q_begin:]
    q = full["q"][:, q_begin:].contiguous().view(B, nq, cfg.q_heads, 128)
    iq = full["idx_q"][:, q_begin:].contiguous().view(B, nq, 4, 128)
    out = torch.empty(B, nq, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, nq, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(B, nq, dtype=torch.int32, device="cuda")
    La.prefill(q, iq, q_begin, nq, out, sel, nsel)

    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    hq, hiq = pin(q), pin(iq)
    hk = pin(full["k"][:, q_begin:].view(B, nq, cfg.kv_heads, 128))
    hv = pin(full["v"][:, q_begin:].view(B, nq, cfg.kv_heads, 128))
    hik = pin(full["idx_k"][:, q_begin:])
    hout = torch.zeros(B, nq, cfg.q_heads, 128, dtype=torch.bfloat16).pin_memory()
    Lb.prefill_from_host(hq, hiq, hk, hv, hik, q_begin, nq, hout, chunk=2048, first=first)
    torch.cuda.synchronize()
    assert torch.equal(hout, out.cpu())
    for name in ("k_cache", "v_cache", "idx_k_cache", "pooled"):
        assert torch.equal(getattr(La, name), getattr(Lb, name)), name
