"""CUDA path (through the C-ABI) against the oracle, element by element, on the
same seeded inputs. Sizes span several query/block tiles with ragged tails;
each stage is fed the GPU's previous-stage output so tolerated differences do
not cascade. Parity rules live in gpu_util."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import (bits, check_attention, check_scores, check_selection, dev_full, f32, score_tol,
                      LSE_ATOL)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_02_b200 as m

    return m


@pytest.fixture(params=[0, 1], ids=["warp_tiles", "tcgen05_tiles"])
def kernel(request, qsa):
    """Runs a prefill test with each sparse-attention kernel."""
    qsa.qsa_set_attention_kernel(request.param)
    yield request.param
    qsa.qsa_set_attention_kernel(0)


@pytest.fixture(params=[0, 1], ids=["step_kernel", "three_kernels"])
def decode_kernel(request, qsa):
    """Runs a decode test with each decode path: one persistent step kernel,
    and the three kernels (scores, selection, attention)."""
    qsa.qsa_set_decode_kernel(request.param)
    yield request.param
    qsa.qsa_set_decode_kernel(1)


def _layer(qsa, w, cap, **over):
    from block_sparse_long_02_b200.layer import QSALayer

    cfg = qsa.Config.of(w)
    for k, v in over.items():
        setattr(cfg, k, v)
    return cfg, QSALayer(cfg, w.batch, cap)


def _fill_caches(w, L, T):
    w.device_fill("k", L.k_cache.view(w.batch, L.cap, -1), rows=(0, T))
    w.device_fill("v", L.v_cache.view(w.batch, L.cap, -1), rows=(0, T))
    w.device_fill("idx_k", L.idx_k_cache, rows=(0, T))


def run_prefill(qsa, w, q_begin=0, nq=None, cap=None, lse=True, **over):
    nq = w.n - q_begin if nq is None else nq
    cap = cap or (q_begin + nq)
    cfg, L = _layer(qsa, w, cap, **over)
    _fill_caches(w, L, q_begin + nq)
    iq = dev_full(w, "idx_q", cap, q_begin + nq)[:, q_begin:q_begin + nq].contiguous()
    qq = dev_full(w, "q", cap, q_begin + nq)[:, q_begin:q_begin + nq].contiguous()
    out = torch.empty(w.batch, nq, cfg.q_heads, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
    sel = torch.full((w.batch, nq, cfg.k_blocks), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((w.batch, nq), -7, dtype=torch.int32, device="cuda")
    lse_t = torch.empty(w.batch, nq, cfg.q_heads, dtype=torch.float32, device="cuda") if lse else None
    if q_begin // cfg.r:
        L.compress(0, q_begin // cfg.r)
    L.prefill(qq, iq.view(w.batch, nq, 4, 128), q_begin, nq, out, sel, nsel, lse_t)
    torch.cuda.synchronize()
    return cfg, {"pooled": bits(L.pooled), "sel": sel.cpu().numpy(), "nsel": nsel.cpu().numpy(),
                 "out": out.float().cpu().numpy(), "lse": None if lse_t is None else lse_t.cpu().numpy()}


def _oracle(w, cfg):
    return oracle.Oracle(r=cfg.r, K=cfg.K, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads,
                         rope_dims=cfg.rope_dims, rope_base=cfg.rope_base, rms_eps=cfg.rms_eps)


def check_rows(w, cfg, res, rows, s=0, q_begin=0, attention=True):
    o = _oracle(w, cfg)
    T = q_begin + res["sel"].shape[1]
    idx_q = w.host_full("idx_q", s, T).reshape(T, 4, 128)
    q = w.host_full("q", s, T).reshape(T, cfg.q_heads, 128)
    k = w.host_full("k", s, T).reshape(T, cfg.kv_heads, 128)
    v = w.host_full("v", s, T).reshape(T, cfg.kv_heads, 128)
    pooled = res["pooled"][s]
    for i in rows:
        j = i - q_begin
        ref = o.row(i, idx_q[i], pooled)
        tol = score_tol(o.rotate_query(idx_q[i], i), pooled, ref["scores"])
        check_selection(res["sel"][s, j], res["nsel"][s, j], ref["scores"], tol, o.k_blocks, f"s{s} row {i}")
        if attention:
            n = res["nsel"][s, j]
            toks = o.token_set(res["sel"][s, j, :n], i)
            out_ref, lse_ref = o.attention(q[i], k, v, toks)
            check_attention(res["out"][s, j], out_ref, f"s{s} row {i}")
            if res["lse"] is not None:
                assert np.abs(res["lse"][s, j] - lse_ref).max() <= LSE_ATOL, i


# ----------------------------------------------------------------------------- a1-a3
@pytest.mark.parametrize("n,batch", [(256, 1), (4096 + 12, 2), (1003, 1)])
def test_compress_matches_oracle(qsa, n, batch):
    w = synth.Workload(name="t", n=n, batch=batch, K=64, q_heads=8, kv_heads=2, base_seed=0xC0 + n)
    cfg, L = _layer(qsa, w, n)
    _fill_caches(w, L, n)
    L.compress(0, n // 4)
    torch.cuda.synchronize()
    got = bits(L.pooled)
    o = _oracle(w, cfg)
    for s in range(batch):
        ref = o.compress(w.host_full("idx_k", s), n // 4)
        d = np.abs(got[s].astype(np.int32) - ref.astype(np.int32))
        assert d.max() <= 1, f"pooled keys differ by {d.max()} bf16 ulp"
        assert (d == 0).mean() > 0.9999


def test_compress_subrange_and_weight(qsa):
    w = synth.Workload(name="t", n=512, K=64, q_heads=4, kv_heads=1, base_seed=0xC1)
    cfg, L = _layer(qsa, w, 512)
    _fill_caches(w, L, 512)
    L.rms_w = torch.linspace(0.5, 2.0, 128, device="cuda", dtype=torch.float32)
    L.pooled.fill_(0)
    L.compress(10, 50)
    torch.cuda.synchronize()
    got = bits(L.pooled)[0]
    ref = _oracle(w, cfg).compress(w.host_full("idx_k", 0), 128, w=L.rms_w.cpu().numpy())
    assert (got[:10] == 0).all() and (got[50:] == 0).all()
    assert np.abs(got[10:50].astype(np.int32) - ref[10:50].astype(np.int32)).max() <= 1


# ----------------------------------------------------------------------------- a4
@pytest.mark.parametrize("n,q_begin", [(256, 0), (2003, 0), (2003, 1100)])
def test_index_scores_match_oracle(qsa, n, q_begin):
    w = synth.Workload(name="t", n=n, K=64, q_heads=4, kv_heads=1, base_seed=0xD0 + n + q_begin)
    cfg, L = _layer(qsa, w, n)
    _fill_caches(w, L, n)
    L.compress(0, n // 4)
    nq = n - q_begin
    iq = dev_full(w, "idx_q", n)[:, q_begin:].contiguous()
    ld = (n - 1) // 4 + 3
    scores = torch.full((1, nq, ld), 7.0, device="cuda")
    ws = qsa.workspace(cfg, qsa.OP_INDEX_SCORES, 1, n, nq)
    qsa.qsa_index_scores(cfg, 1, iq, q_begin, nq, L.pooled, n, scores, ld, ws)
    torch.cuda.synchronize()
    got = scores.cpu().numpy()[0]
    pooled = bits(L.pooled)[0]
    o = _oracle(w, cfg)
    idx_q = w.host_full("idx_q", 0).reshape(n, 4, 128)
    for j in range(nq):
        i = q_begin + j
        c = i // 4
        ref = o.scores(o.rotate_query(idx_q[i], i), pooled, c)
        check_scores(got[j, :c], ref, score_tol(o.rotate_query(idx_q[i], i), pooled, ref), f"row {i}")
        assert np.isneginf(got[j, c:]).all(), i


# ----------------------------------------------------------------------------- a5
def test_select_from_scores_is_exact(qsa):
    """Selection is integer work: given the same scores it must equal the oracle's
    selection exactly, including heavy ties (rounded and zero scores)."""
    rng = np.random.default_rng(3)
    cfg = qsa.Config(K=64, q_heads=4, kv_heads=1)  # k_B = 16
    nq, q_begin = 300, 5000
    ld = (q_begin + nq - 1) // 4
    sc = np.round(rng.standard_normal((1, nq, ld)) * 3).astype(np.float32)
    sc[:, : nq // 3] = 0.0                                # all-tie rows
    sc[:, nq // 3: nq // 2] = np.abs(sc[:, nq // 3: nq // 2])  # many ties
    sc[:, -5:] = rng.standard_normal((5, ld)).astype(np.float32)
    scores = torch.from_numpy(sc).cuda()
    sel = torch.empty(1, nq, 16, dtype=torch.int32, device="cuda")
    nsel = torch.empty(1, nq, dtype=torch.int32, device="cuda")
    qsa.qsa_topk_blocks(cfg, 1, None, q_begin, nq, None, q_begin + nq, scores, ld, sel, nsel, None)
    torch.cuda.synchronize()
    o = oracle.Oracle(K=64, q_heads=4, kv_heads=1)
    g = sel.cpu().numpy()[0]
    for j in range(nq):
        c = (q_begin + j) // 4
        ref = o.select(sc[0, j, :c])
        assert np.array_equal(g[j], ref), j
    assert (nsel.cpu().numpy() == 16).all()


def test_select_candidate_overflow_path(qsa):
    """More than 4096 exactly equal scores at the threshold digit: the general path."""
    cfg = qsa.Config(K=2048, q_heads=4, kv_heads=1)
    ld = 60000
    sc = np.zeros((1, 2, ld), dtype=np.float32)
    sc[0, 1, ::7] = 1.0
    scores = torch.from_numpy(sc).cuda()
    sel = torch.empty(1, 2, 512, dtype=torch.int32, device="cuda")
    nsel = torch.empty(1, 2, dtype=torch.int32, device="cuda")
    qsa.qsa_topk_blocks(cfg, 1, None, 4 * ld, 2, None, 4 * ld + 2, scores, ld, sel, nsel, None)
    torch.cuda.synchronize()
    o = oracle.Oracle(K=2048)
    for j in range(2):
        assert np.array_equal(sel.cpu().numpy()[0, j], o.select(sc[0, j, : (4 * ld + j) // 4]))


# ----------------------------------------------------------------------------- a1..a7 prefill
def test_tiny_prefill_all_rows(qsa, kernel):
    w = synth.WORKLOADS["tiny_prefill_n256"]
    cfg, res = run_prefill(qsa, w)
    check_rows(w, cfg, res, range(w.n))


@pytest.mark.parametrize("q_heads,kv_heads", [(32, 4), (8, 1), (16, 2), (64, 8), (16, 4)])
def test_prefill_ragged_gqa(qsa, q_heads, kv_heads, kernel):
    w = synth.Workload(name="t", n=2003, K=128, q_heads=q_heads, kv_heads=kv_heads,
                       base_seed=0xE0 + q_heads, n_needles_prefill=6)
    cfg, res = run_prefill(qsa, w)
    rows = sorted(set(list(range(0, 40)) + list(range(1960, 2003)) +
                      np.random.default_rng(1).integers(0, 2003, 40).tolist() + [p for _, p in w.needles(0)]))
    check_rows(w, cfg, res, rows)


def test_prefill_chunk_with_offset_and_batch(qsa, kernel):
    w = synth.Workload(name="t", n=1500, batch=2, K=96, q_heads=8, kv_heads=2, base_seed=0xE7)
    cfg, res = run_prefill(qsa, w, q_begin=701, nq=799)
    rows = list(range(701, 740)) + list(range(1460, 1500))
    for s in range(2):
        check_rows(w, cfg, res, rows, s=s, q_begin=701)


def test_budget_covering_all_blocks_is_dense(qsa, kernel):
    """k_B >= visible blocks: every visible block is selected, in order."""
    w = synth.Workload(name="t", n=600, K=4096, q_heads=8, kv_heads=2, base_seed=0xE8)
    cfg, res = run_prefill(qsa, w)
    for i in range(600):
        c = i // 4
        assert res["nsel"][0, i] == c and np.array_equal(res["sel"][0, i, :c], np.arange(c))
    check_rows(w, cfg, res, [0, 1, 3, 4, 5, 77, 598, 599])


@pytest.mark.parametrize("r", [1, 8])
def test_generic_block_size(qsa, r, kernel):
    w = synth.Workload(name="t", n=777, r=r, K=96, q_heads=8, kv_heads=2, base_seed=0xE9 + r)
    cfg, res = run_prefill(qsa, w)
    check_rows(w, cfg, res, list(range(0, 20)) + list(range(700, 777)))


def test_invalid_selection_entries_are_skipped(qsa, kernel):
    """Entries outside [0, floor(i/r)) never read memory; they drop out of the set."""
    w = synth.Workload(name="t", n=512, K=64, q_heads=8, kv_heads=2, base_seed=0xEA)
    cfg, L = _layer(qsa, w, 512)
    _fill_caches(w, L, 512)
    q = dev_full(w, "q", 512)
    nq = 512
    sel = torch.full((1, nq, 16), -1, dtype=torch.int32, device="cuda")
    nsel = torch.full((1, nq), 16, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(4)
    raw = rng.integers(-5, 200, (nq, 16)).astype(np.int32)
    raw[:, 0] = 10**9
    sel.copy_(torch.from_numpy(raw)[None])
    out = torch.empty(1, nq, 8, 128, dtype=torch.bfloat16, device="cuda")
    qsa.qsa_sparse_attention(cfg, 1, q, 0, nq, L.k_cache, L.v_cache, 512, sel, nsel, out)
    torch.cuda.synchronize()
    o = _oracle(w, cfg)
    qh = w.host_full("q", 0).reshape(512, 8, 128)
    k = w.host_full("k", 0).reshape(512, 2, 128)
    v = w.host_full("v", 0).reshape(512, 2, 128)
    got = out.float().cpu().numpy()[0]
    for i in [3, 50, 200, 511]:
        valid = np.array([b for b in raw[i] if 0 <= b < i // 4], dtype=np.int32)
        toks = np.concatenate([np.arange(4 * b, 4 * b + 4) for b in valid] +
                              [np.arange(4 * (i // 4), i + 1)]).astype(np.int64)
        ref, _ = o.attention(qh[i], k, v, toks)
        check_attention(got[i], ref, f"row {i}")


def test_host_errors(qsa):
    cfg = qsa.Config()
    t = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qsa.QSAError) as e:
        qsa.qsa_compress_keys(cfg, 1, t, 16, None, 0, 5, t)
    assert e.value.status == 4
    sel = torch.zeros(512, dtype=torch.int32, device="cuda")
    with pytest.raises(qsa.QSAError) as e:
        qsa.qsa_sparse_attention(cfg, 1, t, 10, 10, t, t, 15, sel, sel, t)
    assert e.value.status == 4
    with pytest.raises(qsa.QSAError) as e:
        qsa.qsa_topk_blocks(cfg, 1, t, 0, 8, t, 64, None, 0, sel, sel, torch.zeros(8, dtype=torch.uint8,
                                                                                  device="cuda"))
    assert e.value.status == 3


# ----------------------------------------------------------------------------- decode
def _decode_run(qsa, w, starts, steps, check=True):
    """Decode `steps` tokens per sequence starting at positions `starts` (one per
    sequence); compare every step with the oracle's decode step."""
    from block_sparse_long_02_b200.layer import QSALayer

    B = w.batch
    cfg = qsa.Config.of(w)
    cap = max(starts) + steps + 3
    L = QSALayer(cfg, B, cap)
    T = max(starts) + steps
    full = {n: dev_full(w, n, cap, T) for n in ("q", "k", "v", "idx_q", "idx_k")}
    for s in range(B):
        for n, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
            c.view(B, cap, -1)[s, : starts[s]] = full[n][s, : starts[s]]
    for s in range(B):
        from block_sparse_long_02_b200 import qsa_compress_keys

        qsa_compress_keys(cfg, 1, L.idx_k_cache[s:s + 1], cap, None, 0, starts[s] // cfg.r, L.pooled[s:s + 1])
    o = _oracle(w, cfg)
    host = [{n: w.host_full(n, s, T) for n in ("q", "k", "v", "idx_q", "idx_k")} for s in range(B)]
    oc = []
    for s in range(B):
        kc = np.zeros((cap, cfg.kv_heads * 128), np.uint16)
        vc = np.zeros_like(kc)
        ik = np.zeros((cap, 128), np.uint16)
        kc[: starts[s]] = host[s]["k"][: starts[s]]
        vc[: starts[s]] = host[s]["v"][: starts[s]]
        ik[: starts[s]] = host[s]["idx_k"][: starts[s]]
        pooled = np.zeros((cap // cfg.r, 128), np.uint16)
        pooled[: starts[s] // cfg.r] = o.compress(ik, starts[s] // cfg.r)
        oc.append((kc, vc, ik, pooled))
    pos = torch.tensor(starts, dtype=torch.int64, device="cuda")
    out = torch.empty(B, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(B, dtype=torch.int32, device="cuda")
    ar = torch.arange(B, device="cuda")
    for step in range(steps):
        p = pos.clone()
        args = [full[n][ar, p].contiguous() for n in ("q", "k", "v", "idx_q", "idx_k")]
        L.decode_step(pos, *args, out, sel, nsel)
        torch.cuda.synchronize()
        if check:
            g_out, g_sel, g_nsel = out.float().cpu().numpy(), sel.cpu().numpy(), nsel.cpu().numpy()
            g_pooled = bits(L.pooled)
            for s in range(B):
                ps = starts[s] + step
                kc, vc, ik, pooled = oc[s]
                hs = host[s]
                # Scores of the oracle on the GPU's pooled keys (stage-by-stage feeding).
                ref = o.row(ps, hs["idx_q"][ps].reshape(4, 128), g_pooled[s])
                tol = score_tol(o.rotate_query(hs["idx_q"][ps].reshape(4, 128), ps), g_pooled[s], ref["scores"])
                check_selection(g_sel[s], g_nsel[s], ref["scores"], tol, cfg.k_blocks, f"s{s} p{ps}")
                res = o.decode_step(ps, hs["q"][ps], hs["k"][ps], hs["v"][ps], hs["idx_q"][ps], hs["idx_k"][ps],
                                    kc, vc, ik, pooled)
                toks = o.token_set(g_sel[s, : g_nsel[s]], ps)
                out_ref, _ = o.attention(hs["q"][ps], kc, vc, toks)
                check_attention(g_out[s], out_ref.reshape(cfg.q_heads, 128), f"s{s} p{ps}")
                # Cache update: the GPU's pooled cache equals the oracle's (<= 1 ulp).
                assert np.abs(g_pooled[s].astype(np.int32)[: (ps + 1) // cfg.r]
                              - pooled.astype(np.int32)[: (ps + 1) // cfg.r]).max(initial=0) <= 1
        pos += 1
    return L


def test_decode_steps_match_oracle(qsa, decode_kernel):
    w = synth.Workload(name="t", n=777, batch=2, decode_steps=12, prefill=False, K=128, q_heads=16,
                       kv_heads=2, base_seed=0xF0, n_needles_decode=3)
    _decode_run(qsa, w, [777, 782], 12)


def test_decode_short_context_and_capacity_flag(qsa, decode_kernel):
    w = synth.Workload(name="t", n=0, batch=1, decode_steps=9, prefill=False, K=16, q_heads=8,
                       kv_heads=2, base_seed=0xF1)
    L = _decode_run(qsa, w, [0], 9)
    # A position at or beyond the capacity is skipped and flagged in the workspace.
    cfg = L.cfg
    pos = torch.tensor([L.cap], dtype=torch.int64, device="cuda")
    z = torch.zeros(1, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, cfg.kv_heads, 128, dtype=torch.bfloat16, device="cuda")
    iq = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    ik = torch.zeros(1, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(z)
    L.decode_step(pos, z, kv, kv, iq, ik, out)
    ws = L.workspace(qsa.OP_DECODE_STEP)
    assert qsa.qsa_workspace_status(ws) == 4
    assert qsa.qsa_workspace_status(ws) == 0


# ----------------------------------------------------------------------------- fused top-k specifics
@pytest.mark.parametrize("n,K", [(8192, 128), (8192, 2048), (6001, 2048)])
def test_fused_topk_with_buffer_compaction(qsa, n, K):
    """More than 896 visible blocks per query: candidate buffers are compacted
    many times during the sweep (k_B = 32 and 512)."""
    w = synth.Workload(name="t", n=n, K=K, q_heads=8, kv_heads=2, base_seed=0xB0 + n + K, n_needles_prefill=8)
    cfg, res = run_prefill(qsa, w, lse=False)
    rng = np.random.default_rng(n + K)
    rows = sorted(set(rng.integers(0, n, 40).tolist() + list(range(n - 10, n)) + [p for _, p in w.needles(0)]
                      + [4 * 513, 4 * 513 + 3, 4 * 897, 4 * 1024 + 1]))
    check_rows(w, cfg, res, [i for i in rows if i < n], attention=False)
    for b, p in w.needles(0):
        assert b in set(res["sel"][0, p, : res["nsel"][0, p]].tolist()), (b, p)


@pytest.mark.parametrize("n", [6000, 36000])
def test_fused_topk_exact_ties(qsa, n):
    """rope_dims = 0 and a periodic key pattern make many pooled keys identical:
    exactly equal scores must resolve to the lower block index, as in the oracle.
    At n = 36000 a query sees up to 71 key tiles, so the sweep visits the sample
    tiles 0, 16, 32, ... before tiles 1-15: equal-score blocks of lower index
    then arrive after higher-index ones and must still win."""
    period = 37
    w = synth.Workload(name="t", n=n, K=256, rope_dims=0, q_heads=8, kv_heads=2, base_seed=0xB7)
    cfg, L = _layer(qsa, w, n)
    _fill_caches(w, L, n)
    base_rows = L.idx_k_cache[:, : 4 * period].clone()
    reps = -(-n // (4 * period))
    L.idx_k_cache[:, :n] = base_rows.repeat(1, reps, 1)[:, :n]
    iq = dev_full(w, "idx_q", n)
    nq = n
    sel = torch.empty(1, nq, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(1, nq, dtype=torch.int32, device="cuda")
    L.compress(0, n // 4)
    ws = L.workspace(qsa.OP_TOPK_BLOCKS, nq)
    qsa.qsa_topk_blocks(cfg, 1, iq, 0, nq, L.pooled, n, None, 0, sel, nsel, ws)
    torch.cuda.synchronize()
    o = _oracle(w, cfg)
    idx_k = bits(L.idx_k_cache)[0]
    pooled = o.compress(idx_k, n // 4)
    assert np.array_equal(pooled, bits(L.pooled)[0])
    idx_q = w.host_full("idx_q", 0).reshape(n, 4, 128)
    g_sel, g_n = sel.cpu().numpy()[0], nsel.cpu().numpy()[0]
    rows = [300, 1999, 4000, 5555, 5999] + ([9000, 17777, 26000, 35999] if n > 6000 else [])
    for i in rows:
        ref = o.row(i, idx_q[i], pooled)
        # Scores are bit-identical between equal blocks on both sides, so the set
        # must match exactly (near-ties with other blocks are still tolerated).
        tol = score_tol(o.rotate_query(idx_q[i], i), pooled, ref["scores"])
        check_selection(g_sel[i], g_n[i], ref["scores"], tol, o.k_blocks, f"row {i}")
        got = set(g_sel[i, : g_n[i]].tolist())
        for b in got:  # every selected block's earlier twins with the same score are selected too
            for b2 in range(b % period, b, period):
                if ref["scores"][b2] == ref["scores"][b]:
                    assert b2 in got, (i, b, b2)


def test_fused_topk_all_zero_scores(qsa):
    """Zero indexer queries make every score 0: the k_B lowest blocks win."""
    n = 5000
    w = synth.Workload(name="t", n=n, K=512, q_heads=8, kv_heads=2, base_seed=0xB8)
    cfg, L = _layer(qsa, w, n)
    _fill_caches(w, L, n)
    L.compress(0, n // 4)
    iq = torch.zeros(1, n, 4, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(1, n, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(1, n, dtype=torch.int32, device="cuda")
    qsa.qsa_topk_blocks(cfg, 1, iq, 0, n, L.pooled, n, None, 0, sel, nsel, L.workspace(qsa.OP_TOPK_BLOCKS, n))
    torch.cuda.synchronize()
    g, gn = sel.cpu().numpy()[0], nsel.cpu().numpy()[0]
    for i in range(0, n, 97):
        m = min(128, i // 4)
        assert gn[i] == m and np.array_equal(g[i, :m], np.arange(m)), i


def test_fused_topk_unrepresentative_sample_is_redone_exactly(qsa):
    """Make the estimate phase fail on purpose: blocks of every 16th 128-block
    tile (the sweep's sample) get keys along a direction all queries share, so the
    threshold estimated from them admits too few candidates elsewhere. The check
    must catch it and the exact redo must give the oracle's selection."""
    n = 32768 + 40
    w = synth.Workload(name="t", n=n, K=2048, q_heads=8, kv_heads=2, base_seed=0xB9)
    cfg, L = _layer(qsa, w, n)
    _fill_caches(w, L, n)
    c = torch.zeros(128, device="cuda")
    c[64:] = torch.randn(64, generator=torch.Generator().manual_seed(3)).cuda()
    c = c / c.norm()
    blk = torch.arange(n // 4, device="cuda")
    sample_blocks = blk[(blk // 128) % 16 == 0]
    rows = (sample_blocks[:, None] * 4 + torch.arange(4, device="cuda")[None, :]).reshape(-1)
    L.idx_k_cache[0, rows] = (24.0 * c).to(torch.bfloat16)
    iq = dev_full(w, "idx_q", n).view(1, n, 4, 128)
    iq = (iq.float() + 3.0 * c).to(torch.bfloat16).contiguous()
    L.compress(0, n // 4)
    sel = torch.empty(1, n, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(1, n, dtype=torch.int32, device="cuda")
    qsa.qsa_topk_blocks(cfg, 1, iq, 0, n, L.pooled, n, None, 0, sel, nsel, L.workspace(qsa.OP_TOPK_BLOCKS, n))
    torch.cuda.synchronize()
    o = _oracle(w, cfg)
    pooled = bits(L.pooled)[0]
    iq_bits = bits(iq)[0].reshape(n, 4, 128)
    g, gn = sel.cpu().numpy()[0], nsel.cpu().numpy()[0]
    for i in [4200, 9000, 20001, 32767, n - 1]:
        ref = o.row(i, iq_bits[i], pooled)
        tol = score_tol(o.rotate_query(iq_bits[i], i), pooled, ref["scores"])
        check_selection(g[i], gn[i], ref["scores"], tol, o.k_blocks, f"row {i}")


def test_fused_topk_split_key_ranges(qsa):
    """A short chunk against a long context (6 query tiles, ~15K visible blocks):
    the fused indexer splits each tile's key range over several CTAs and merges
    the per-split top-k lists; every row must still be the exact selection."""
    w = synth.Workload(name="t", n=60300, batch=2, K=2048, q_heads=4, kv_heads=1, base_seed=0x5B1)
    n0 = qsa.qsa_launch_count()
    cfg, res = run_prefill(qsa, w, q_begin=60000, nq=300)
    # prefix compress, compress, rotate, fused indexer, split merge, attention
    assert qsa.qsa_launch_count() - n0 == 6
    for s in range(w.batch):
        check_rows(w, cfg, res, range(60000, 60300), s=s, q_begin=60000, attention=False)
        check_rows(w, cfg, res, [60000, 60001, 60150, 60299], s=s, q_begin=60000)


def test_forced_timeout_is_reported_and_the_context_survives(qsa):
    """Failure path of the fused indexer, without a GPU fault: with fault
    injection the key tiles of each CTA's first unit are withheld, the MMA
    warp's bounded wait runs out (0.25 s), the kernel reports QSA_ERR_TIMEOUT
    in the workspace status, drains and returns; the next call is normal."""
    import time

    n = 4096 + 8
    w = synth.Workload(name="t", n=n, K=2048, q_heads=4, kv_heads=1, base_seed=0xE1)
    cfg, L = _layer(qsa, w, n)
    _fill_caches(w, L, n)
    L.compress(0, n // 4)
    iq = dev_full(w, "idx_q", n).view(1, n, 4, 128).contiguous()
    sel = torch.empty(1, n, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(1, n, dtype=torch.int32, device="cuda")
    ws = L.workspace(qsa.OP_TOPK_BLOCKS, n)
    assert qsa.qsa_workspace_status(ws) == 0
    qsa.qsa_set_fault_injection(1, 0.25)
    try:
        t0 = time.time()
        qsa.qsa_topk_blocks(cfg, 1, iq, 0, n, L.pooled, n, None, 0, sel, nsel, ws)
        torch.cuda.synchronize()
        elapsed = time.time() - t0
    finally:
        qsa.qsa_set_fault_injection(0)
    assert qsa.qsa_workspace_status(ws) == 6  # QSA_ERR_TIMEOUT (read and cleared)
    assert elapsed >= 0.2
    qsa.qsa_topk_blocks(cfg, 1, iq, 0, n, L.pooled, n, None, 0, sel, nsel, ws)
    torch.cuda.synchronize()
    assert qsa.qsa_workspace_status(ws) == 0
    o = _oracle(w, cfg)
    pooled = bits(L.pooled)[0]
    iq_bits = bits(iq)[0].reshape(n, 4, 128)
    g, gn = sel.cpu().numpy()[0], nsel.cpu().numpy()[0]
    for i in [100, 2051, 3000, n - 1]:
        ref = o.row(i, iq_bits[i], pooled)
        tol = score_tol(o.rotate_query(iq_bits[i], i), pooled, ref["scores"])
        check_selection(g[i], gn[i], ref["scores"], tol, o.k_blocks, f"row {i}")


def test_decode_graph_replay_matches_eager(qsa, decode_kernel):
    """Decode steps captured into one CUDA graph and replayed give the same
    outputs, bit for bit, and the same caches as the eager calls (the kernels'
    programmatic dependencies become graph edges)."""
    from block_sparse_long_02_b200.layer import QSALayer

    n, S = 9000, 6
    w = synth.Workload(name="t", n=n, batch=2, decode_steps=S, prefill=False, K=2048, q_heads=32, kv_heads=4,
                       base_seed=0xF7)
    B = w.batch
    cfg = qsa.Config.of(w)
    cap = n + S + 4
    full = {nm: dev_full(w, nm, cap, n + S) for nm in ("q", "k", "v", "idx_q", "idx_k")}

    def make():
        L = QSALayer(cfg, B, cap)
        _fill_caches(w, L, n)
        L.compress(0, n // cfg.r)
        return L

    def steps():
        return [{"pos": torch.full((B,), n + k, dtype=torch.int64, device="cuda"),
                 **{nm: full[nm][:, n + k].contiguous() for nm in ("q", "k", "v", "idx_q", "idx_k")},
                 "out": torch.empty(B, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")} for k in range(S)]

    La, Lb = make(), make()
    sa, sb = steps(), steps()
    for d in sa:
        La.decode_step(d["pos"], d["q"], d["k"], d["v"], d["idx_q"], d["idx_k"], d["out"])
    g = Lb.capture_decode(sb)
    g.replay()
    torch.cuda.synchronize()
    for k in range(S):
        assert torch.equal(sa[k]["out"], sb[k]["out"]), k
    for name in ("k_cache", "v_cache", "idx_k_cache", "pooled"):
        assert torch.equal(getattr(La, name), getattr(Lb, name)), name
    assert qsa.qsa_workspace_status(La.workspace(qsa.OP_DECODE_STEP)) == 0
    assert qsa.qsa_workspace_status(Lb.workspace(qsa.OP_DECODE_STEP)) == 0


# ----------------------------------------------------------------------------- fp8 (E4M3) caches
def test_quantize_rows_matches_oracle_bit_for_bit(qsa):
    """Codes and scales of the row quantizer equal the oracle's: random rows
    over many magnitudes, a zero row, rows on the scaled E4M3 grid (exact ties
    between codes) and rows whose values saturate."""
    rng = np.random.default_rng(81)
    rows = 3000
    x = (rng.standard_normal((rows, 128)) * np.exp(rng.uniform(-12, 12, (rows, 1)))).astype(np.float32)
    x[5] = 0.0
    o = oracle.Oracle()
    grid = np.array([o.e4m3_value(c) for c in range(127)])
    for r in range(10, 60):  # midpoints between adjacent codes, times a power of two
        a = rng.integers(0, 125, 128)
        x[r] = ((grid[a] + grid[a + 1]) / 2 * rng.choice([-1, 1], 128) * 2.0 ** int(rng.integers(-8, 8))).astype(
            np.float32)
        x[r, 0] = 448.0 * 2.0 ** int(rng.integers(-8, 8))
    xb = torch.from_numpy(x).to(torch.bfloat16)
    ref_codes, ref_scales = o.quant_rows(xb.view(torch.int16).numpy().view(np.uint16))
    codes = torch.full((rows, 128), 7, dtype=torch.uint8, device="cuda")
    scales = torch.full((rows,), -1.0, dtype=torch.float32, device="cuda")
    qsa.qsa_quantize_rows(xb.cuda(), rows, 128, codes, scales)
    torch.cuda.synchronize()
    assert np.array_equal(scales.cpu().numpy(), ref_scales)
    g = codes.cpu().numpy()
    # +0 and -0 codes of a zero value are the same value
    same = (g == ref_codes) | (((g & 0x7F) == 0) & ((ref_codes & 0x7F) == 0))
    assert same.all(), np.argwhere(~same)[:5]


@pytest.mark.parametrize("q_heads,kv_heads", [(32, 4), (16, 1)])
def test_prefill_with_fp8_caches_matches_oracle(qsa, q_heads, kv_heads):
    """Prefill with the attention on fp8 K/V caches: the selection is the
    bf16 path's; each output row matches the oracle's fp8-cache attention on
    the GPU's own codes, scales and selection (several tiles, ragged tail)."""
    n = 3000 + 37
    w = synth.Workload(name="t", n=n, K=512, q_heads=q_heads, kv_heads=kv_heads, base_seed=0xF8 + q_heads)
    cfg, L = _layer(qsa, w, n)
    _fill_caches(w, L, n)
    L.quantize_kv(0, n)
    iq = dev_full(w, "idx_q", n).view(1, n, 4, 128).contiguous()
    qq = dev_full(w, "q", n).view(1, n, q_heads, 128).contiguous()
    out = torch.empty(1, n, q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(1, n, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(1, n, dtype=torch.int32, device="cuda")
    lse = torch.empty(1, n, q_heads, dtype=torch.float32, device="cuda")
    L.prefill_q8(qq, iq, 0, n, out, sel, nsel, lse)
    torch.cuda.synchronize()
    o = _oracle(w, cfg)
    k8, v8 = L.k8[0].cpu().numpy(), L.v8[0].cpu().numpy()
    ks, vs = L.ks[0].cpu().numpy(), L.vs[0].cpu().numpy()
    # The GPU's quantized caches are the oracle's quantization of the bf16 caches.
    rk, rks = o.quant_rows(bits(L.k_cache)[0, :n].reshape(n, kv_heads, 128))
    assert np.array_equal(rks, ks[:n])
    assert (((rk == k8[:n]) | (((rk & 0x7F) == 0) & ((k8[:n] & 0x7F) == 0)))).all()
    q_bits = bits(qq)[0].reshape(n, q_heads, 128)
    g_out, g_lse = out.float().cpu().numpy()[0], lse.cpu().numpy()[0]
    g_sel, g_n = sel.cpu().numpy()[0], nsel.cpu().numpy()[0]
    rng = np.random.default_rng(n)
    for i in sorted(set(rng.integers(0, n, 24).tolist() + [0, 1, 3, 2047, 2048, n - 1])):
        toks = o.token_set(g_sel[i, : g_n[i]], i)
        ref, ref_lse = o.attention_q8(q_bits[i], k8, ks, v8, vs, toks)
        check_attention(g_out[i], ref, f"row {i}")
        assert np.abs(g_lse[i] - ref_lse).max() <= LSE_ATOL, i


def test_decode_steps_with_fp8_caches_match_oracle(qsa, decode_kernel):
    """Decode on fp8 caches, step by step across block boundaries: the appended
    K/V rows and each newly pooled block are quantized exactly as the oracle
    does; the selection is the oracle's on the fp8 pooled keys (near-ties
    aside); the output matches the oracle's fp8-cache attention."""
    from gpu_util import SCORE_COND_ATOL, SCORE_RTOL

    from block_sparse_long_02_b200.layer import QSALayer

    n0, S = 3001, 9
    w = synth.Workload(name="t", n=n0, batch=2, decode_steps=S, prefill=False, K=512, q_heads=32, kv_heads=4,
                       base_seed=0xF9)
    B = w.batch
    cfg = qsa.Config.of(w)
    cap = n0 + S + 3
    L = QSALayer(cfg, B, cap)
    _fill_caches(w, L, n0)
    L.compress(0, n0 // cfg.r)
    L.quantize_kv(0, n0)
    L.quantize_pooled(0, n0 // cfg.r)
    full = {nm: dev_full(w, nm, cap, n0 + S) for nm in ("q", "k", "v", "idx_q", "idx_k")}
    o = _oracle(w, cfg)
    out = torch.empty(B, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(B, dtype=torch.int32, device="cuda")
    for step in range(S):
        p = n0 + step
        pos = torch.full((B,), p, dtype=torch.int64, device="cuda")
        args = [full[nm][:, p].contiguous() for nm in ("q", "k", "v", "idx_q", "idx_k")]
        L.decode_step_q8(pos, *args, out, sel, nsel)
        torch.cuda.synchronize()
        assert qsa.qsa_workspace_status(L.workspace(qsa.OP_DECODE_STEP)) == 0
        k8, v8, ks, vs = (t.cpu().numpy() for t in (L.k8, L.v8, L.ks, L.vs))
        p8, ps = L.pooled8.cpu().numpy(), L.pscale.cpu().numpy()
        pooled = bits(L.pooled)
        g_out, g_sel, g_n = out.float().cpu().numpy(), sel.cpu().numpy(), nsel.cpu().numpy()
        for s in range(B):
            hs = {nm: w.host_full(nm, s, n0 + S) for nm in ("q", "k", "v", "idx_q")}
            for src, c8, sc in ((hs["k"], k8, ks), (hs["v"], v8, vs)):  # appended rows
                rc, rs = o.quant_rows(src[p].reshape(cfg.kv_heads, 128))
                assert np.array_equal(rs, sc[s, p]) and np.array_equal(rc, c8[s, p]), (s, p)
            if (p + 1) % cfg.r == 0:  # the block the token closed
                b = p // cfg.r
                rc, rs = o.quant_rows(pooled[s, b:b + 1])
                assert np.array_equal(rs, ps[s, b:b + 1]) and np.array_equal(rc, p8[s, b:b + 1]), (s, b)
            nvis = p // cfg.r
            qrot = o.rotate_query(hs["idx_q"][p].reshape(4, 128), p)
            ref = o.scores_q8(qrot, p8[s], ps[s], nvis)
            kd = o.dequant(p8[s, :nvis], ps[s, :nvis])
            tol = SCORE_RTOL * np.abs(ref.astype(np.float64)) + SCORE_COND_ATOL * (
                np.abs(kd) @ np.abs(f32(qrot).astype(np.float64)).T).sum(axis=1)
            check_selection(g_sel[s], g_n[s], ref, tol, o.k_blocks, f"s{s} p{p}")
            toks = o.token_set(g_sel[s, : g_n[s]], p)
            ref_out, _ = o.attention_q8(hs["q"][p], k8[s], ks[s], v8[s], vs[s], toks)
            check_attention(g_out[s], ref_out.reshape(cfg.q_heads, 128), f"s{s} p{p}")


# ----------------------------------------------------------------------------- host-offloaded K/V
@pytest.mark.parametrize("n0,S,H,batch", [(9002, 8, 97, 2), (4097, 6, 61, 24)])
def test_decode_offload_matches_hbm_decode_bit_for_bit(qsa, n0, S, H, batch, decode_kernel):
    """K/V caches in pinned host memory with a small direct-mapped HBM hot
    cache (a prime number of slots, so selected blocks collide): every step's
    selection and output match the oracle on sampled sequences and equal the
    all-HBM decode's bit for bit; the appended
    rows reach host memory; every tagged hot slot holds a copy of its block.
    The same query for every step makes later steps hit blocks installed by
    earlier ones. The larger batch runs fewer warps per sequence, so a warp
    holds more than 32 selection entries (their tags are looked up when
    their chunks are issued)."""
    from block_sparse_long_02_b200.layer import QSALayer

    # n0 inside a block: the first steps read the tail from host memory
    w = synth.Workload(name="t", n=n0, batch=batch, decode_steps=S, prefill=False, K=2048, q_heads=32, kv_heads=4,
                       base_seed=0xFA)
    B = w.batch
    cfg = qsa.Config.of(w)
    cap = -(-(n0 + S + 8) // cfg.r) * cfg.r  # a multiple of r
    full = {nm: dev_full(w, nm, cap, n0 + S) for nm in ("q", "k", "v", "idx_q", "idx_k")}

    def make():
        L = QSALayer(cfg, B, cap)
        _fill_caches(w, L, n0)
        L.compress(0, n0 // cfg.r)
        return L

    La, Lb = make(), make()
    Lb.offload_kv(H)
    o = _oracle(w, cfg)
    seqs = sorted({0, B // 2, B - 1})
    T = n0 + S
    host = {s: {nm: w.host_full(nm, s, T) for nm in ("q", "k", "v", "idx_q")} for s in seqs}
    hits_seen = False
    for step in range(S):
        p = n0 + step
        pos = torch.full((B,), p, dtype=torch.int64, device="cuda")
        q = full["q"][:, n0].contiguous()          # the same query every step
        iq = full["idx_q"][:, n0].contiguous()
        k, v, ik = (full[nm][:, p].contiguous() for nm in ("k", "v", "idx_k"))
        outs, sels, nsels = [], [], []
        for L, fn in ((La, La.decode_step), (Lb, Lb.decode_step_offload)):
            out = torch.empty(B, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
            sel = torch.empty(B, cfg.k_blocks, dtype=torch.int32, device="cuda")
            nsel = torch.empty(B, dtype=torch.int32, device="cuda")
            tags_before = Lb.hot_tags.clone()
            fn(pos, q, k, v, iq, ik, out, sel, nsel)
            torch.cuda.synchronize()
            outs.append(out)
            sels.append(sel)
            nsels.append(nsel)
        assert torch.equal(outs[0], outs[1]), step
        assert torch.equal(nsels[0], nsels[1]), step
        assert torch.equal(sels[0], sels[1]), step
        # The offloaded step against the oracle: the selection on the GPU's
        # pooled keys, the attention on the caches' values over that selection.
        g_sel, g_out, g_pooled = sels[1].cpu().numpy(), outs[1].float().cpu().numpy(), bits(Lb.pooled)
        for s in seqs:
            hs = host[s]
            iq_row = hs["idx_q"][n0].reshape(4, 128)
            ref = o.row(p, iq_row, g_pooled[s])
            tol = score_tol(o.rotate_query(iq_row, p), g_pooled[s], ref["scores"])
            m = int(nsels[1][s].item())
            check_selection(g_sel[s], m, ref["scores"], tol, cfg.k_blocks, f"offload s{s} p{p}")
            toks = o.token_set(g_sel[s, :m], p)
            out_ref, _ = o.attention(hs["q"][n0], hs["k"], hs["v"], toks)
            check_attention(g_out[s], out_ref.reshape(cfg.q_heads, 128), f"offload s{s} p{p}")
        # blocks this step found in the hot cache
        sb = sels[1].long()
        slot = sb.clamp(min=0) % H
        hit = (tags_before.gather(1, slot) == sels[1]) & (sels[1] >= 0)
        hits_seen = hits_seen or bool(hit.any())
        assert qsa.qsa_workspace_status(Lb.workspace(qsa.OP_DECODE_STEP)) == 0
    assert hits_seen
    assert torch.equal(Lb.host_k.cuda(), La.k_cache) and torch.equal(Lb.host_v.cuda(), La.v_cache)
    tags = Lb.hot_tags.cpu().numpy()
    hk, hv = Lb.hot_k.cpu(), Lb.hot_v.cpu()
    ck, cv = Lb.host_k.view(B, cap // cfg.r, cfg.r, cfg.kv_heads, 128), Lb.host_v.view(B, cap // cfg.r, cfg.r,
                                                                                       cfg.kv_heads, 128)
    n_tagged = 0
    for s in range(B):
        for sl in range(H):
            b = int(tags[s, sl])
            if b < 0:
                continue
            n_tagged += 1
            assert b % H == sl
            assert torch.equal(hk[s, sl], ck[s, b]) and torch.equal(hv[s, sl], cv[s, b]), (s, sl, b)
        # the tail slot: the last step's block, rows up to its position (the
        # steps ran from n0, so they opened that block when n0 + S - 1 crossed
        # a block boundary after n0)
        p_last = n0 + S - 1
        cur = p_last // cfg.r
        expect = cur if cur * cfg.r >= n0 else -1
        assert int(tags[s, H]) == expect, (s, int(tags[s, H]), expect)
        if expect >= 0:
            e = p_last % cfg.r + 1
            assert torch.equal(hk[s, H, :e], ck[s, cur, :e]) and torch.equal(hv[s, H, :e], cv[s, cur, :e])
    assert n_tagged > 0
