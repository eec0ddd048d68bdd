"""Parity at the measured workloads' full sizes, in the launch configuration
bench.py times (QSALayer: qsa_compress_keys -> fused qsa_topk_blocks ->
qsa_sparse_attention for prefill; qsa_decode_step for decode).

The oracle recomputes sampled rows one by one (scores over every visible block,
selection, attention over the selected tokens, fetching only the K/V rows it
needs); every row of the GPU output is checked against the invariants that
hold at any size (selection count, range, order, padding; needle recall)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bits, check_attention, check_selection, score_tol

pytestmark = pytest.mark.gpu


def _oracle(w):
    return oracle.Oracle.for_workload(w)


def check_all_rows_invariants(sel: torch.Tensor, nsel: torch.Tensor, q_begin: int, r: int, kB: int,
                              chunk: int = 1 << 16):
    """Every row: nsel = min(k_B, floor(i/r)); entries strictly ascending in
    [0, floor(i/r)); -1 padding after nsel. (Checked in row chunks.)"""
    for j0 in range(0, sel.shape[0], chunk):
        _invariants(sel[j0:j0 + chunk].cpu().numpy(), nsel[j0:j0 + chunk].cpu().numpy(), q_begin + j0, r, kB)


def _invariants(sel: np.ndarray, nsel: np.ndarray, q_begin: int, r: int, kB: int):
    nq = sel.shape[0]
    i = q_begin + np.arange(nq)
    vis = i // r
    want = np.minimum(kB, vis)
    assert np.array_equal(nsel, want), np.nonzero(nsel != want)[0][:5]
    cols = np.arange(kB)[None, :]
    valid = cols < want[:, None]
    assert (sel[~valid] == -1).all()
    v = np.where(valid, sel, 0)
    assert (v[valid] >= 0).all() and (np.where(valid, sel, -1) < vis[:, None]).all()
    d = np.diff(np.where(valid, sel, np.iinfo(np.int32).max), axis=1)
    both = valid[:, 1:] & valid[:, :-1]
    assert (d[both] > 0).all()


def oracle_row_check(w, o, s, i, idx_q_row, q_row, pooled_gpu, sel_row, nsel_i, out_row, what):
    ref = o.row(i, idx_q_row, pooled_gpu)
    tol = score_tol(o.rotate_query(idx_q_row, i), pooled_gpu, ref["scores"])
    check_selection(sel_row, nsel_i, ref["scores"], tol, o.k_blocks, what)
    toks = o.token_set(sel_row[:nsel_i], i)
    kc = w.host_rows("k", s, toks)
    vc = w.host_rows("v", s, toks)
    out_ref, _ = o.attention(q_row, kc, vc, np.arange(toks.size, dtype=np.int64))
    check_attention(out_row, out_ref, what)


def _prefill(w, device="cuda"):
    import block_sparse_long_02_b200 as qsa
    from block_sparse_long_02_b200.layer import QSALayer

    cfg = qsa.Config.of(w)
    B, n, S = w.batch, w.n, w.decode_steps
    cap = -(-(n + S) // w.r) * w.r
    L = QSALayer(cfg, B, cap, device=device)
    w.device_fill("k", L.k_cache.view(B, cap, -1), rows=(0, n))
    w.device_fill("v", L.v_cache.view(B, cap, -1), rows=(0, n))
    w.device_fill("idx_k", L.idx_k_cache, rows=(0, n))
    q = torch.empty(B, n, cfg.q_heads, cfg.head_dim, dtype=torch.bfloat16, device=device)
    iq = torch.empty(B, n, cfg.idx_heads, cfg.idx_dim, dtype=torch.bfloat16, device=device)
    w.device_fill("q", q.view(B, n, -1), rows=(0, n))
    w.device_fill("idx_q", iq.view(B, n, -1), rows=(0, n))
    out = torch.empty_like(q)
    sel = torch.empty(B, n, cfg.k_blocks, dtype=torch.int32, device=device)
    nsel = torch.empty(B, n, dtype=torch.int32, device=device)
    L.prefill(q, iq, 0, n, out, sel, nsel)
    torch.cuda.synchronize()
    return cfg, L, q, iq, out, sel, nsel


def _sample_rows(w, count, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.integers(w.r * (w.k_blocks + 1), w.n, count).tolist())
    rows |= {w.n - 1, w.r * w.k_blocks, w.r * w.k_blocks + w.r - 1, 3, 4 * 37 + 2}
    return sorted(rows)


def _check_prefill(w, cfg, L, q, iq, out, sel, nsel, rows, needles):
    o = _oracle(w)
    s = 0
    check_all_rows_invariants(sel[s], nsel[s], 0, w.r, cfg.k_blocks)
    probe_rows = sorted(set(rows) | {p for _, p in needles if p < w.n})
    pr = torch.tensor(probe_rows, device=sel.device)
    g_sel = dict(zip(probe_rows, sel[s, pr].cpu().numpy()))
    g_nsel = dict(zip(probe_rows, nsel[s, pr].cpu().numpy()))
    # Needles: each probe selects its planted block.
    for b, p in needles:
        if p < w.n:
            assert b in set(g_sel[p][: g_nsel[p]].tolist()), (b, p)
    pooled = bits(L.pooled)[s, : w.n // w.r]
    idx_q = w.host_rows("idx_q", s, rows).reshape(len(rows), 4, 128)
    q_rows = w.host_rows("q", s, rows).reshape(len(rows), cfg.q_heads, 128)
    out_rows = out[s, torch.tensor(rows, device=out.device)].float().cpu().numpy()
    for k, i in enumerate(rows):
        oracle_row_check(w, o, s, i, idx_q[k], q_rows[k], pooled, g_sel[i], int(g_nsel[i]), out_rows[k],
                         f"{w.name} row {i}")
    # The GPU's pooled keys match the oracle's on a sample of blocks (<= 1 ulp).
    nb = w.n // w.r
    blocks = np.unique(np.concatenate([np.arange(64), np.random.default_rng(5).integers(0, nb, 512), [nb - 1]]))
    for b in blocks[::16]:
        raw = w.host_rows("idx_k", s, np.arange(w.r * b, w.r * b + w.r))
        ref = o.pool_block(raw, w.r * b)["out"]
        assert np.abs(ref.astype(np.int32) - pooled[b].astype(np.int32)).max() <= 1, b
    return o


@pytest.mark.parametrize("kernel", [0, 1], ids=["warp_tiles", "tcgen05_tiles"])
def test_prefill_128k_full_size(kernel):
    import block_sparse_long_02_b200 as qsa

    qsa.qsa_set_attention_kernel(kernel)
    try:
        _prefill_128k()
    finally:
        qsa.qsa_set_attention_kernel(0)


def _prefill_128k():
    w = synth.WORKLOADS["prefill_n128k"]
    cfg, L, q, iq, out, sel, nsel = _prefill(w)
    rows = _sample_rows(w, 24, 1) + sorted({p for _, p in w.needles(0)})[:16]
    _check_prefill(w, cfg, L, q, iq, out, sel, nsel, sorted(set(rows)), w.needles(0))


def _decode_inputs(w, L, s_idx, step):
    """New-token tensors [batch][...] for decode step `step` (position n + step)."""
    B = w.batch
    p = w.n + step
    out = {}
    for name in ("q", "k", "v", "idx_q", "idx_k"):
        t = torch.empty(B, w.row_len(name), dtype=torch.bfloat16, device="cuda")
        for s in range(B):
            synth.fill_device(w.seed(s), synth.TENSOR_IDS[name], p * w.row_len(name), w.row_len(name),
                              t[s].data_ptr())
        out[name] = t
    return out


def _check_decode_step(w, o, L, step, out, sel, nsel, seqs):
    cfg = L.cfg
    p = w.n + step
    g_sel, g_nsel = sel.cpu().numpy(), nsel.cpu().numpy()
    g_out = out.float().cpu().numpy()
    for s in seqs:
        pooled = bits(L.pooled[s, : p // w.r])
        idx_q = w.host_rows("idx_q", s, [p]).reshape(4, 128)
        q_row = w.host_rows("q", s, [p]).reshape(cfg.q_heads, 128)
        m = int(g_nsel[s])
        assert m == min(cfg.k_blocks, p // w.r)
        assert (g_sel[s, m:] == -1).all() and np.all(np.diff(g_sel[s, :m]) > 0)
        for b, pp in w.needles(s):
            if pp == p:
                assert b in set(g_sel[s, :m].tolist()), (s, b, p)
        oracle_row_check(w, o, s, p, idx_q, q_row, pooled, g_sel[s], m, g_out[s].reshape(cfg.q_heads, 128),
                         f"{w.name} seq {s} step {step}")


def _decode_setup(w):
    import block_sparse_long_02_b200 as qsa
    from block_sparse_long_02_b200.layer import QSALayer

    cfg = qsa.Config.of(w)
    B, n = w.batch, w.n
    cap = -(-(n + w.decode_steps) // w.r) * w.r
    L = QSALayer(cfg, B, cap)
    w.device_fill("k", L.k_cache.view(B, cap, -1), rows=(0, n))
    w.device_fill("v", L.v_cache.view(B, cap, -1), rows=(0, n))
    w.device_fill("idx_k", L.idx_k_cache, rows=(0, n))
    L.compress(0, n // w.r)
    return cfg, L


@pytest.mark.parametrize("name", ["decode_b1_n32k", "decode_b8_n256k"])
def test_decode_full_size(name):
    w = synth.WORKLOADS[name]
    cfg, L = _decode_setup(w)
    B = w.batch
    o = _oracle(w)
    pos = torch.full((B,), w.n, dtype=torch.int64, device="cuda")
    inp = _decode_inputs(w, L, None, 0)
    out = torch.empty(B, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(B, dtype=torch.int32, device="cuda")
    L.decode_step(pos, inp["q"].view(B, -1, 128), inp["k"].view(B, -1, 128), inp["v"].view(B, -1, 128),
                  inp["idx_q"].view(B, 4, 128), inp["idx_k"], out, sel, nsel)
    torch.cuda.synchronize()
    _check_decode_step(w, o, L, 0, out, sel, nsel, range(B))


def test_prefill_1m_then_64_decode_steps_sampled():
    """The benchmark's workload end to end: 1M-token prefill (sampled rows and all
    row invariants), then 64 decode steps (4 of them checked against the oracle)."""
    w = synth.WORKLOADS["prefill_n1m_decode64"]
    cfg, L, q, iq, out, sel, nsel = _prefill(w)
    needles = w.needles(0)
    rows = _sample_rows(w, 6, 2) + sorted({p for _, p in needles if p < w.n})[:4]
    o = _check_prefill(w, cfg, L, q, iq, out, sel, nsel, sorted(set(rows)), needles)
    del q, iq, out, sel, nsel
    torch.cuda.empty_cache()
    B = w.batch
    dout = torch.empty(B, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    dsel = torch.empty(B, cfg.k_blocks, dtype=torch.int32, device="cuda")
    dn = torch.empty(B, dtype=torch.int32, device="cuda")
    for step in range(w.decode_steps):
        pos = torch.full((B,), w.n + step, dtype=torch.int64, device="cuda")
        inp = _decode_inputs(w, L, None, step)
        L.decode_step(pos, inp["q"].view(B, -1, 128), inp["k"].view(B, -1, 128), inp["v"].view(B, -1, 128),
                      inp["idx_q"].view(B, 4, 128), inp["idx_k"], dout, dsel, dn)
        if step in (0, 3, 31, 63):
            torch.cuda.synchronize()
            _check_decode_step(w, o, L, step, dout, dsel, dn, range(B))


def test_train_32k_full_size():
    """The training step bench.py times on train_n32k (forward, sparse-attention
    gradient, stage-1 target, indexer scores, KL), through bench's own Bench.
    Sampled rows against the oracle (dq, target, KL and its gradient); every
    row and token against identities that hold at any size: target rows are
    distributions over the visible blocks, KL >= 0 with a gradient summing to
    0, the dv rows of a kv head sum to the sum of its heads' upstream gradients
    (every P row sums to 1) and the dk rows to 0 (every dS row sums to 0)."""
    import bench

    w = synth.WORKLOADS["train_n32k"]
    b = bench.Bench(w, torch.device("cuda", 0))
    b.step()
    torch.cuda.synchronize()
    p, cfg, n, r = b.pre, b.cfg, w.n, w.r
    o = _oracle(w)
    G, hk = cfg.q_heads // cfg.kv_heads, cfg.kv_heads
    # every row: distributions, zeros past the visible blocks, KL >= 0, sum of dKL/dI = 0
    tgt = p["target"][0]
    vis = torch.arange(n, device="cuda") // r
    cols = torch.arange(p["ld"], device="cuda")[None, :]
    inside = cols < vis[:, None]
    assert (tgt[~inside] == 0).all() and (tgt >= 0).all()
    sums = tgt.double().sum(1)
    assert ((sums - 1).abs()[vis > 0] < 1e-4).all() and (sums[vis == 0] == 0).all()
    assert (p["kl"][0] > -1e-5).all()
    ds_sum = p["dscores"][0].double().sum(1)
    assert (ds_sum.abs() < 1e-4).all()
    # dv / dk column identities per kv head
    dv = p["dv"][0, :n].double().sum(0)                      # [kv][128]
    dk = p["dk"][0, :n].double().sum(0)
    dout = p["dout"][0].double().view(n, hk, G, 128).sum(dim=(0, 2))
    scale_v = p["dout"][0].double().abs().view(n, hk, G, 128).sum(dim=(0, 2))
    assert ((dv - dout).abs() <= 1e-2 * scale_v).all(), (dv - dout).abs().max().item()
    scale_k = p["dk"][0, :n].double().abs().sum(0)
    assert (dk.abs() <= 2e-2 * scale_k + 1e-6).all(), (dk.abs() / scale_k).max().item()
    # sampled rows against the oracle
    rows = _sample_rows(w, 5, 0x7A)
    sel, nsel = p["sel"][0].cpu().numpy(), p["nsel"][0].cpu().numpy()
    dq = p["dq"][0]
    k_all = w.host_full("k", 0, n)
    for i in rows:
        qi = w.host_rows("q", 0, [i]).reshape(cfg.q_heads, 128)
        gi = w.host_rows("dout", 0, [i]).reshape(cfg.q_heads, 128)
        toks = o.token_set(sel[i, :nsel[i]], i)
        kc, vc = w.host_rows("k", 0, toks), w.host_rows("v", 0, toks)
        ref_dq, _, _ = o.attention_backward(qi, kc, vc, np.arange(toks.size, dtype=np.int64), gi)
        got = dq[i].cpu().numpy()
        assert np.abs(got - ref_dq).max() <= 1e-2 * np.abs(ref_dq).max(), f"dq row {i}"
        ref_t = o.distill_target(i, qi, k_all)
        got_t = tgt[i, : i // r].cpu().numpy()
        assert (np.abs(got_t - ref_t) <= 2e-3 * ref_t + 1e-7).all(), f"target row {i}"
        ref_kl, ref_ds = o.distill_kl(got_t.astype(np.float64), p["scores"][0, i, : i // r].cpu().numpy())
        assert abs(p["kl"][0, i].item() - ref_kl) <= 1e-4 * (1 + abs(ref_kl)), f"kl row {i}"
        got_ds = p["dscores"][0, i, : i // r].cpu().numpy()
        big = np.abs(ref_ds).max() if ref_ds.size else 0.0
        assert (np.abs(got_ds - ref_ds) <= 1e-4 * np.abs(ref_ds) + 1e-6 * big + 1e-9).all(), f"dscores row {i}"


def test_decode_offload_full_size():
    """decode_b8_n256k with the K/V caches in pinned host memory behind a
    16384-block hot cache (the configuration bench.py --offload 16384 times),
    through bench's own Bench: on a first step (every block misses) and on the
    same step again (the selected blocks are then hot), the offloaded step's
    selection and output match the oracle on sampled sequences, and equal the
    all-HBM step's bit for bit; the appended rows reach host memory."""
    import bench

    w = synth.WORKLOADS["decode_b8_n256k"]
    dev = torch.device("cuda", 0)
    ha = bench.Bench(w, dev)
    hb = bench.Bench(w, dev, offload=16384)
    d_a, d_b = ha.dec[0], hb.dec[0]
    cfg = hb.cfg
    o = _oracle(w)
    sels = [torch.empty(w.batch, cfg.k_blocks, dtype=torch.int32, device="cuda") for _ in range(2)]
    nsels = [torch.empty(w.batch, dtype=torch.int32, device="cuda") for _ in range(2)]
    for it in range(2):
        ha.L.decode_step(d_a["pos"], d_a["q"], d_a["k"], d_a["v"], d_a["idx_q"], d_a["idx_k"], d_a["out"],
                         sels[0], nsels[0])
        hb.L.decode_step_offload(d_b["pos"], d_b["q"], d_b["k"], d_b["v"], d_b["idx_q"], d_b["idx_k"], d_b["out"],
                                 sels[1], nsels[1])
        torch.cuda.synchronize()
        assert torch.equal(d_a["out"], d_b["out"]), it
        assert torch.equal(sels[0], sels[1]) and torch.equal(nsels[0], nsels[1]), it
        if it == 0:
            assert (hb.L.hot_tags[:, :16384] >= 0).sum().item() > 0  # the first step installed blocks
        _check_decode_step(w, o, hb.L, 0, d_b["out"], sels[1], nsels[1], (0, 3, 7))
    p = w.n
    assert torch.equal(hb.L.host_k[:, p].cuda(), ha.L.k_cache[:, p])
    assert torch.equal(hb.L.host_v[:, p].cuda(), ha.L.v_cache[:, p])


def test_decode_fp8_full_size():
    """decode_b8_n256k on fp8 caches (the configuration bench.py --kv fp8
    times), through bench's own Bench: for sampled sequences, the appended
    rows are quantized exactly as the oracle does, the selection is the
    oracle's on the fp8 pooled keys (near-ties aside) and the output matches
    the oracle's fp8-cache attention."""
    import bench
    from gpu_util import SCORE_COND_ATOL, SCORE_RTOL, f32

    w = synth.WORKLOADS["decode_b8_n256k"]
    b = bench.Bench(w, torch.device("cuda", 0), kv="fp8")
    cfg, L, d = b.cfg, b.L, b.dec[0]
    sel = torch.empty(w.batch, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(w.batch, dtype=torch.int32, device="cuda")
    L.decode_step_q8(d["pos"], d["q"], d["k"], d["v"], d["idx_q"], d["idx_k"], d["out"], sel, nsel)
    torch.cuda.synchronize()
    o = _oracle(w)
    p = w.n
    nvis = p // cfg.r
    g_out, g_sel, g_n = d["out"].float().cpu().numpy(), sel.cpu().numpy(), nsel.cpu().numpy()
    for s in (0, 5):
        k8, v8 = L.k8[s].cpu().numpy(), L.v8[s].cpu().numpy()
        ks, vs = L.ks[s].cpu().numpy(), L.vs[s].cpu().numpy()
        p8, ps = L.pooled8[s].cpu().numpy(), L.pscale[s].cpu().numpy()
        for name, c8, sc in (("k", k8, ks), ("v", v8, vs)):  # the appended row
            row = w.host_rows(name, s, [p]).reshape(cfg.kv_heads, 128)
            rc, rs = o.quant_rows(row)
            assert np.array_equal(rs, sc[p]) and np.array_equal(rc, c8[p]), (s, name)
        qrot = o.rotate_query(w.host_rows("idx_q", s, [p]).reshape(4, 128), p)
        ref = o.scores_q8(qrot, p8, ps, nvis)
        kd = o.dequant(p8[:nvis], ps[:nvis])
        tol = SCORE_RTOL * np.abs(ref.astype(np.float64)) + SCORE_COND_ATOL * (
            np.abs(kd) @ np.abs(f32(qrot).astype(np.float64)).T).sum(axis=1)
        check_selection(g_sel[s], g_n[s], ref, tol, o.k_blocks, f"s{s}")
        toks = o.token_set(g_sel[s, : g_n[s]], p)
        ref_out, _ = o.attention_q8(w.host_rows("q", s, [p])[0], k8, ks, v8, vs, toks)
        check_attention(g_out[s], ref_out.reshape(cfg.q_heads, 128), f"s{s}")
