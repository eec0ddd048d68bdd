"""The decode step as one persistent kernel (qsa_set_decode_kernel(0)):
launch shapes whose CTA bookkeeping differs (one CTA per sequence
over two waves, fewer CTAs per sequence than kv heads, a split count that does
not divide the CTAs), the same selection as the three-kernel path bit for bit,
the failure path of its bounded inter-CTA waits, and the listed-block
pre-filter of its selection (the pick never depends on the estimate)."""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import bits, check_attention, check_selection, dev_full, score_tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_02_b200 as m

    m.qsa_set_decode_kernel(m.DECODE_STEP_KERNEL)
    yield m
    m.qsa_set_decode_kernel(m.DECODE_THREE_KERNELS)


def _setup(qsa, n, batch, K, q_heads, kv_heads, seed):
    """A layer whose caches hold n tokens per sequence, and the inputs of the
    step at position n."""
    from block_sparse_long_02_b200.layer import QSALayer

    w = synth.Workload(name="t", n=n, batch=batch, decode_steps=1, prefill=False, K=K, q_heads=q_heads,
                       kv_heads=kv_heads, base_seed=seed)
    cfg = qsa.Config.of(w)
    cap = n + 8
    L = QSALayer(cfg, batch, cap)
    full = {nm: dev_full(w, nm, cap, n + 1) for nm in ("q", "k", "v", "idx_q", "idx_k")}
    for nm, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
        c.view(batch, cap, -1)[:, :n] = full[nm][:, :n]
    L.compress(0, n // cfg.r)
    step = [full[nm][:, n].contiguous() for nm in ("q", "k", "v", "idx_q", "idx_k")]
    return w, cfg, L, step


def _step(L, cfg, step, n):
    B = L.batch
    pos = torch.full((B,), n, dtype=torch.int64, device="cuda")
    out = torch.empty(B, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, cfg.k_blocks, dtype=torch.int32, device="cuda")
    nsel = torch.empty(B, dtype=torch.int32, device="cuda")
    L.decode_step(pos, *step, out, sel, nsel)
    torch.cuda.synchronize()
    return out, sel, nsel


def _check(w, cfg, L, n, res, seqs):
    out, sel, nsel = (t.cpu() for t in res)
    o = oracle.Oracle(r=cfg.r, K=cfg.K, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads)
    pooled = bits(L.pooled)
    for s in seqs:
        hq = w.host_full("q", s, n + 1).reshape(n + 1, cfg.q_heads, 128)
        hk = w.host_full("k", s, n + 1).reshape(n + 1, cfg.kv_heads, 128)
        hv = w.host_full("v", s, n + 1).reshape(n + 1, cfg.kv_heads, 128)
        iq = w.host_full("idx_q", s, n + 1)[n].reshape(4, 128)
        ref = o.row(n, iq, pooled[s])
        tol = score_tol(o.rotate_query(iq, n), pooled[s], ref["scores"])
        g_sel, g_n = sel.numpy()[s], int(nsel[s])
        check_selection(g_sel, g_n, ref["scores"], tol, o.k_blocks, f"s{s}")
        toks = o.token_set(g_sel[:g_n], n)
        ref_out, _ = o.attention(hq[n], hk, hv, toks)
        check_attention(out.float().numpy()[s], ref_out.reshape(cfg.q_heads, 128), f"s{s}")


@pytest.mark.parametrize("n,batch,K,q_heads,kv_heads", [
    (1201, 160, 256, 16, 2),   # more sequences than SMs: one CTA per sequence, two waves, no waits
    (3001, 40, 512, 32, 4),    # 3 CTAs per sequence for 4 kv heads: CTAs loop over heads
    (3001, 20, 512, 64, 8),    # 7 CTAs per sequence for 8 kv heads
    (20003, 8, 2048, 32, 4),   # 18 CTAs per sequence: 4 splits per kv head, 2 CTAs without attention
    (8191, 1, 512, 8, 1),      # every CTA of the GPU on one sequence, 16 splits of one kv head
])
def test_step_kernel_launch_shapes_match_oracle(qsa, n, batch, K, q_heads, kv_heads):
    w, cfg, L, step = _setup(qsa, n, batch, K, q_heads, kv_heads, 0xD1 + batch)
    res = _step(L, cfg, step, n)
    assert qsa.qsa_workspace_status(L.workspace(qsa.OP_DECODE_STEP)) == 0
    seqs = sorted({0, batch // 2, batch - 1})
    _check(w, cfg, L, n, res, seqs)
    # The step left its state zero: a second identical step gives the same bits.
    res2 = _step(L, cfg, step, n)
    for a, b in zip(res, res2):
        assert torch.equal(a, b)


def test_step_kernel_falls_back_for_groups_above_8(qsa):
    """q_heads / kv_heads = 16 is outside the step kernel (one n8 tile of heads):
    with the step kernel selected the step runs the three kernels, and matches
    the oracle."""
    n, batch = 3001, 2
    w, cfg, L, step = _setup(qsa, n, batch, 512, 64, 4, 0xDE)
    res = _step(L, cfg, step, n)
    assert qsa.qsa_workspace_status(L.workspace(qsa.OP_DECODE_STEP)) == 0
    _check(w, cfg, L, n, res, [0, 1])


@pytest.mark.parametrize("n,batch", [(20003, 8), (5000, 3), (700, 2)])
def test_step_kernel_and_three_kernels_select_the_same_blocks(qsa, n, batch):
    """Same inputs through both decode paths: the selections are equal bit for
    bit (the same scores and the same exact pick); the outputs differ only by
    the fp32 order of the split merges."""
    w, cfg, L, step = _setup(qsa, n, batch, 2048, 32, 4, 0xD7 + n)
    out0, sel0, nsel0 = _step(L, cfg, step, n)
    qsa.qsa_set_decode_kernel(qsa.DECODE_THREE_KERNELS)
    try:
        out1, sel1, nsel1 = _step(L, cfg, step, n)
    finally:
        qsa.qsa_set_decode_kernel(qsa.DECODE_STEP_KERNEL)
    assert torch.equal(sel0, sel1) and torch.equal(nsel0, nsel1)
    d = (out0.float() - out1.float()).abs().max().item()
    assert d <= 2e-2, d
    _check(w, cfg, L, n, (out0, sel0, nsel0), [0, batch - 1])


def test_step_kernel_forced_timeout_is_reported_and_the_context_survives(qsa):
    """Failure path of the step kernel's inter-CTA waits, without a GPU fault:
    fault injection mode 4 makes the last CTA of sequence 0 withhold its arrival
    after the score stream; that sequence's CTAs wait 0.25 s, record QSA_ERR_TIMEOUT
    and skip the rest of the step, while sequence 1 completes normally. After
    the workspace is zeroed the next step is normal and matches the oracle."""
    n, batch = 9001, 2
    w, cfg, L, step = _setup(qsa, n, batch, 512, 32, 4, 0xDD)
    ws = L.workspace(qsa.OP_DECODE_STEP)
    assert qsa.qsa_workspace_status(ws) == 0
    qsa.qsa_set_fault_injection(4, 0.25)
    try:
        t0 = time.time()
        res = _step(L, cfg, step, n)
        elapsed = time.time() - t0
    finally:
        qsa.qsa_set_fault_injection(0)
    assert qsa.qsa_workspace_status(ws) == 6  # QSA_ERR_TIMEOUT (read and cleared)
    assert elapsed >= 0.2
    _check(w, cfg, L, n, res, [1])  # the other sequence was not held up
    ws.zero_()
    res = _step(L, cfg, step, n)
    assert qsa.qsa_workspace_status(ws) == 0
    _check(w, cfg, L, n, res, [0, 1])


# ----------------------------------------------------------------------------- the listed-block pre-filter
LIST_CAP = 4096  # blocks the score pass can list per sequence
FACTOR = 0.8      # threshold = FACTOR x estimate x the query's summed head norms


def _estimates(L, qsa):
    """[batch][2] float32 view of the per-sequence pre-filter estimate in the
    decode workspace: (k-th score per unit of summed head norms, the last
    step's summed norms)."""
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    B, kv = L.batch, L.cfg.kv_heads
    off = 256 + al(B * 2048 * 4) + al(B * 4 * 4) + al(B * (3 + kv) * 4)
    ws = L.workspace(qsa.OP_DECODE_STEP)
    return ws[off: off + 8 * B].view(torch.float32).view(B, 2)


def test_pick_does_not_depend_on_the_estimate(qsa):
    """The score pass lists the blocks at or above an estimated threshold and
    the selection picks from that list alone when it holds at least k_B (then
    it holds every top-k_B block). The same step replayed with estimates that
    list a few more than k_B blocks, exactly about k_B, fewer than k_B, more
    than the list holds, or that are zero, negative, infinite or NaN, gives the
    selection and the output of the step without an estimate, bit for bit."""
    n, B = 4 * 20000 + 3, 2  # 20000 visible blocks, k_B = 512
    w, cfg, L, step = _setup(qsa, n, B, 2048, 32, 4, 0x9F1)
    est = _estimates(L, qsa)
    assert torch.count_nonzero(est) == 0
    res0 = _step(L, cfg, step, n)  # no estimate yet: the full selection
    _check(w, cfg, L, n, res0, [0, 1])
    e = est.cpu().numpy().astype(np.float64)
    assert (e[:, 1] > 0).all()
    o = oracle.Oracle(r=cfg.r, K=cfg.K, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads)
    pooled = bits(L.pooled)
    scores = [o.row(n, w.host_full("idx_q", s, n + 1)[n].reshape(4, 128), pooled[s])["scores"] for s in range(B)]
    kB = cfg.k_blocks
    for s in range(B):  # the recorded estimate: k-th selected score / summed norms
        kth = np.sort(scores[s])[::-1][kB - 1]
        assert abs(e[s, 0] * e[s, 1] - kth) <= 1e-3 * abs(kth), (s, e[s], kth)

    def listing(m):
        """Estimates whose threshold lies between the m-th and (m+1)-th
        largest scores (about m blocks listed)."""
        out = []
        for s in range(B):
            srt = np.sort(scores[s])[::-1]
            out.append(0.5 * (srt[m - 1] + srt[m]) / (FACTOR * e[s, 1]))
        return out

    cases = {
        "recorded": e[:, 0].tolist(),
        "kB_plus_100": listing(kB + 100),
        "about_kB": listing(kB + 1),
        "too_few": listing(kB - 40),
        "overflow": listing(LIST_CAP + 700),
        "zero": [0.0] * B, "negative": [-1.0] * B, "inf": [float("inf")] * B, "nan": [float("nan")] * B,
        "tiny": [1e-30] * B,
    }
    for name, xs in cases.items():
        est[:, 0] = torch.tensor(xs, dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        res = _step(L, cfg, step, n)
        assert qsa.qsa_workspace_status(L.workspace(qsa.OP_DECODE_STEP)) == 0, name
        for a, b in zip(res, res0):
            assert torch.equal(a, b), name


def test_listed_pick_with_exact_ties(qsa):
    """Pooled keys that repeat 5 distinct rows: thousands of blocks tie at the
    k-th score; the pick is the lowest block indices among them on the list
    path as on the full path, with thresholds at and just below each of the
    top score values."""
    n, B = 4 * 3000 + 1, 1
    w, cfg, L, step = _setup(qsa, n, B, 512, 32, 4, 0x9F2)
    nb = n // cfg.r
    L.pooled[0, :nb] = L.pooled[0, :5].clone().repeat((nb + 4) // 5, 1)[:nb]
    res0 = _step(L, cfg, step, n)
    o = oracle.Oracle(r=cfg.r, K=cfg.K, q_heads=cfg.q_heads, kv_heads=cfg.kv_heads)
    sc = o.row(n, w.host_full("idx_q", 0, n + 1)[n].reshape(4, 128), bits(L.pooled)[0])["scores"]
    kB = cfg.k_blocks
    order = np.lexsort((np.arange(sc.size), -sc.astype(np.float64)))
    assert np.array_equal(res0[1].cpu().numpy()[0, :kB], np.sort(order[:kB]))
    est = _estimates(L, qsa)
    y = float(est[0, 1])
    for v in np.unique(sc)[::-1][:4]:
        for tau in (float(v), float(np.nextafter(np.float32(v), np.float32(-np.inf)))):
            est[0, 0] = tau / (FACTOR * y)
            torch.cuda.synchronize()
            res = _step(L, cfg, step, n)
            for a, b in zip(res, res0):
                assert torch.equal(a, b), tau
