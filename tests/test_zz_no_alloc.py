"""qsa_decode_step_noalloc: the decode step for callers that cannot allocate
device memory (pool-owning serving engines, plugin hosts without an allocator,
loops that cannot take cudaMalloc's synchronisation). It uses the library's
fixed device scratch instead of a workspace; here it must give what the
workspace entry point gives, call after call.

Kept in its own file, collected last, so that a failure here stops a `-x` run
only after every other test has run."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import bits, dev_full

pytestmark = pytest.mark.gpu


def _setup(qsa, w, start):
    from block_sparse_long_02_b200.layer import QSALayer

    cfg = qsa.Config.of(w)
    B = w.batch
    cap = start + w.decode_steps + 4
    T = start + w.decode_steps
    full = {n: dev_full(w, n, cap, T) for n in ("q", "k", "v", "idx_q", "idx_k")}
    layers = []
    for _ in range(2):
        L = QSALayer(cfg, B, cap)
        for n, c in (("k", L.k_cache), ("v", L.v_cache), ("idx_k", L.idx_k_cache)):
            c.view(B, cap, -1)[:, :start] = full[n][:, :start]
        L.compress(0, start // cfg.r)
        layers.append(L)
    return cfg, cap, full, layers


def test_noalloc_decode_matches_workspace_decode_two_calls():
    import block_sparse_long_02_b200 as qsa

    w = synth.Workload(name="noalloc", n=1022, batch=2, decode_steps=2, prefill=False, K=256, q_heads=16,
                       kv_heads=2, base_seed=0x6E6F61, n_needles_decode=2)
    start = 1022  # the second step (position 1023) closes block 255 and pools it
    cfg, cap, full, (L_ws, L_na) = _setup(qsa, w, start)
    B = w.batch
    ar = torch.arange(B, device="cuda")
    outs = [torch.empty(B, cfg.q_heads, 128, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    sels = [torch.empty(B, cfg.k_blocks, dtype=torch.int32, device="cuda") for _ in range(2)]
    nsels = [torch.empty(B, dtype=torch.int32, device="cuda") for _ in range(2)]
    for step in range(2):
        pos = torch.full((B,), start + step, dtype=torch.int64, device="cuda")
        args = [full[n][ar, pos].contiguous() for n in ("q", "k", "v", "idx_q", "idx_k")]
        L_ws.decode_step(pos, *args, outs[0], sels[0], nsels[0])
        qsa.qsa_decode_step_noalloc(cfg, B, pos, *args, L_na.k_cache, L_na.v_cache, L_na.idx_k_cache,
                                    L_na.pooled, cap, None, outs[1], sels[1], nsels[1])
        torch.cuda.synchronize()
        assert torch.equal(nsels[0], nsels[1]), step
        assert torch.equal(sels[0], sels[1]), step
        # The same deterministic kernels on the same values: equal bit for bit.
        assert torch.equal(outs[0], outs[1]), step
        for a, b in ((L_ws.k_cache, L_na.k_cache), (L_ws.v_cache, L_na.v_cache),
                     (L_ws.idx_k_cache, L_na.idx_k_cache)):
            assert torch.equal(a, b), step
        assert np.array_equal(bits(L_ws.pooled), bits(L_na.pooled)), step
    # The block closed by the second call was pooled.
    assert bits(L_na.pooled)[:, 255].any()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import block_sparse_long_02_b200 as qsa

    cfg = qsa.Config()
    t = torch.zeros(1 << 10, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(64, dtype=torch.int64, device="cuda")
    with pytest.raises(qsa.QSAError) as e:
        qsa.qsa_decode_step_noalloc(cfg, 64, pos, t, t, t, t, t, t, t, t, t, 1 << 22, None, t)
    assert e.value.status == 3
    assert "noalloc" in str(e.value) and "scratch" in str(e.value)


def test_noalloc_bad_argument_queues_no_work():
    """A bad argument (here a NULL query) is reported before the fixed scratch
    is touched: a stream captured around the failing call records no work at
    all, not even the clearing of the scratch's state."""
    import block_sparse_long_02_b200 as qsa
    from cuda.bindings import runtime as rt

    cfg = qsa.Config()
    B, cap = 1, 64
    z = lambda *shape: torch.zeros(*shape, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    pos = torch.tensor([9], dtype=torch.int64, device="cuda")
    q, kv, iq, ik = z(B, cfg.q_heads, 128), z(B, cfg.kv_heads, 128), z(B, 4, 128), z(B, 128)
    kc, vc, ikc, pooled = z(B, cap, cfg.kv_heads, 128), z(B, cap, cfg.kv_heads, 128), z(B, cap, 128), z(B, cap // 4, 128)
    out = z(B, cfg.q_heads, 128)
    # A valid call first: the first call in a context loads the device code.
    qsa.qsa_decode_step_noalloc(cfg, B, pos, q, kv, kv, iq, ik, kc, vc, ikc, pooled, cap, None, out)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    (err,) = rt.cudaStreamBeginCapture(s.cuda_stream, rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
    assert err == rt.cudaError_t.cudaSuccess
    try:
        with pytest.raises(qsa.QSAError) as e:
            qsa.qsa_decode_step_noalloc(cfg, B, pos, None, kv, kv, iq, ik, kc, vc, ikc, pooled, cap, None, out,
                                        stream=s)
    finally:
        err, graph = rt.cudaStreamEndCapture(s.cuda_stream)
    assert err == rt.cudaError_t.cudaSuccess
    assert e.value.status == 1 and "q" in str(e.value)
    err, _, n_nodes = rt.cudaGraphGetNodes(graph, 0)
    assert err == rt.cudaError_t.cudaSuccess
    rt.cudaGraphDestroy(graph)
    assert n_nodes == 0
