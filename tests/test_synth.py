"""The seeded input generator shared by both sides (no layer arithmetic in it)."""
import numpy as np
import pytest

import synth


def test_host_draws_are_reproducible_and_row_addressable():
    a = synth.fill_host(123, 4, 0, 4096)
    b = synth.fill_host(123, 4, 0, 4096)
    assert np.array_equal(a, b)
    rows = synth.fill_rows_host(123, 4, [3, 0, 7], 512)
    assert np.array_equal(rows[0], a[3 * 512:4 * 512])
    assert np.array_equal(rows[1], a[:512])
    assert np.array_equal(rows[2], a[7 * 512:8 * 512])
    assert not np.array_equal(synth.fill_host(124, 4, 0, 64), a[:64])
    assert not np.array_equal(synth.fill_host(123, 5, 0, 64), a[:64])
    # every tensor of a workload has its own stream (distinct ids)
    assert len(set(synth.TENSOR_IDS.values())) == len(synth.TENSOR_IDS)


def test_host_draws_look_standard_normal():
    x = synth.bf16_bits_to_f32(synth.fill_host(7, 1, 0, 1 << 20)).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1.0) < 5e-3
    assert np.abs(x).max() <= 6.0
    # Irwin-Hall values are multiples of 2^-16 (so sums of 4 are exact in fp32).
    assert np.array_equal(np.round(x * 65536), x * 65536)


def test_needles_are_disjoint_visible_and_planted():
    w = synth.WORKLOADS["prefill_n128k"]
    nd = w.needles(0)
    assert len(nd) == 64 and len({b for b, _ in nd}) == 64
    assert all(w.r * (b + 1) <= p < w.n for b, p in nd)
    rows = w.needle_rows(0)
    b, p = nd[0]
    got = w.host_rows("idx_k", 0, [w.r * b])[0]
    assert np.array_equal(got, rows[w.r * b])
    f = synth.bf16_bits_to_f32(got)
    assert (f[:64] == 0).all() and abs(np.linalg.norm(f[64:]) - 32.0) < 0.2
    d = synth.WORKLOADS["prefill_n1m_decode64"].needles(0)
    assert len(d) == 128 and sum(p >= 1048576 for _, p in d) == 64


@pytest.mark.gpu
def test_device_generator_matches_host_bit_for_bit():
    import torch

    w = synth.WORKLOADS["tiny_prefill_n256"]
    for name in ("idx_q", "idx_k", "q", "k", "v", "dout"):
        t = torch.zeros(1, w.total, w.row_len(name), dtype=torch.bfloat16, device="cuda")
        w.device_fill(name, t)
        torch.cuda.synchronize()
        got = t.view(torch.int16).cpu().numpy().view(np.uint16)[0]
        assert np.array_equal(got, w.host_full(name, 0)), name
    big = torch.empty(1 << 22, dtype=torch.bfloat16, device="cuda")
    synth.fill_device(99, 3, 1 << 30, big.numel(), big.data_ptr())
    torch.cuda.synchronize()
    idx = np.random.default_rng(0).integers(0, big.numel(), 4096)
    got = big.view(torch.int16).cpu().numpy().view(np.uint16)[idx]
    want = np.array([synth.fill_host(99, 3, (1 << 30) + int(i), 1)[0] for i in idx])
    assert np.array_equal(got, want)


def test_device_fill_rejects_rows_outside_the_tensor():
    """Rows are absolute positions: a buffer that holds fewer rows is refused
    on the host, before any device write."""
    import torch

    w = synth.WORKLOADS["tiny_prefill_n256"]
    t = torch.empty(1, 16, w.row_len("q"), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        w.device_fill("q", t, rows=(200, 216))
