"""Pins for the oracle: checks against what the pages and mathematics fix.

Each ``pin_*`` takes a factory ``make(**cfg) -> oracle.Oracle`` and raises
AssertionError when the oracle it builds is wrong. ``test_oracle_pins.py`` runs
them on the oracle; ``test_oracle_mutants.py`` runs them on copies of the oracle
with planted mistakes and requires every mistake to be caught by some pin.

Sources: "QSA (Qwen Sparse Attention)" concept page, "Key math / How it works"
(A) indexer and (B) sparse core attention, "Config"; "Qwen Sparse Attention"
gallery page, "How block selection works" and its budget table.
"""
from __future__ import annotations

import os

import numpy as np

import bruteforce as bfm
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

TINY = synth.Workload(name="pin_tiny", n=256, K=32, q_heads=4, kv_heads=1, base_seed=0x70696E01)
GQA = synth.Workload(name="pin_gqa", n=96, K=16, q_heads=8, kv_heads=2, base_seed=0x70696E02)
NEEDLE = synth.Workload(name="pin_needle", n=8192, K=64, q_heads=4, kv_heads=1,
                        base_seed=0x70696E03, n_needles_prefill=12)


def _inputs(w, seq=0):
    n = w.total
    return (w.host_full("idx_q", seq).reshape(n, w.idx_heads, w.idx_dim),
            w.host_full("idx_k", seq),
            w.host_full("q", seq).reshape(n, w.q_heads, w.head_dim),
            w.host_full("k", seq).reshape(n, w.kv_heads, w.head_dim),
            w.host_full("v", seq).reshape(n, w.kv_heads, w.head_dim))


def _bits(x):
    return bfm.f64_to_bf16(np.asarray(x, dtype=np.float64))


# ----------------------------------------------------------------------------- golden
def pin_budget_golden(make):
    """The gallery page's budget table: a 2,048-token budget with 4-token blocks
    selects up to 512 blocks (k_B = ceil(K/r)); and the selection never holds
    more than k_B blocks."""
    rows = [ln.split("#")[0].split() for ln in open(os.path.join(GOLDEN, "budget.txt"))]
    for row in rows:
        if not row:
            continue
        kv = dict(x.split("=") for x in row)
        o = make(r=int(kv["r"]), K=int(kv["K"]))
        assert o.k_blocks == int(kv["k_B"]), (kv, o.k_blocks)
    o = make(r=4, K=2048)
    rng = np.random.default_rng(1)
    s = rng.standard_normal(5000).astype(np.float32)
    assert o.select(s).size == 512


# ----------------------------------------------------------------------------- bf16 storage
def _f32_patterns_to_f64(bits32):
    with np.errstate(invalid="ignore"):  # NaN patterns are dropped by the caller
        return np.asarray(bits32, dtype=np.uint32).view(np.float32).astype(np.float64)


def pin_bf16_rounding(make):
    """Pooled keys and rotated indexer queries are stored as bf16, rounded once
    to nearest with ties to even. Inputs that fp32 holds exactly are checked
    against torch's float32 -> bfloat16 conversion (a library rounding);
    every input, fp32-exact or not, against a nearest-value search over the
    table of all bf16 values. Cases: exact halfway ties with odd and even last
    kept bits, ties and near-ties that carry into the exponent, signed zeros,
    the subnormal range, the largest finite values and the overflow edge, and
    fp64 values one hair off a tie (fp32 would first round them onto it)."""
    import torch

    o = make()
    rng = np.random.default_rng(16)
    pats = [rng.integers(0, 2 ** 32, 60000, dtype=np.uint64).astype(np.uint32)]
    h = rng.integers(0, 0x7F7F, 4000).astype(np.uint32)
    for low in (0x8000, 0x7FFF, 0x8001, 0x0000, 0xFFFF):
        pats.append((h << 16) | low)
    pats.append(np.array([0x3F7F8000, 0x3F7FFFFF, 0x3FFF8000, 0x3F808000, 0x3F818000,  # carries / ties
                          0x00000000, 0x80000000, 0x00008000, 0x00018000, 0x00017FFF,   # zeros, subnormals
                          0x00000001, 0x007F8000, 0x007FFFFF, 0x00800000,
                          0x7F7F7FFF, 0x7F7F8000, 0x7F7EFFFF, 0x7F7F0000, 0x7F7FFFFF], dtype=np.uint32))
    p32 = np.concatenate(pats)
    p32 = np.concatenate([p32, p32 | np.uint32(0x80000000)])
    x32 = _f32_patterns_to_f64(p32)
    x32 = x32[np.isfinite(x32)]
    got = o.round_bf16(x32)
    lib = torch.from_numpy(x32.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    bad = np.nonzero(got != lib)[0]
    assert bad.size == 0, (x32[bad[:4]], got[bad[:4]], lib[bad[:4]])
    assert np.array_equal(got, bfm.f64_to_bf16(x32))
    # fp64 inputs: random magnitudes over the whole range, and ties shifted by
    # less than fp32's last bit.
    mag = rng.uniform(-140.0, 128.5, 40000)
    x64 = rng.choice([-1.0, 1.0], mag.size) * np.exp2(mag) * (1.0 + rng.random(mag.size) * 2.0 ** -30)
    ties = _f32_patterns_to_f64((h << 16) | np.uint32(0x8000))
    x64 = np.concatenate([x64, ties * (1 + 2.0 ** -40), ties * (1 - 2.0 ** -40), -ties * (1 + 2.0 ** -40)])
    x64 = x64[np.isfinite(x64)]
    assert np.array_equal(o.round_bf16(x64), bfm.f64_to_bf16(x64))
    # a tie nudged up rounds up although its fp32 rounding is the tie itself
    t = float(_f32_patterns_to_f64(np.array([0x3F808000], dtype=np.uint32))[0]) * (1 + 2.0 ** -40)
    assert int(o.round_bf16(np.array([t]))[0]) == 0x3F81


# ----------------------------------------------------------------------------- RoPE
def pin_rope_textbook(make):
    """RoPE = complex rotation z_j * e^{i pos theta_j}, theta_j = base^(-2j/64),
    on dims 0..63 only; position 0 is the identity; each (j, j+32) pair keeps
    its norm; rotations compose (R_a R_b = R_{a+b})."""
    o = make()
    rng = np.random.default_rng(2)
    x = rng.standard_normal(128)
    for pos in (0, 1, 3, 4, 4095, 131068, 1048572):
        got = o.rope(x, pos)
        want = bfm.rope_complex(x, pos, 64, 10000.0)
        assert np.allclose(got, want, rtol=0, atol=1e-9), pos
        assert np.array_equal(got[64:], x[64:])
        assert np.allclose(np.hypot(got[:32], got[32:64]), np.hypot(x[:32], x[32:64]), atol=1e-12)
    assert np.array_equal(o.rope(x, 0), x)
    assert np.allclose(o.rope(o.rope(x, 17), 1000), o.rope(x, 1017), atol=1e-9)


def _basis_angle(vec, j=0):
    return np.arctan2(vec[j + 32], vec[j])


def pin_rope_first_position_of_block(make):
    """The pooled key of block b is rotated at the block's FIRST position r*b
    (gallery page); the indexer query at its own position i. With a key/query
    along dim 0 the rotated pair (0, 32) is (cos(pos), sin(pos)) * norm."""
    o = make()
    e = np.zeros((4, 128))
    e[:, 0] = 1.0
    e[:, 64] = 1.0
    keys = _bits(e)
    for b in (0, 1, 5, 1000):
        res = o.pool_block(keys, pos=4 * b)
        ang = _basis_angle(res["krot"])
        assert abs(np.angle(np.exp(1j * (ang - 4 * b)))) < 1e-9, b
    idx_k = _bits(np.tile(e[0], (4 * 6, 1)))
    pooled = o.compress(idx_k, 6)
    for b in range(6):
        v = bfm.bf16_to_f64(pooled[b])
        ang = _basis_angle(v)
        assert abs(np.angle(np.exp(1j * (ang - 4 * b)))) < 1e-2, (b, ang)
    q = np.zeros((4, 128))
    q[:, 0] = 1.0
    for i in (0, 2, 7, 999):
        qr = bfm.bf16_to_f64(o.rotate_query(_bits(q), i))
        for h in range(4):
            assert abs(np.angle(np.exp(1j * (_basis_angle(qr[h]) - i)))) < 1e-2, (i, h)


# ----------------------------------------------------------------------------- pooling + norm
def pin_pool_mean(make):
    """The pooled key before RMSNorm is the exact mean of the block's r keys:
    keys c + d_t with sum_t d_t = 0 pool to c; order of the keys is irrelevant."""
    o = make()
    rng = np.random.default_rng(3)
    c = np.round(rng.standard_normal(128) * 64) / 64
    d = np.round(rng.standard_normal((2, 128)) * 16) / 64
    keys = np.stack([c + d[0], c - d[0], c + d[1], c - d[1]])
    res = o.pool_block(_bits(keys), pos=0)
    assert np.array_equal(res["kbar"], c)
    perm = o.pool_block(_bits(keys[[2, 0, 3, 1]]), pos=0)
    assert np.array_equal(perm["kbar"], res["kbar"])
    # Needle-style block: 4 identical keys pool to that key.
    same = o.pool_block(_bits(np.tile(c, (4, 1))), pos=0)
    assert np.array_equal(same["kbar"], c)


def pin_rmsnorm_closed_form(make):
    """RMSNorm (w = 1): knorm = kbar / sqrt(ms + eps), so mean(knorm^2) =
    ms / (ms + eps) and knorm is parallel to kbar; the weight scales per dim."""
    o = make()
    rng = np.random.default_rng(4)
    for scale in (1.0, 1e-3):  # at 1e-3 the eps term is half the denominator
        keys = _bits(rng.standard_normal((4, 128)) * scale)
        res = o.pool_block(keys, pos=0)
        ms = np.mean(res["kbar"] ** 2)
        assert np.isclose(np.mean(res["knorm"] ** 2), ms / (ms + 1e-6), rtol=1e-12)
        cos = res["knorm"] @ res["kbar"] / np.linalg.norm(res["knorm"]) / np.linalg.norm(res["kbar"])
        assert np.isclose(cos, 1.0, atol=1e-12)
        wts = rng.uniform(0.5, 2.0, 128).astype(np.float32)
        rw = o.pool_block(keys, pos=0, w=wts)
        assert np.allclose(rw["knorm"], res["knorm"] * wts.astype(np.float64), rtol=1e-12)


# ----------------------------------------------------------------------------- scores
def pin_scores_relu_sum(make):
    """I_ib = sum_h ReLU(<q_i^h, k_b>): with per-head dots (+1, -2, +3, -4) * s
    the score is 4s; scores are >= 0; doubling q doubles I exactly."""
    o = make()
    q = np.zeros((4, 128))
    q[:, 64] = [1.0, -2.0, 3.0, -4.0]
    k = np.zeros((3, 128))
    k[:, 64] = [0.5, 2.0, -1.0]
    s = o.scores(_bits(q), _bits(k), 3)
    assert np.array_equal(s, np.array([0.5 * 4, 2.0 * 4, 1.0 * 6], dtype=np.float32)), s
    rng = np.random.default_rng(5)
    qr = _bits(rng.standard_normal((4, 128)))
    kp = _bits(rng.standard_normal((50, 128)))
    s1 = o.scores(qr, kp, 50)
    assert (s1 >= 0).all()
    s2 = o.scores(_bits(bfm.bf16_to_f64(qr) * 2), kp, 50)
    assert np.array_equal(s2, s1 * 2)
    assert np.array_equal(o.select(s2, 7), o.select(s1, 7))


def pin_block_causal(make):
    """Query i scores only complete blocks b < floor(i/r); blocks at or after
    its own block are never read (poisoned here with NaN)."""
    w = TINY
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    idx_q, idx_k, *_ = _inputs(w)
    pooled = o.compress(idx_k, w.n // w.r)
    for i in (0, 3, 4, 7, 8, 101, 255):
        c = i // w.r
        poisoned = pooled.copy()
        poisoned[c:] = 0x7FC0  # bf16 NaN
        res = o.row(i, idx_q[i], poisoned)
        assert res["scores"].size == c
        assert np.isfinite(res["scores"]).all()


# ----------------------------------------------------------------------------- select
def pin_select_order(make):
    """Top-k_B by (score desc, block asc), returned ascending: equals numpy's
    lexsort; all-equal scores pick the lowest indices; k_B >= visible selects
    all; the set grows monotonically with the budget."""
    o = make()
    rng = np.random.default_rng(6)
    for n, k in ((1, 512), (300, 512), (5000, 512), (2000, 7)):
        s = np.round(rng.standard_normal(n) * 4).astype(np.float32)  # many ties
        s[rng.random(n) < 0.2] = 0.0
        want = np.sort(np.lexsort((np.arange(n), -s.astype(np.float64)))[: min(k, n)])
        assert np.array_equal(o.select(s, k), want), (n, k)
    z = np.zeros(1000, dtype=np.float32)
    assert np.array_equal(o.select(z, 10), np.arange(10))
    s = rng.standard_normal(700).astype(np.float32)
    prev = set()
    for k in range(1, 60):
        cur = set(o.select(s, k).tolist())
        assert prev <= cur and len(cur) == k
        prev = cur


# ----------------------------------------------------------------------------- expand
def pin_token_count(make):
    """|T_i| = r * min(k_B, floor(i/r)) + (i mod r) + 1; every t <= i; no
    duplicates; the tail r*floor(i/r) .. i is always in."""
    w = TINY
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    idx_q, idx_k, *_ = _inputs(w)
    pooled = o.compress(idx_k, w.n // w.r)
    kB = o.k_blocks
    for i in range(w.n):
        res = o.row(i, idx_q[i], pooled, want_scores=False)
        assert res["nsel"] == min(kB, i // w.r), i
        toks = o.token_set(res["sel"], i)
        assert toks.size == w.r * min(kB, i // w.r) + i % w.r + 1, i
        assert toks.max() <= i and np.unique(toks).size == toks.size
        assert set(range(w.r * (i // w.r), i + 1)) <= set(toks.tolist())


# ----------------------------------------------------------------------------- attention
def pin_attention_sdpa(make):
    """Sparse attention on a token set equals torch's scaled_dot_product_attention
    (fp64, CPU) on the gathered keys/values, with GQA heads h -> floor(h/g)."""
    import torch

    w = GQA
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    _, _, q, k, v = _inputs(w)
    rng = np.random.default_rng(7)
    for i in (5, 40, 95):
        toks = np.sort(rng.choice(i + 1, size=min(i + 1, 30), replace=False))
        out, lse = o.attention(q[i], k, v, toks)
        qt = torch.from_numpy(bfm.bf16_to_f64(q[i]))[:, None, :]           # [Hq][1][d]
        kt = torch.from_numpy(bfm.bf16_to_f64(k[toks])).permute(1, 0, 2)   # [Hkv][T][d]
        vt = torch.from_numpy(bfm.bf16_to_f64(v[toks])).permute(1, 0, 2)
        g = w.q_heads // w.kv_heads
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt.repeat_interleave(g, 0), vt.repeat_interleave(g, 0))[:, 0, :].numpy()
        assert np.allclose(out, ref, rtol=0, atol=1e-10), i
        logits = torch.einsum("hd,htd->ht", qt[:, 0], kt.repeat_interleave(g, 0)) / np.sqrt(128)
        assert np.allclose(lse, torch.logsumexp(logits, -1).numpy(), atol=1e-10)


def pin_dense_when_budget_covers(make):
    """When k_B >= the visible complete blocks, QSA is dense causal attention:
    compare with torch's causal SDPA over the whole tiny sequence (K = 1024),
    and rows i < r*(k_B+1) at the tiny config's K = 32."""
    import torch

    w = TINY
    _, idx_k, q, k, v = _inputs(w)
    idx_q = _inputs(w)[0]
    qt = torch.from_numpy(bfm.bf16_to_f64(q)).permute(1, 0, 2)  # [H][n][d]
    kt = torch.from_numpy(bfm.bf16_to_f64(k)).permute(1, 0, 2)
    vt = torch.from_numpy(bfm.bf16_to_f64(v)).permute(1, 0, 2)
    g = w.q_heads // w.kv_heads
    dense = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(g, 0), vt.repeat_interleave(g, 0), is_causal=True)
    dense = dense.permute(1, 0, 2).numpy()
    for K, rows in ((1024, range(0, w.n, 7)), (w.K, range(0, 4 * (8 + 1)))):
        o = make(r=w.r, K=K, q_heads=w.q_heads, kv_heads=w.kv_heads)
        pooled = o.compress(idx_k, w.n // w.r)
        for i in rows:
            res = o.row(i, idx_q[i], pooled, q[i], k, v, want_scores=False)
            assert np.allclose(res["out"], dense[i], rtol=0, atol=1e-9), (K, i)


def pin_bruteforce_dense_mask(make):
    """Every step on the tiny workload equals the dense brute force of
    tests/bruteforce.py: pooled keys (bit-exact), scores, the selected block
    sets (exact) and the attention output through a [n x n] mask."""
    w = TINY
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    idx_q, idx_k, q, k, v = _inputs(w)
    ref = bfm.layer(w, idx_q, idx_k, q, k, v)
    pooled = o.compress(idx_k, w.n // w.r)
    assert np.array_equal(pooled, ref["pooled"])
    for i in range(w.n):
        res = o.row(i, idx_q[i], pooled, q[i], k, v)
        c = i // w.r
        assert np.array_equal(o.rotate_query(idx_q[i], i), ref["qrot"][i])
        assert np.allclose(res["scores"], ref["scores"][i, :c], rtol=1e-6, atol=0), i
        assert np.array_equal(res["sel"], np.nonzero(ref["block_sel"][i])[0]), i
        assert np.allclose(res["out"], ref["out"][i], rtol=0, atol=1e-9), i
        assert np.allclose(res["lse"], ref["lse"][i], rtol=0, atol=1e-9), i


def pin_needle_recall(make):
    """Each planted needle block (keys along its probe query's direction, x4) is
    selected by its probe query, with budget to spare for the other blocks."""
    w = NEEDLE
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    idx_k = w.host_full("idx_k", 0)
    pooled = o.compress(idx_k, w.n // w.r)
    needles = w.needles(0)
    probes = sorted({p for _, p in needles})
    iq = w.host_rows("idx_q", 0, probes).reshape(len(probes), w.idx_heads, w.idx_dim)
    for p, qrow in zip(probes, iq):
        res = o.row(p, qrow, pooled)
        want = {b for b, pp in needles if pp == p}
        assert want <= set(res["sel"].tolist()), p
        top = np.argsort(-res["scores"], kind="stable")[: len(want)]
        assert set(top.tolist()) == want, p


def pin_decode_matches_prefill_row(make):
    """A decode step at position p (append, then query p, then pool the block it
    closes) gives the prefill row p's selection and output, and leaves the
    pooled cache equal to pooling the sequence."""
    w = GQA
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    idx_q, idx_k, q, k, v = _inputs(w)
    n0 = 80
    kc = np.zeros_like(k)
    vc = np.zeros_like(v)
    ikc = np.zeros_like(idx_k)
    kc[:n0], vc[:n0], ikc[:n0] = k[:n0], v[:n0], idx_k[:n0]
    pooled = np.zeros((w.n // w.r, w.idx_dim), dtype=np.uint16)
    pooled[: n0 // w.r] = o.compress(idx_k, n0 // w.r)
    full_pooled = o.compress(idx_k, w.n // w.r)
    for p in range(n0, w.n):
        res = o.decode_step(p, q[p], k[p], v[p], idx_q[p], idx_k[p], kc, vc, ikc, pooled)
        ref = o.row(p, idx_q[p], full_pooled, q[p], k, v, want_scores=False)
        assert np.array_equal(res["sel"], ref["sel"]), p
        assert np.allclose(res["out"], ref["out"], rtol=0, atol=1e-12), p
    assert np.array_equal(pooled, full_pooled)


# ---------------------------------------------------------------- fp8 caches
# Reading (the pages name a quantized variant but not its format): OCP FP8 E4M3
# codes with one fp32 scale per row, scale = fl32(max|x| / 448).

def pin_e4m3_codec_matches_library(make):
    """Every code decodes, and every fp32 value within the finite range encodes,
    as torch's float8_e4m3fn (an independent implementation of the OCP format
    with round-to-nearest-even) does."""
    import torch

    o = make()
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([o.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(mine) == nan).all() and (mine[~nan] == ref[~nan]).all()
    rng = np.random.default_rng(8)
    grid = ref[~nan]
    mids = (np.sort(np.unique(grid))[1:] + np.sort(np.unique(grid))[:-1]) / 2  # exact ties
    ys = np.concatenate([rng.uniform(-448, 448, 3000), rng.uniform(-0.02, 0.02, 3000),
                         np.exp(rng.uniform(-12, 6, 2000)) * rng.choice([-1, 1], 2000), mids, grid])
    ys = ys.astype(np.float32)
    lib = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    enc = np.array([o.e4m3_encode(float(y)) for y in ys], dtype=np.uint8)
    # (+0 and -0 are both fine for a zero input)
    same = (enc == lib) | ((ys == 0) & ((enc & 0x7F) == 0) & ((lib & 0x7F) == 0))
    assert same.all(), ys[~same][:5]
    # Saturation beyond the largest finite value (448, code 0x7E).
    assert o.e4m3_encode(1000.0) == 0x7E and o.e4m3_encode(-1e30) == 0xFE and o.e4m3_encode(464.0) == 0x7E


def pin_quant_rows_closed_forms(make):
    """scale = max|x| / 448 (fp32); a row already on the scaled E4M3 grid comes
    back exactly; an all-zero row has scale 0 and codes 0; the round trip error
    is at most half a unit in the last place of the code."""
    o = make()
    rng = np.random.default_rng(9)
    grid = np.array([o.e4m3_value(c) for c in range(127)])  # non-negative finite values
    x = np.zeros((4, 128))
    for r in range(3):
        v = rng.choice(grid, 128) * rng.choice([-1, 1], 128)
        v[rng.integers(128)] = 448.0 * (1 if r % 2 else -1)
        x[r] = v * 2.0 ** (r - 3)  # exact in bf16 (at most 4 significant bits)
    xb = _bits(x.astype(np.float32))
    codes, scales = o.quant_rows(xb)
    assert scales[0] == np.float32(2.0 ** -3) and scales[1] == np.float32(2.0 ** -2) and scales[3] == 0.0
    back = o.dequant(codes, scales)
    assert np.array_equal(back[:3], x[:3]) and (codes[3] == 0).all()
    # Random rows: |x - E4M3(code) * scale| <= 2^-4 |x| (normal codes) or 2^-10 scale (subnormal).
    y = rng.standard_normal((64, 128)).astype(np.float32) * np.exp(rng.uniform(-8, 8, (64, 1))).astype(np.float32)
    yb = _bits(y)
    yv = np.array([[float(np.uint32(int(v) << 16).view(np.float32)) for v in row] for row in yb])
    c2, s2 = o.quant_rows(yb)
    err = np.abs(o.dequant(c2, s2) - yv)
    amax = np.abs(yv).max(axis=1)
    assert np.allclose(s2, (amax / 448.0).astype(np.float32), rtol=0, atol=0)
    bound = np.maximum(2.0 ** -4 * np.abs(yv), 2.0 ** -10 * s2[:, None].astype(np.float64)) * (1 + 2.0 ** -20)
    assert (err <= bound).all()


def pin_q8_attention_and_scores_on_exact_values(make):
    """On K, V and pooled-key rows that the format holds exactly, the fp8-cache
    attention and scores equal the bf16 ones (same values, same arithmetic)."""
    w = GQA
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    rng = np.random.default_rng(10)
    grid = np.array([o.e4m3_value(c) for c in range(127)])
    n, hk, d = 40, w.kv_heads, w.head_dim

    def exact_rows(shape):
        v = rng.choice(grid, shape) * rng.choice([-1, 1], shape)
        v[..., 0] = 448.0
        return (v * 2.0 ** rng.integers(-9, -5, shape[:-1] + (1,))).astype(np.float32)

    k = exact_rows((n, hk, d))
    v = exact_rows((n, hk, d))
    kb, vb = _bits(k), _bits(v)
    kc, ks = o.quant_rows(kb)
    vc, vs = o.quant_rows(vb)
    q = _bits(rng.standard_normal((w.q_heads, d)).astype(np.float32))
    toks = np.array([0, 3, 4, 5, 17, 30, 31, 39], dtype=np.int64)
    out, lse = o.attention(q, kb.reshape(n, -1), vb.reshape(n, -1), toks)
    out8, lse8 = o.attention_q8(q, kc, ks, vc, vs, toks)
    assert np.abs(out8 - out).max() < 1e-12 and np.abs(lse8 - lse).max() < 1e-12
    pk = exact_rows((12, d))
    pb = _bits(pk)
    pc, ps = o.quant_rows(pb)
    qr = _bits(rng.standard_normal((w.idx_heads, d)).astype(np.float32))
    assert np.array_equal(o.scores_q8(qr, pc, ps, 12), o.scores(qr, pb, 12))


# ----------------------------------------------------------------------------- training (f3)
# "QSA (Qwen Sparse Attention)" concept page, "Native trainability via 2-stage
# continued pretraining": stage 1 fits the indexer to a block-max-pooled dense
# teacher distribution by KL; stage 2 trains through the sparse attention.
def _f3_oracle(make, q_heads=4, kv_heads=2, head_dim=16):
    return make(r=4, K=16, q_heads=q_heads, kv_heads=kv_heads, head_dim=head_dim)


def pin_attention_f64_is_the_bf16_attention(make):
    """The fp64-operand attention used for the gradient checks is the pinned
    bf16 attention: the same outputs bit for bit on widened bf16 operands."""
    w = GQA
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    _, _, q, k, v = _inputs(w)
    i = 61
    toks = np.array([0, 1, 2, 3, 20, 21, 22, 23, 36, 37, 38, 39, 60, 61], dtype=np.int64)
    out, lse = o.attention(q[i], k.reshape(w.total, -1), v.reshape(w.total, -1), toks)
    wid = bfm.bf16_to_f64
    out2, lse2 = o.attention_f64(wid(q[i]), wid(k[toks]), wid(v[toks]))
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def pin_attention_backward_finite_differences(make):
    """Every entry of dq, dk, dv matches a central difference of the loss
    sum_h <dout_h, out_h> computed with the forward attention."""
    o = _f3_oracle(make)
    c = o.cfg
    rng = np.random.default_rng(31)
    ntok = 7
    q = rng.standard_normal((c.q_heads, c.head_dim))
    kt = rng.standard_normal((ntok, c.kv_heads, c.head_dim))
    vt = rng.standard_normal((ntok, c.kv_heads, c.head_dim))
    dout = rng.standard_normal((c.q_heads, c.head_dim))
    grads = o.attention_backward_f64(q, kt, vt, dout)
    base = [q, kt, vt]
    h = 1e-6

    def loss(args):
        out, _ = o.attention_f64(*args)
        return float((out * dout).sum())

    for which in range(3):
        for idx in np.ndindex(base[which].shape):
            plus = [a.copy() for a in base]
            minus = [a.copy() for a in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            g = grads[which][idx]
            assert abs(fd - g) <= 1e-6 * (1.0 + abs(g)), (which, idx, fd, g)


def pin_attention_backward_matches_autograd(make):
    """The gradient equals torch autograd's (float64) through a plain GQA
    softmax attention over the same tokens."""
    import torch

    o = _f3_oracle(make, q_heads=8, kv_heads=2, head_dim=32)
    c = o.cfg
    rng = np.random.default_rng(32)
    ntok, G = 11, c.q_heads // c.kv_heads
    q = rng.standard_normal((c.q_heads, c.head_dim))
    kt = rng.standard_normal((ntok, c.kv_heads, c.head_dim))
    vt = rng.standard_normal((ntok, c.kv_heads, c.head_dim))
    dout = rng.standard_normal((c.q_heads, c.head_dim))
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, kt, vt))
    kx, vx = tk.repeat_interleave(G, dim=1), tv.repeat_interleave(G, dim=1)
    p = torch.softmax(torch.einsum("hd,thd->ht", tq, kx) / np.sqrt(c.head_dim), dim=1)
    out = torch.einsum("ht,thd->hd", p, vx)
    out.backward(torch.tensor(dout))
    dq, dk, dv = o.attention_backward_f64(q, kt, vt, dout)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(mine - ref.numpy()).max() < 1e-12


def pin_attention_backward_bf16_gather(make):
    """The bf16-operand gradient is the fp64 one on the listed tokens' widened
    rows (one row per listed token, in list order)."""
    w = GQA
    o = make(r=w.r, K=w.K, q_heads=w.q_heads, kv_heads=w.kv_heads)
    _, _, q, k, v = _inputs(w)
    i = 50
    toks = np.array([4, 5, 6, 7, 28, 29, 30, 31, 48, 49, 50], dtype=np.int64)
    dout = _bits(np.random.default_rng(33).standard_normal((w.q_heads, w.head_dim)))
    got = o.attention_backward(q[i], k.reshape(w.total, -1), v.reshape(w.total, -1), toks, dout)
    wid = bfm.bf16_to_f64
    ref = o.attention_backward_f64(wid(q[i]), wid(k[toks]), wid(v[toks]), wid(dout))
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


def pin_distill_target_closed_forms(make):
    """Closed forms of the stage-1 target. (1) Identical keys: every head is
    uniform, so the target is uniform over the visible blocks. (2) Dominant
    tokens: heads of kv head 0 put 1/4 on each of tokens 5, 6, 13 and the tail
    token 20, heads of kv head 1 put everything on token 13; the head average
    is 1/8, 1/8, 5/8, 1/8, block 1's maximum is 1/8 and block 3's 5/8, so the
    target over blocks 0..4 is (0, 1/6, 0, 5/6, 0) (a mean pool, or a maximum
    over heads, gives other values). Keys after the query (here a dominant
    one and NaNs) are never read. (3) One key with logit L = 1 among zeros:
    the target over blocks 0, 1 of query 8 is (e/(e+1), 1/(e+1))."""
    o = _f3_oracle(make)
    c = o.cfg
    rng = np.random.default_rng(34)
    d, hk = c.head_dim, c.kv_heads
    nan = np.uint16(0x7FC0)
    # (1)
    i = 37
    kc = np.full((i + 9, hk, d), _bits(np.float32(0.5)), dtype=np.uint16)
    kc[i + 1:] = nan
    q = _bits(rng.standard_normal((c.q_heads, d)).astype(np.float32))
    t = o.distill_target(i, q, kc)
    assert t.size == i // c.r and np.abs(t - 1.0 / t.size).max() < 1e-15
    # (2)
    i = 20
    k = np.zeros((i + 9, hk, d), dtype=np.float32)
    for j in (5, 6, 13, 20):
        k[j, 0, 0] = 16.0
    k[13, 1, 0] = 16.0
    k[22, :, 0] = 64.0
    kc = _bits(k)
    kc[i + 3:] = nan
    qf = np.zeros((c.q_heads, d), dtype=np.float32)
    qf[:, 0] = 16.0
    t = o.distill_target(i, _bits(qf), kc)
    assert np.abs(t - np.array([0.0, 1 / 6, 0.0, 5 / 6, 0.0])).max() < 1e-12, t
    # (3)
    i = 8
    k = np.zeros((i + 1, hk, d), dtype=np.float32)
    k[1, :, 0] = 2.0
    qf = np.zeros((c.q_heads, d), dtype=np.float32)
    qf[:, 0] = 2.0  # logit 2 * 2 / sqrt(16) = 1
    t = o.distill_target(i, _bits(qf), _bits(k))
    e = np.e
    assert np.abs(t - np.array([e / (e + 1), 1 / (e + 1)])).max() < 1e-14, t
    # no visible block: nothing
    assert o.distill_target(3, _bits(qf), _bits(k)).size == 0


def pin_distill_target_other_block_sizes(make):
    """For r = 1 and r = 16 as for r = 4: identical keys give a uniform target
    over the floor(i/r) visible blocks; with r = 1 and one dominant token j
    below i, the target is the one-hot vector of block j."""
    rng = np.random.default_rng(36)
    for r in (1, 16):
        o = make(r=r, K=64, q_heads=4, kv_heads=2, head_dim=16)
        c = o.cfg
        i = 70
        kc = np.full((i + 1, c.kv_heads, c.head_dim), _bits(np.float32(0.25)), dtype=np.uint16)
        q = _bits(rng.standard_normal((c.q_heads, c.head_dim)).astype(np.float32))
        t = o.distill_target(i, q, kc)
        assert t.size == i // r and np.abs(t - 1.0 / t.size).max() < 1e-15, r
    o = make(r=1, K=64, q_heads=4, kv_heads=2, head_dim=16)
    c = o.cfg
    i, j = 40, 17
    k = np.zeros((i + 1, c.kv_heads, c.head_dim), dtype=np.float32)
    k[j, :, 0] = 32.0
    qf = np.zeros((c.q_heads, c.head_dim), dtype=np.float32)
    qf[:, 0] = 32.0  # logit 256 for token j, 0 elsewhere
    t = o.distill_target(i, _bits(qf), _bits(k))
    want = np.zeros(i)
    want[j] = 1.0
    assert np.abs(t - want).max() < 1e-12


def pin_attention_backward_properties(make):
    """The gradient is linear in dout (doubling dout doubles dq, dk, dv; a sum
    of two upstream gradients gives the sum of the gradients), and the rows of
    dS sum to zero, so sum_t dk_t = 0 for every kv head (the softmax is
    invariant to a shift of a head's logits)."""
    o = _f3_oracle(make, q_heads=8, kv_heads=2, head_dim=16)
    c = o.cfg
    rng = np.random.default_rng(37)
    ntok = 9
    q = rng.standard_normal((c.q_heads, c.head_dim))
    kt = rng.standard_normal((ntok, c.kv_heads, c.head_dim))
    vt = rng.standard_normal((ntok, c.kv_heads, c.head_dim))
    g1 = rng.standard_normal((c.q_heads, c.head_dim))
    g2 = rng.standard_normal((c.q_heads, c.head_dim))
    a = o.attention_backward_f64(q, kt, vt, g1)
    b = o.attention_backward_f64(q, kt, vt, g2)
    ab = o.attention_backward_f64(q, kt, vt, g1 + g2)
    a2 = o.attention_backward_f64(q, kt, vt, 2.0 * g1)
    for x, y, xy, x2 in zip(a, b, ab, a2):
        assert np.abs(xy - (x + y)).max() < 1e-12 and np.abs(x2 - 2.0 * x).max() < 1e-12
    assert np.abs(a[1].sum(axis=0)).max() < 1e-12


def pin_distill_kl_properties(make):
    """KL >= 0 on random targets and scores; its gradient sums to zero over the
    blocks (a normalised target); adding a constant to every score changes
    neither the KL nor its gradient."""
    o = _f3_oracle(make)
    rng = np.random.default_rng(38)
    for _ in range(20):
        n = int(rng.integers(1, 60))
        t = rng.random(n)
        t /= t.sum()
        s = (np.round(rng.standard_normal(n) * 4 * 256) / 256).astype(np.float32)  # + 8 stays exact
        kl, ds = o.distill_kl(t, s)
        assert kl >= -1e-12 and abs(ds.sum()) < 1e-12
        kl2, ds2 = o.distill_kl(t, s + np.float32(8.0))
        assert abs(kl2 - kl) < 1e-9 and np.abs(ds2 - ds).max() < 1e-9


def pin_distill_kl_library_and_gradient(make):
    """KL(t || softmax(s)) equals scipy's relative entropy (zero target entries
    included); it is 0 with a zero gradient at s = log t + const; its gradient
    matches central differences on exactly representable fp32 scores; no
    blocks gives 0."""
    from scipy.special import softmax
    from scipy.stats import entropy

    o = _f3_oracle(make)
    rng = np.random.default_rng(35)
    t = rng.random(50)
    t[[3, 17, 40]] = 0.0
    t /= t.sum()
    s = (np.round(rng.standard_normal(50) * 3 * 256) / 256).astype(np.float32)
    kl, ds = o.distill_kl(t, s)
    assert abs(kl - entropy(t, softmax(s.astype(np.float64)))) < 1e-12
    t2 = rng.random(20) + 0.1
    t2 /= t2.sum()
    kl0, ds0 = o.distill_kl(t2, (np.log(t2) + 3.0).astype(np.float32))
    assert abs(kl0) < 1e-12 and np.abs(ds0).max() < 1e-6
    h = 2.0 ** -12
    for b in range(0, 50, 7):
        sp, sm = s.copy(), s.copy()
        sp[b] += np.float32(h)
        sm[b] -= np.float32(h)
        fd = (o.distill_kl(t, sp)[0] - o.distill_kl(t, sm)[0]) / (2 * h)
        assert abs(fd - ds[b]) < 1e-6, (b, fd, ds[b])
    assert o.distill_kl(np.zeros(0), np.zeros(0, dtype=np.float32))[0] == 0.0


ALL_PINS = [v for kname, v in sorted(globals().items()) if kname.startswith("pin_")]
