"""Pins of the fp64 oracle against facts that the pages and mathematics fix.

Nothing here compares the oracle with itself: every expected value is a
page constant (tests/golden), a closed form worked out by hand, an
invariant, a library routine (torch's fp32->bf16 rounding, numpy matmul,
scipy softmax) or brute force on tiny inputs.  CPU only.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth

POOL = oracle.POOL
K = oracle.TOPK_BLOCKS


def bits_of(values):
    """bf16 bits of values that are exactly representable in bf16."""
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(values, dtype=np.float32)))
    return t.view(torch.int16).numpy().view(np.uint16).copy()


# ----------------------------------------------------------------------------
# Page constants
# ----------------------------------------------------------------------------
def test_page_constants(golden_constants):
    g = golden_constants
    assert oracle.POOL == g["pool_size"] == g["block_tokens"] == g["index_reduction"]
    assert oracle.TOPK_BLOCKS == g["topk_blocks"]
    assert g["topk_blocks"] * g["block_tokens"] == g["topk_tokens"] == g["dense_threshold"]
    assert synth.IDX_HEADS == g["indexer_heads"]
    assert g["qk_rope_head_dim"] == 0
    # the budget of a query: 512 blocks plus at most pool-1 unscored tail tokens
    pos = oracle.token_set(np.arange(K, dtype=np.int32), K * POOL + POOL - 1)
    assert pos.size == g["topk_tokens"] + POOL - 1


# ----------------------------------------------------------------------------
# bf16 rounding used by the pooled-key store
# ----------------------------------------------------------------------------
def test_bf16_rne_matches_library_on_fp32_values():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 7,
        (rng.integers(-(1 << 20), 1 << 20, 20000) / 64.0).astype(np.float32),
        np.float32([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-38, -5e-39]),
    ])
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_rne(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rne_closed_forms():
    # exactly half way between 1 and 1+2^-7: ties to the even significand (1.0)
    assert oracle.bf16_rne(1.0 + 2.0 ** -8) == 0x3F80
    # half way between 1+2^-7 and 1+2^-6: ties to even (1+2^-6)
    assert oracle.bf16_rne(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # a hair above half way must round up; double rounding through fp32 would
    # first land on the tie and then round down to 1.0
    assert oracle.bf16_rne(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    assert oracle.bf16_rne(-0.0) == 0x8000
    assert oracle.bf16_rne(-(1.0 + 2.0 ** -8 + 2.0 ** -30)) == 0xBF81
    # 5 + 1/64 lies half way between the bf16 neighbours 5 and 5 + 1/32
    assert oracle.bf16_rne(5.0 + 1 / 64) == 0x40A0
    assert oracle.bf16_rne(5.0 + 3 / 64) == 0x40A2


# ----------------------------------------------------------------------------
# IndexPool
# ----------------------------------------------------------------------------
def test_pool_identical_keys_return_the_key():
    rng = np.random.default_rng(1)
    key = rng.integers(-8, 9, 128).astype(np.float32)
    raw = bits_of(np.tile(key, (8, 1)))
    for w in ([0.5, 0.25, 0.125, 0.125], [0.25] * 4, [0.046875, 0.234375, 0.609375, 0.109375]):
        pooled = oracle.pool(raw, w)
        assert pooled.shape == (2, 128)
        assert np.array_equal(oracle.bf16_to_f64(pooled[0]), key.astype(np.float64))
        assert np.array_equal(pooled[0], pooled[1])


def test_pool_one_hot_weights_subsample():
    rng = np.random.default_rng(2)
    vals = rng.integers(-8, 9, (4 * 37 + 3, 128)).astype(np.float32)
    raw = bits_of(vals)
    for i in range(4):
        w = np.zeros(4)
        w[i] = 1.0
        pooled = oracle.pool(raw, w)
        assert pooled.shape == (37, 128)  # the 3 trailing tokens form no block
        assert np.array_equal(pooled, raw[i:4 * 37:4])


def test_pool_worked_example():
    # one dim; blocks [8, 4, 2, 0] and [6, 5, 0, 0]
    raw = bits_of(np.array([[8.0], [4.0], [2.0], [0.0], [6.0], [5.0], [0.0], [0.0]]))
    p = oracle.bf16_to_f64(oracle.pool(raw, [0.5, 0.25, 0.125, 0.125]))
    assert p.tolist() == [[4 + 1 + 0.25 + 0.0], [3 + 1.25]]
    # 6/64 + 5*63/64 = 5 + 1/64: exactly between two bf16 values -> 5.0 (even)
    p = oracle.bf16_to_f64(oracle.pool(raw, [1 / 64, 63 / 64, 0.0, 0.0]))
    assert p[1, 0] == 5.0
    # 8/64 + 4*63/64 = 4 + 1/16: a multiple of the bf16 spacing 1/32 on [4, 8)
    assert p[0, 0] == 4.0625


def test_pool_is_weighted_mean_bound():
    rng = np.random.default_rng(3)
    vals = rng.integers(-8, 9, (400, 128)).astype(np.float32)
    w = synth.workload("mid").pool_weights()
    p = oracle.bf16_to_f64(oracle.pool(bits_of(vals), w)).reshape(100, 128)
    blocks = vals.reshape(100, 4, 128).astype(np.float64)
    assert (p >= blocks.min(axis=1)).all() and (p <= blocks.max(axis=1)).all()
    exact = np.einsum("i,bid->bd", w, blocks)
    # one bf16 rounding: relative error <= 2^-8 (unit roundoff of 8 significant bits)
    assert (np.abs(p - exact) <= np.abs(exact) * 2.0 ** -8).all()


# ----------------------------------------------------------------------------
# IndexPool with a weight per token
# ----------------------------------------------------------------------------
def _bf16_rne_exact(x: Fraction) -> float:
    """Nearest-even bf16 value of an exact rational (8 significant bits, no
    double rounding): an independent rounding for the brute-force pins."""
    if x == 0:
        return 0.0
    sign = -1.0 if x < 0 else 1.0
    a = abs(x)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    # a in [1, 2): keep 7 fraction bits
    scaled = a * 128
    lo = scaled.numerator // scaled.denominator
    rem = scaled - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * float(Fraction(lo, 128) * Fraction(2) ** e)


def test_pool_tok_exact_rational_brute_force():
    """Each pooled value equals the exact rational weighted sum of the bf16
    keys with the fp32 per-token weights, rounded once to bf16."""
    rng = np.random.default_rng(41)
    n_tok, dim = 4 * 25 + 2, 6
    vals = (rng.standard_normal((n_tok, dim)) * np.exp2(rng.integers(-12, 12, (n_tok, 1))))
    raw = synth.f32_to_bf16_bits_np(vals.astype(np.float32))  # nearest bf16 values
    g = rng.standard_normal(n_tok)
    wt = np.empty(n_tok, np.float32)
    for b in range(n_tok // 4):
        e = np.exp(g[4 * b:4 * b + 4])
        wt[4 * b:4 * b + 4] = e / e.sum()
    wt[4 * 25:] = 0.5  # trailing tokens: no block
    got = oracle.bf16_to_f64(oracle.pool_tok(raw, wt.astype(np.float64)))
    kf = oracle.bf16_to_f64(raw)
    assert got.shape == (25, dim)
    for b in range(25):
        for d in range(dim):
            exact = sum(Fraction(float(wt[4 * b + i])) * Fraction(float(kf[4 * b + i, d]))
                        for i in range(4))
            assert got[b, d] == _bf16_rne_exact(exact), (b, d)
    # a block whose sum, 1 + 2^-8 + 2^-30, sits just above a bf16 tie by less
    # than an fp32 step: one rounding gives 1 + 2^-7, a sum rounded to fp32
    # first would land on the tie and give 1.0
    keys = bits_of(np.array([[4.0], [2.0 ** -6], [2.0 ** -28], [0.0]], np.float32))
    got = oracle.bf16_to_f64(oracle.pool_tok(keys, np.full(4, 0.25)))
    assert got[0, 0] == 1.0 + 2.0 ** -7


def test_pool_tok_per_block_one_hot_picks_one_token():
    rng = np.random.default_rng(42)
    n_blk = 40
    raw = synth.f32_to_bf16_bits_np(rng.standard_normal((4 * n_blk, 128)).astype(np.float32))
    pick = rng.integers(0, 4, n_blk)
    wt = np.zeros(4 * n_blk)
    wt[4 * np.arange(n_blk) + pick] = 1.0
    got = oracle.pool_tok(raw, wt)
    assert np.array_equal(got, raw[4 * np.arange(n_blk) + pick])


def test_pool_tok_identical_keys_and_static_weights():
    rng = np.random.default_rng(43)
    key = rng.integers(-8, 9, 128).astype(np.float32)
    # identical keys in a block, dyadic weights summing to exactly 1 per block
    wt = np.tile([0.5, 0.25, 0.125, 0.125], 3)
    wt[4:8] = [1 / 64, 3 / 64, 12 / 64, 48 / 64]
    got = oracle.pool_tok(bits_of(np.tile(key, (12, 1))), wt)
    assert all(np.array_equal(oracle.bf16_to_f64(got[b]), key.astype(np.float64)) for b in range(3))
    # the same weights on every block give the static-weight pooling
    vals = rng.integers(-8, 9, (4 * 30, 128)).astype(np.float32)
    w = synth.workload("mid").pool_weights()
    assert np.array_equal(oracle.pool_tok(bits_of(vals), np.tile(w, 30)), oracle.pool(bits_of(vals), w))


# ----------------------------------------------------------------------------
# Indexer scores
# ----------------------------------------------------------------------------
def bf16_round(x):
    """Nearest-even bf16 value of fp32 data (library rounding), as fp32."""
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def _rand_case(rng, nblk, heads=32, dim=128):
    q = rng.integers(-4, 5, (heads, dim)).astype(np.float32)
    k = bf16_round(rng.integers(-512, 513, (nblk, dim)) / 64.0)
    w = np.array([0.25, 0.5, 1.0])[rng.integers(0, 3, heads)]
    return q, k, w


def test_score_one_hot_heads_pick_elements():
    rng = np.random.default_rng(4)
    heads, dim, nblk = 32, 128, 50
    k = bf16_round(rng.integers(-512, 513, (nblk, dim)) / 64.0)
    q = np.zeros((heads, dim), np.float32)
    dsel = rng.permutation(dim)[:heads]
    q[np.arange(heads), dsel] = 1.0
    for h in (0, 7, 31):
        w = np.zeros(heads)
        w[h] = 1.0
        s = oracle.score(bits_of(q), w, bits_of(k))
        assert np.array_equal(s, np.maximum(k[:, dsel[h]], 0.0).astype(np.float64))
        # a negative head weight keeps the sign: ReLU acts on the dot only
        w[h] = -0.5
        s = oracle.score(bits_of(q), w, bits_of(k))
        assert np.array_equal(s, -0.5 * np.maximum(k[:, dsel[h]], 0.0).astype(np.float64))


def test_score_matches_matmul_and_integer_closed_form():
    rng = np.random.default_rng(5)
    q, k, w = _rand_case(rng, 300)
    s = oracle.score(bits_of(q), w, bits_of(k))
    # library matmul (non-square operands: a transposed operand cannot pass)
    ref = np.maximum(k.astype(np.float64) @ q.T.astype(np.float64), 0.0) @ w
    assert np.array_equal(s, ref)
    # exact integers: 256*s = sum_h (4 w_h) relu(sum_d q (64 k))
    qi = q.astype(np.int64)
    ki = np.round(k.astype(np.float64) * 64).astype(np.int64)
    wi = np.round(w * 4).astype(np.int64)
    exact = (np.maximum(ki @ qi.T, 0) * wi).sum(axis=1)
    assert np.array_equal(np.round(s * 256).astype(np.int64), exact)
    assert np.array_equal(s * 256, exact.astype(np.float64))


def test_score_relu_and_threads():
    rng = np.random.default_rng(6)
    q, k, w = _rand_case(rng, 5000)
    s1 = oracle.score(bits_of(q), w, bits_of(k), nthreads=1)
    s4 = oracle.score(bits_of(q), w, bits_of(k), nthreads=4)
    assert np.array_equal(s1, s4)
    assert (s1 >= 0).all()
    # negating q turns ReLU(x) into ReLU(-x): s(q) + s(-q) = sum_h w_h |q_h . k|
    sn = oracle.score(bits_of(-q), w, bits_of(k))
    ref = np.abs(k.astype(np.float64) @ q.T.astype(np.float64)) @ w
    assert np.array_equal(s1 + sn, ref)


# ----------------------------------------------------------------------------
# Top-k
# ----------------------------------------------------------------------------
def _is_valid_topk(s, sel, K_):
    s32 = np.asarray(s, np.float64).astype(np.float32)
    n = len(s)
    sel = list(sel)
    if len(sel) != min(K_, n) or sel != sorted(set(sel)):
        return False
    inside = set(sel)
    for i in sel:
        for j in range(n):
            if j in inside:
                continue
            if not (s32[i] > s32[j] or (s32[i] == s32[j] and i < j)):
                return False
    return True


def test_topk_brute_force_tiny_with_ties():
    rng = np.random.default_rng(7)
    for trial in range(300):
        n = int(rng.integers(1, 24))
        s = rng.integers(-2, 3, n).astype(np.float64)
        s[rng.random(n) < 0.2] = -0.0
        for K_ in (1, 2, 3, 5, n, n + 3):
            sel = oracle.topk(s, K_)
            assert _is_valid_topk(s, sel, K_), (s, K_, sel)


def test_topk_exhaustive_small():
    # every selection of size k from n=7 is checked against the definition
    s = np.array([3.0, 1.0, 3.0, 0.0, -0.0, 1.0, 2.0])
    for K_ in range(1, 8):
        sel = tuple(oracle.topk(s, K_))
        valid = [c for c in itertools.combinations(range(7), K_) if _is_valid_topk(s, c, K_)]
        assert valid == [sel]


def test_topk_special_cases():
    assert oracle.topk(np.zeros(1000), 512).tolist() == list(range(512))
    assert oracle.topk(np.arange(100.0), 512).tolist() == list(range(100))
    assert oracle.topk(np.arange(1000.0), 512).tolist() == list(range(488, 1000))
    # decision in fp32: 1 + 2^-40 rounds to 1.0 and ties with block 0
    assert oracle.topk(np.array([1.0, 1.0 + 2.0 ** -40]), 1).tolist() == [0]
    assert oracle.topk(np.array([-0.0, 0.0, -0.0]), 2).tolist() == [0, 1]
    assert oracle.topk(np.zeros(0), 512).tolist() == []


def test_token_set():
    assert oracle.token_set([1], 10).tolist() == [4, 5, 6, 7, 8, 9]
    assert oracle.token_set([0, 2], 12).tolist() == [0, 1, 2, 3, 8, 9, 10, 11]
    assert oracle.token_set([0, 1], 11).tolist() == [0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10]
    assert oracle.token_set([], 3).tolist() == [0, 1, 2]
    assert oracle.token_set([], 0).tolist() == []


# ----------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------
def _normal_bits(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def test_attention_single_token_returns_row():
    rng = np.random.default_rng(8)
    q = _normal_bits(rng, (16, 512), 0.05)
    row = _normal_bits(rng, (1, 512))
    out, lse = oracle.attention(q, row, 1.0)
    c = oracle.bf16_to_f64(row[0])
    assert np.array_equal(out, np.tile(c, (16, 1)))
    assert np.allclose(lse, oracle.bf16_to_f64(q) @ c, rtol=0, atol=1e-12)


def test_attention_equal_logits_give_mean():
    rng = np.random.default_rng(9)
    rows = _normal_bits(rng, (37, 512))
    q = np.zeros((4, 512), np.uint16)
    out, lse = oracle.attention(q, rows, 1.0)
    assert np.allclose(out, oracle.bf16_to_f64(rows).mean(axis=0)[None, :], atol=1e-14)
    assert np.allclose(lse, np.log(37.0), atol=1e-14)


def test_attention_matches_scipy_softmax_and_is_order_free():
    rng = np.random.default_rng(10)
    q = _normal_bits(rng, (8, 512), 1 / np.sqrt(512))
    rows = _normal_bits(rng, (300, 512))
    qd, cd = oracle.bf16_to_f64(q), oracle.bf16_to_f64(rows)
    z = 0.7 * (qd @ cd.T)
    ref = scipy.special.softmax(z, axis=1) @ cd
    out, lse = oracle.attention(q, rows, 0.7)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
    assert np.allclose(lse, scipy.special.logsumexp(z, axis=1), rtol=0, atol=1e-12)
    perm = rng.permutation(300)
    out2, _ = oracle.attention(q, rows[perm], 0.7)
    assert np.allclose(out, out2, rtol=0, atol=1e-13)


def test_attention_logit_shift_invariance():
    # a constant last latent component shifts every logit of a head by the
    # same amount (sm_scale * q_last * a): the softmax weights do not change
    rng = np.random.default_rng(11)
    rows = _normal_bits(rng, (64, 512))
    rows[:, -1] = bits_of([2.0])[0]
    q = _normal_bits(rng, (4, 512), 0.05)
    q2 = q.copy()
    q2[:, -1] = bits_of([1.5])[0]
    o1, l1 = oracle.attention(q, rows, 1.0)
    o2, l2 = oracle.attention(q2, rows, 1.0)
    assert np.allclose(o1, o2, atol=1e-13)
    shift = 2.0 * (1.5 - oracle.bf16_to_f64(q[:, -1]))
    assert np.allclose(l2 - l1, shift, atol=1e-12)


def test_attention_two_tokens_closed_form():
    q = np.zeros((1, 512), np.float32)
    q[0, 0] = 1.0
    rows = np.zeros((2, 512), np.float32)
    rows[0, 0], rows[1, 0] = 1.0, -1.0
    rows[0, 1], rows[1, 1] = 3.0, 5.0
    out, lse = oracle.attention(bits_of(q), bits_of(rows), 2.0)
    e1, e2 = np.exp(2.0), np.exp(-2.0)
    assert np.isclose(out[0, 0], (e1 - e2) / (e1 + e2), atol=1e-15)
    assert np.isclose(out[0, 1], (3 * e1 + 5 * e2) / (e1 + e2), atol=1e-15)
    assert np.isclose(lse[0], np.log(e1 + e2), atol=1e-15)


def test_attention_empty_set():
    out, lse = oracle.attention(np.zeros((2, 512), np.uint16), np.zeros((0, 512), np.uint16), 1.0)
    assert (out == 0).all() and np.isneginf(lse).all()


# ----------------------------------------------------------------------------
# Whole decode query: sparse equals dense below the budget
# ----------------------------------------------------------------------------
def _decode_case(seed, n_vis, H=8):
    w = synth.workload("tiny")
    raw = w.raw_keys_np(0, 0, n_vis)
    pooled = oracle.pool(raw, w.pool_weights())
    rng = np.random.default_rng(seed)
    q_idx = rng.integers(-4, 5, (32, 128)).astype(np.float32)
    w_head = np.array([0.25, 0.5, 1.0])[rng.integers(0, 3, 32)]
    q = _normal_bits(rng, (H, 512), 1 / np.sqrt(512))
    latent = _normal_bits(rng, (n_vis, 512))
    return pooled, bits_of(q_idx), w_head, q, latent


@pytest.mark.parametrize("n_vis", [1, 3, 4, 5, 1536, 2047, 2048, 2049, 2051])
def test_sparse_equals_dense_within_budget(n_vis):
    pooled, q_idx, w_head, q, latent = _decode_case(12, n_vis)
    r = oracle.decode_query(q_idx, w_head, pooled, n_vis, q, lambda pos: latent[pos], 1.0)
    assert r["positions"].tolist() == list(range(n_vis))
    cd = oracle.bf16_to_f64(latent)
    z = oracle.bf16_to_f64(q) @ cd.T
    ref = scipy.special.softmax(z, axis=1) @ cd
    assert np.allclose(r["out"], ref, rtol=0, atol=1e-12)


def test_sparse_drops_lowest_block_above_budget():
    n_vis = 2052 + 2  # 513 complete blocks + 2 tail tokens
    pooled, q_idx, w_head, q, latent = _decode_case(13, n_vis)
    r = oracle.decode_query(q_idx, w_head, pooled, n_vis, q, lambda pos: latent[pos], 1.0)
    s32 = r["scores"].astype(np.float32)
    order = sorted(range(513), key=lambda b: (-s32[b], b))
    dropped = order[-1]
    assert sorted(set(range(513)) - set(r["idx"].tolist())) == [dropped]
    assert r["positions"].size == 512 * 4 + 2
    assert r["positions"][-2:].tolist() == [2052, 2053]
    keep = [p for p in range(n_vis) if p // 4 != dropped]
    cd = oracle.bf16_to_f64(latent[keep])
    ref = scipy.special.softmax(oracle.bf16_to_f64(q) @ cd.T, axis=1) @ cd
    assert np.allclose(r["out"], ref, atol=1e-12)


def test_all_zero_scores_pick_first_blocks():
    pooled, q_idx, w_head, q, latent = _decode_case(14, 8192)
    zero_q = np.zeros_like(q_idx)
    r = oracle.decode_query(zero_q, w_head, pooled, 8192, q, lambda pos: latent[pos], 1.0)
    assert r["idx"].tolist() == list(range(512))


def test_generator_scores_are_exact_in_fp32():
    """The workloads' integer/dyadic data keep every fp32 partial sum exact."""
    for name in ("tiny", "mid"):
        w = synth.workload(name)
        raw = w.raw_keys_np(0, 0, 4096)
        pooled = oracle.pool(raw, w.pool_weights())
        k = oracle.bf16_to_f64(pooled)
        assert np.array_equal(k * 64, np.round(k * 64))
        q = oracle.bf16_to_f64(w.q_idx_np([0])[0])
        wh = w.w_head_np([0])[0].astype(np.float64)
        dots = k @ q.T
        assert np.abs(dots).max() * 64 < 2 ** 24
        s = oracle.score(w.q_idx_np([0])[0], wh, pooled)
        # every partial sum over heads is a multiple of 2^-8 below 2^16
        partial = np.cumsum(np.maximum(dots, 0) * wh, axis=1)
        assert partial.max() < 2 ** 16
        assert np.array_equal(s * 256, np.round(s * 256))


# ----------------------------------------------------------------------------
# INT8 pooled-key cache
# ----------------------------------------------------------------------------
def test_quant_i8_closed_forms():
    # values already on the grid with max |x| in [64, 127]: scale 1, codes = x
    x = np.array([127, -64, 3, 0, -1, 100], np.float64)
    c, e = oracle.quant_i8(x)
    assert e == 0 and c.tolist() == x.astype(int).tolist()
    # half-way cases go to the even code
    c, e = oracle.quant_i8([127, 0.5, 1.5, 2.5, -2.5, -3.5])
    assert e == 0 and c.tolist() == [127, 0, 2, 2, -2, -4]
    # 127 * 2^e itself keeps that e; just above it needs e + 1
    assert oracle.quant_i8([127 * 2.0 ** -5])[1] == -5
    c, e = oracle.quant_i8([127.5, 1.0, 3.0])
    assert e == 1 and c.tolist() == [64, 0, 2]
    # the workload's query range: |q| <= 4 -> 2^-4, codes 16 q
    c, e = oracle.quant_i8([4, -3, 1, 0.5])
    assert e == -4 and c.tolist() == [64, -48, 16, 8]
    # an all-zero vector: e = 0, zero codes
    c, e = oracle.quant_i8(np.zeros(128))
    assert e == 0 and not c.any()


def test_quant_i8_invariants_random():
    rng = np.random.default_rng(21)
    for t in range(300):
        mag = 2.0 ** rng.integers(-60, 60)
        x = (rng.standard_normal(128) * mag).astype(np.float32).astype(np.float64)
        if t % 7 == 0:
            x[rng.integers(0, 128, 40)] = 0.0
        c, e = oracle.quant_i8(x)
        ci = c.astype(np.int64)
        amax = np.abs(x).max()
        # e is the smallest exponent that keeps every code within 127
        assert amax <= 127 * 2.0 ** e and amax > 127 * 2.0 ** (e - 1)
        assert 64 <= np.abs(ci).max() <= 127
        # one rounding of an exact scaling: error at most half a step
        assert (np.abs(x - ci * 2.0 ** e) <= 2.0 ** (e - 1)).all()
        # a power-of-two change of the input only moves the exponent
        c2, e2 = oracle.quant_i8(x * 2.0 ** 9)
        assert e2 == e + 9 and np.array_equal(c2, c)


def _grid_ints(rng, shape):
    """Integers in [-127, 127] with every row's max |x| in [64, 127]."""
    v = rng.integers(-127, 128, shape)
    v[..., 0] = rng.choice([-1, 1], shape[:-1]) * rng.integers(64, 128, shape[:-1])
    return v


def test_pool_i8_on_grid_and_one_hot():
    rng = np.random.default_rng(22)
    key = _grid_ints(rng, (20, 128)).astype(np.float32)
    raw = bits_of(np.repeat(key, POOL, axis=0))
    # identical keys pool to the key itself, already on the grid: scale 1
    codes, scale = oracle.pool_i8(raw, np.array([0.125, 0.5, 0.25, 0.125]))
    assert np.array_equal(codes.astype(np.float32), key) and (scale == 1.0).all()
    # one-hot weights subsample, then quantise: keys scaled by 2^-3 keep
    # their codes and get scale 2^-3
    raw2 = _grid_ints(rng, (80, 128)).astype(np.float32) / 8
    for i in range(POOL):
        w = np.zeros(POOL)
        w[i] = 1.0
        codes, scale = oracle.pool_i8(bits_of(raw2), w)
        assert np.array_equal(codes.astype(np.float32), raw2[i::POOL] * 8)
        assert (scale == 0.125).all()


def test_pool_i8_dequantises_within_half_step_of_exact_pool():
    """The codes quantise the exact pooled sum: within half a step of it.
    With the workloads' 1/64-dyadic weights the sums need up to 11
    significant bits, so a bf16 rounding before the quantisation would move
    some codes by one step and break the bound."""
    rng = np.random.default_rng(23)
    cases = [(bits_of(rng.integers(-8, 9, (400, 128)).astype(np.float32)),
              np.array([0.5, 0.25, 0.125, 0.125]))]
    mid = synth.workload("mid")
    cases.append((mid.raw_keys_np(0, 0, 16384), mid.pool_weights()))
    for raw, w in cases:
        codes, scale = oracle.pool_i8(raw, w)
        r = oracle.bf16_to_f64(raw).reshape(-1, POOL, 128)
        exact = np.einsum("bid,i->bd", r, w)
        deq = codes.astype(np.float64) * scale[:, None]
        assert (np.abs(deq - exact) <= scale[:, None] / 2).all()
        assert (np.abs(codes).max(axis=1) >= 64).all()
    # the second case really needs more than bf16's 8 significant bits
    assert not np.array_equal(exact, oracle.bf16_to_f64(oracle.pool(raw, w)))


def test_score_i8_integer_closed_form():
    rng = np.random.default_rng(24)
    heads, nblk = 32, 300
    q = _grid_ints(rng, (heads, 128))
    k = _grid_ints(rng, (nblk, 128))
    w = np.array([0.25, 0.5, 1.0])[rng.integers(0, 3, heads)]
    w[3] = -0.5  # a negative head weight keeps its sign
    s = oracle.score_i8(bits_of(q.astype(np.float32)), w, k.astype(np.int8), np.ones(nblk))
    # 4 s = sum_h (4 w_h) relu(k_b . q_h), in exact integers
    exact = (np.maximum(k @ q.T, 0) * np.round(w * 4).astype(np.int64)).sum(axis=1)
    assert np.array_equal(s * 4, exact.astype(np.float64))
    # block scales multiply the block's score; a head quantised with scale
    # 2^-3 (query / 8) contributes its dot times 2^-3
    sc = 2.0 ** rng.integers(-6, 7, nblk)
    s2 = oracle.score_i8(bits_of(q.astype(np.float32) / 8), w, k.astype(np.int8), sc)
    assert np.array_equal(s2, s * sc / 8)


def test_score_i8_is_bf16_score_of_dequantised_operands():
    """Dequantised codes (<= 7 bits times a power of two) are exact in bf16,
    so the INT8 score equals the bf16 score of the dequantised query and
    keys, an independently pinned routine."""
    w_ = synth.workload("mid")
    raw = w_.raw_keys_np(0, 0, 8192)
    codes, scale = oracle.pool_i8(raw, w_.pool_weights())
    qb = w_.q_idx_np([1])[0]
    wh = w_.w_head_np([1])[0].astype(np.float64)
    q = oracle.bf16_to_f64(qb)
    deq_q = np.stack([c * 2.0 ** e for c, e in (oracle.quant_i8(q[h]) for h in range(32))])
    deq_k = codes.astype(np.float64) * scale[:, None]
    s = oracle.score_i8(qb, wh, codes, scale)
    ref = oracle.score(bits_of(deq_q), wh, bits_of(deq_k))
    assert np.array_equal(s, ref)
    # and the quantised scores rank close to the bf16 ones: the top 512 sets overlap
    s_bf = oracle.score(qb, wh, oracle.pool(raw, w_.pool_weights()))
    common = np.intersect1d(oracle.topk(s), oracle.topk(s_bf)).size
    assert common >= 400


def test_generator_i8_scores_are_exact_in_fp32():
    """On the workloads, sum_h (w_h 2^e_h) relu(dot) is a sum of multiples of
    its smallest head factor whose total stays below 2^24 of them, and every
    dot is below 2^24: the device's fp32 head sum is exact in any order."""
    for name in ("tiny", "mid", "1m", "prefill"):
        w_ = synth.workload(name)
        raw = w_.raw_keys_np(0, 0, 32768)
        codes, scale = oracle.pool_i8(raw, w_.pool_weights())
        # decode rows are sequences; prefill rows are the chunk's query positions
        rows = (w_.L, w_.L + w_.T - 1) if name == "prefill" else (0, w_.B - 1)
        for row in rows:
            q = oracle.bf16_to_f64(w_.q_idx_np([row])[0])
            wh = w_.w_head_np([row])[0].astype(np.float64)
            qc, qe = zip(*(oracle.quant_i8(q[h]) for h in range(32)))
            f = wh * 2.0 ** np.array(qe)
            dots = codes.astype(np.int64) @ np.stack(qc).astype(np.int64).T
            assert np.abs(dots).max() < 2 ** 24
            units = np.abs(f) / np.abs(f).min()
            assert np.array_equal(units, np.round(units))
            assert (np.maximum(dots, 0) * units).sum(axis=1).max() < 2 ** 24


# ----------------------------------------------------------------------------
# FP8 (E4M3) latent cache
# ----------------------------------------------------------------------------
def test_e4m3_rounding_matches_library():
    rng = np.random.default_rng(41)
    x = np.concatenate([
        rng.uniform(-448, 448, 20000),
        rng.standard_normal(20000) * 2.0 ** rng.integers(-12, 8, 20000),
        # exact half-way points between neighbouring E4M3 values
        (np.arange(1, 480) + 0.5) * 2.0 ** -9,
        ((np.arange(8, 16) + 0.5)[None, :] * 2.0 ** np.arange(-6, 6)[:, None]).ravel(),
    ]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_bits(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)
    # and the decoder inverts the library's encoding on every finite pattern
    finite = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], dtype=np.uint8)
    lib = torch.tensor(finite).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(oracle.e4m3_value(finite), lib)


def test_e4m3_closed_forms():
    # 16..32 has spacing 2: 17 and 19 are ties, going to the even mantissa
    assert [oracle.e4m3_value(oracle.e4m3_bits(v)) for v in (17, 19, 448, 0.3)] == \
        [16.0, 20.0, 448.0, 0.3125]
    # subnormal step 2^-9: 2^-10 ties to 0, 3 * 2^-10 ties up to 2^-8
    assert oracle.e4m3_bits(2.0 ** -10) == 0 and oracle.e4m3_bits(3 * 2.0 ** -10) == 2
    assert oracle.e4m3_bits(2.0 ** -9) == 1 and oracle.e4m3_bits(2.0 ** -6) == 8
    assert oracle.e4m3_bits(-5.5) == 0x80 | (9 << 3) | 3


def test_quant_e4m3_invariants():
    rng = np.random.default_rng(42)
    for t in range(200):
        x = (rng.standard_normal(512) * 2.0 ** rng.integers(-40, 40)).astype(np.float32)
        x = x.astype(np.float64)
        if t % 5 == 0:
            x[rng.integers(0, 512, 100)] = 0.0
        c, e = oracle.quant_e4m3(x)
        v = oracle.e4m3_value(c)
        amax = np.abs(x).max()
        # the smallest exponent that keeps every value within 448
        assert amax <= 448 * 2.0 ** e and amax > 448 * 2.0 ** (e - 1)
        assert 224 <= np.abs(v).max() <= 448
        # one nearest rounding: within half the local spacing (4 significant
        # bits, subnormal step 2^-9 in code units)
        y = np.abs(x) * 2.0 ** -e
        spacing = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -9))) - 3), 2.0 ** -9)
        assert (np.abs(x * 2.0 ** -e - v) <= spacing / 2).all()
        c2, e2 = oracle.quant_e4m3(x * 2.0 ** 7)
        assert e2 == e + 7 and np.array_equal(c2, c)
    c, e = oracle.quant_e4m3(np.zeros(512))
    assert e == 0 and not c.any()


def test_fp8_latent_attention():
    rng = np.random.default_rng(43)
    H, S, D = 8, 40, 512
    q = _normal_bits(rng, (H, D), 1 / np.sqrt(D))
    rows = _normal_bits(rng, (S, D))
    codes, e = oracle.latent_fp8(rows)
    deq = oracle.dequant_fp8_bits(codes, e)
    # attention over the FP8 cache is attention over the dequantised rows
    out8, lse8 = oracle.attention_fp8(q, rows, 1.0)
    out, lse = oracle.attention(q, deq, 1.0)
    assert np.array_equal(out8, out) and np.array_equal(lse8, lse)
    # rows already on the grid (4 significant bits, max in (224, 448]) are stored exactly
    grid = oracle.e4m3_value(rng.integers(0, 126, (S, D)).astype(np.uint8))
    grid[:, 0] = 448.0
    gbits = bits_of(grid * 2.0 ** -6)
    c2, e2 = oracle.latent_fp8(gbits)
    assert (e2 == -6).all()
    assert np.array_equal(oracle.dequant_fp8_bits(c2, e2), gbits)
    out_g, _ = oracle.attention_fp8(q, gbits, 1.0)
    assert np.array_equal(out_g, oracle.attention(q, gbits, 1.0)[0])
    # the error of a 512-wide N(0,1) row: below 2^-4 of its scale per element
    x = oracle.bf16_to_f64(rows)
    assert (np.abs(oracle.bf16_to_f64(deq) - x) <= 2.0 ** (e[:, None] + 8 - 4)).all()
