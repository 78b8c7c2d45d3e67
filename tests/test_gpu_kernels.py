"""Per-kernel parity of the CUDA path against the fp64 oracle, through the
C ABI, on seeded inputs that span several tiles and ragged tails, plus the
edge cases of each step (empty rows, fewer blocks than the budget, ties,
-0, skipped block ids)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import (LSE_ATOL, assert_attention_close, bits_of, f64_of, need_gpu,
                          oracle_attention_rows, to_dev_bf16)

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------------------
# IndexPool append
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("lens,n_new", [([0, 5, 10, 3], 7), ([3, 0, 1, 2], 1), ([2, 9, 0, 4], 1003),
                                        ([0, 0, 0, 0], 4)])
def test_pool_append_ragged(lens, n_new):
    spx = need_gpu()
    w = synth.workload("mid")
    pw = w.pool_weights()
    d = spx.dims(64)
    B = len(lens)
    total = max(lens) + n_new
    cap_blk = (total + 3) // 4 + 2
    raw = [w.raw_keys_np(b, 0, total) for b in range(B)]
    tail0 = np.zeros((B, 3, 128), np.uint16)
    for b, L0 in enumerate(lens):
        for p in range((L0 // 4) * 4, L0):
            tail0[b, p % 4] = raw[b][p]
    new = np.stack([raw[b][lens[b]:lens[b] + n_new] for b in range(B)])
    pooled = torch.zeros(B, cap_blk, 128, dtype=torch.bfloat16, device="cuda")
    tail = to_dev_bf16(tail0)
    len_dev = torch.tensor(lens, dtype=torch.int64, device="cuda")
    spx.spx_pool_append(d, B, to_dev_bf16(new), n_new, pw.astype(np.float32), tail, pooled,
                        cap_blk, len_dev, total)
    torch.cuda.synchronize()
    got = bits_of(pooled)
    got_tail = bits_of(tail)
    for b, L0 in enumerate(lens):
        end = L0 + n_new
        ref = oracle.pool(raw[b][:end], pw)
        lo, hi = L0 // 4, end // 4
        assert np.array_equal(got[b, lo:hi], ref[lo:hi]), f"seq {b}"
        assert (got[b, :lo] == 0).all() and (got[b, hi:] == 0).all()
        for p in range((end // 4) * 4, end):
            assert np.array_equal(got_tail[b, p % 4], raw[b][p])


def _learned_pool_case(seed):
    """Pool weights as a learned layer would hold them: the softmax of N(0,1)
    logits in fp32 (not dyadic), and bf16 keys over a wide range of
    magnitudes with exact zeros and -0 mixed in."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(4).astype(np.float32)
    pw = np.exp(z - z.max()).astype(np.float32)
    pw = (pw / pw.sum()).astype(np.float32)
    assert abs(float(pw.astype(np.float64).sum()) - 1.0) <= 1e-6
    assert any(float(x) * 64 != int(float(x) * 64) for x in pw)  # not 1/64-dyadic
    return rng, pw


def _fp32_route_bits(raw_bits, pw):
    """bf16 bits of the pooled key summed in fp32 (one rounding per step)
    and then rounded to bf16: the double rounding the single-rounding
    reading avoids.  Used only to show that the test data tells the two
    apart."""
    k = synth.bf16_bits_to_f64_np(raw_bits).astype(np.float32).reshape(-1, 4, raw_bits.shape[-1])
    acc = np.zeros(k[:, 0].shape, np.float32)
    for i in range(4):
        acc = (acc + (k[:, i] * np.float32(pw[i])).astype(np.float32)).astype(np.float32)
    return synth.f32_to_bf16_bits_np(acc)


@pytest.mark.parametrize("lens,n_new", [([0, 6, 13], 4001), ([1, 2, 3], 2)])
def test_pool_append_learned_weights_single_rounding(lens, n_new):
    """[W1] "IndexPool": the pooling weights are learned.  With fp32 weights
    that are not dyadic, the pooled key must still be the single
    round-to-nearest-even of the exact weighted sum (the oracle's reading),
    bit for bit; the data are chosen so that an fp32 sum would differ."""
    spx = need_gpu()
    rng, pw = _learned_pool_case(17 + n_new)
    B = len(lens)
    total = max(lens) + n_new
    cap_blk = (total + 3) // 4 + 1
    raws = []
    for b in range(B):
        v = rng.standard_normal((total, 128)) * np.exp2(rng.integers(-30, 30, (total, 1)))
        v[rng.random((total, 128)) < 0.02] = 0.0
        v[rng.random((total, 128)) < 0.01] = -0.0
        raws.append(synth.f32_to_bf16_bits_np(v.astype(np.float32)))
    tail0 = np.zeros((B, 3, 128), np.uint16)
    for b, L0 in enumerate(lens):
        for p in range((L0 // 4) * 4, L0):
            tail0[b, p % 4] = raws[b][p]
    new = np.stack([raws[b][lens[b]:lens[b] + n_new] for b in range(B)])
    pooled = torch.zeros(B, cap_blk, 128, dtype=torch.bfloat16, device="cuda")
    tail = to_dev_bf16(tail0)
    len_dev = torch.tensor(lens, dtype=torch.int64, device="cuda")
    d = spx.dims(64)
    spx.spx_pool_append(d, B, to_dev_bf16(new), n_new, pw, tail, pooled, cap_blk, len_dev, total)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    got = bits_of(pooled)
    differs = 0
    for b, L0 in enumerate(lens):
        end = L0 + n_new
        ref = oracle.pool(raws[b][:end], pw.astype(np.float64))
        lo, hi = L0 // 4, end // 4
        assert np.array_equal(got[b, lo:hi], ref[lo:hi]), f"seq {b}"
        differs += int((_fp32_route_bits(raws[b][4 * lo:4 * hi], pw) != ref[lo:hi]).sum())
    if n_new > 100:
        assert differs > 0, "the data do not separate single from double rounding"


@pytest.mark.parametrize("lens,n_new", [([0, 6, 13], 4001)])
def test_pool_append_i8_learned_weights(lens, n_new):
    """The INT8 cache under learned fp32 weights: codes and block scales of
    the exact weighted sum (one round-half-even after an exact power-of-two
    scaling), bit for bit as in the oracle."""
    spx = need_gpu()
    rng, pw = _learned_pool_case(5)
    B = len(lens)
    total = max(lens) + n_new
    cap_blk = (total + 3) // 4 + 1
    raws = [synth.f32_to_bf16_bits_np((rng.standard_normal((total, 128)) *
                                       np.exp2(rng.integers(-40, 24, (total, 1)))).astype(np.float32))
            for _ in range(B)]
    tail0 = np.zeros((B, 3, 128), np.uint16)
    for b, L0 in enumerate(lens):
        for p in range((L0 // 4) * 4, L0):
            tail0[b, p % 4] = raws[b][p]
    new = np.stack([raws[b][lens[b]:lens[b] + n_new] for b in range(B)])
    codes = torch.zeros(B, cap_blk, 128, dtype=torch.int8, device="cuda")
    scale = torch.zeros(B, cap_blk, dtype=torch.float32, device="cuda")
    len_dev = torch.tensor(lens, dtype=torch.int64, device="cuda")
    spx.spx_pool_append_i8(spx.dims(64), B, to_dev_bf16(new), n_new, pw, to_dev_bf16(tail0),
                           codes, scale, cap_blk, len_dev, total)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    got, gscale = codes.cpu().numpy(), scale.cpu().numpy().astype(np.float64)
    for b, L0 in enumerate(lens):
        end = L0 + n_new
        ref, rscale = oracle.pool_i8(raws[b][:end], pw.astype(np.float64))
        lo, hi = L0 // 4, end // 4
        assert np.array_equal(got[b, lo:hi], ref[lo:hi]), f"seq {b}"
        assert np.array_equal(gscale[b, lo:hi], rscale[lo:hi]), f"seq {b}"


def _token_weights(rng, n_tok):
    """Per-token pooling weights: each block's four are the softmax of N(0,1)
    logits (fp32), as a learned gate normalised over its block would give."""
    g = rng.standard_normal(n_tok + 4)
    wt = np.empty(n_tok, np.float32)
    for b in range(0, n_tok, 4):
        e = np.exp(g[b:b + 4])
        wt[b:b + 4] = (e / e.sum())[:min(4, n_tok - b)]
    return wt


@pytest.mark.parametrize("lens,n_new", [([0, 5, 10, 3], 7), ([3, 0, 1, 2], 1), ([2, 9, 0, 4], 1003)])
def test_pool_append_tok_ragged(lens, n_new):
    """[W1] "IndexPool" with a weight per token: pooled rows, the key tail and
    the weight tail bit for bit against the oracle, over ragged appends that
    complete blocks half from the tail and half from the new tokens."""
    spx = need_gpu()
    rng = np.random.default_rng(100 + n_new)
    w = synth.workload("mid")
    d = spx.dims(64)
    B = len(lens)
    total = max(lens) + n_new
    cap_blk = (total + 3) // 4 + 2
    raw = [synth.f32_to_bf16_bits_np(rng.standard_normal((total, 128)).astype(np.float32))
           for _ in range(B)]
    wts = [_token_weights(rng, total) for _ in range(B)]
    tail0 = np.zeros((B, 3, 128), np.uint16)
    tailw0 = np.zeros((B, 3), np.float32)
    for b, L0 in enumerate(lens):
        for p_ in range((L0 // 4) * 4, L0):
            tail0[b, p_ % 4] = raw[b][p_]
            tailw0[b, p_ % 4] = wts[b][p_]
    new = np.stack([raw[b][lens[b]:lens[b] + n_new] for b in range(B)])
    neww = np.stack([wts[b][lens[b]:lens[b] + n_new] for b in range(B)])
    pooled = torch.zeros(B, cap_blk, 128, dtype=torch.bfloat16, device="cuda")
    tail = to_dev_bf16(tail0)
    tail_w = torch.from_numpy(tailw0).cuda()
    len_dev = torch.tensor(lens, dtype=torch.int64, device="cuda")
    spx.spx_pool_append_tok(d, B, to_dev_bf16(new), torch.from_numpy(neww).cuda(), n_new, tail,
                            tail_w, pooled, cap_blk, len_dev, total)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    got, got_tail, got_tw = bits_of(pooled), bits_of(tail), tail_w.cpu().numpy()
    for b, L0 in enumerate(lens):
        end = L0 + n_new
        ref = oracle.pool_tok(raw[b][:end], wts[b][:end].astype(np.float64))
        lo, hi = L0 // 4, end // 4
        assert np.array_equal(got[b, lo:hi], ref[lo:hi]), f"seq {b}"
        assert (got[b, :lo] == 0).all() and (got[b, hi:] == 0).all()
        for p_ in range((end // 4) * 4, end):
            assert np.array_equal(got_tail[b, p_ % 4], raw[b][p_])
            assert got_tw[b, p_ % 4] == wts[b][p_]


# ----------------------------------------------------------------------------
# Indexer scoring (tcgen05)
# ----------------------------------------------------------------------------
def _score_case(spx, n_vis, cap_blk, q_bits, w_head, keys_bits, stride=None):
    B = len(n_vis)
    d = spx.dims(64)
    max_len = max(n_vis) if max(n_vis) > 0 else 4
    stride = stride or (cap_blk + 7) // 8 * 8
    scores = torch.full((B, stride), float("nan"), device="cuda")
    spx.spx_index_score(d, B, to_dev_bf16(q_bits), torch.from_numpy(w_head.astype(np.float32)).cuda(),
                        to_dev_bf16(keys_bits), cap_blk,
                        torch.tensor(n_vis, dtype=torch.int64, device="cuda"), max_len, scores,
                        stride)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    return scores.cpu().numpy()


def test_index_score_exact_ragged():
    spx = need_gpu()
    w = synth.workload("1m")
    pw = w.pool_weights()
    n_vis = [10403, 517, 3, 4 * 128, 4 * 129 + 1]
    B = len(n_vis)
    cap_blk = 2601
    keys = np.zeros((B, cap_blk, 128), np.uint16)
    for b, n in enumerate(n_vis):
        nb = n // 4
        if nb:
            keys[b, :nb] = oracle.pool(w.raw_keys_np(b, 0, nb * 4), pw)
    q = w.q_idx_np(np.arange(B))
    wh = w.w_head_np(np.arange(B))
    got = _score_case(spx, n_vis, cap_blk, q, wh, keys)
    for b, n in enumerate(n_vis):
        nb = n // 4
        ref = oracle.score(q[b], wh[b].astype(np.float64), keys[b, :nb])
        assert np.array_equal(got[b, :nb], ref.astype(np.float32)), f"row {b}"
        assert np.array_equal(ref.astype(np.float32).astype(np.float64), ref)  # exact data
        assert np.isnan(got[b, nb:]).all()


def test_index_score_needles_and_zero_query():
    spx = need_gpu()
    w = synth.workload("1m")
    pw = w.pool_weights()
    nb = 5000
    raw = w.raw_keys_np(0, 0, nb * 4)
    raw_f = synth.bf16_bits_to_f64_np(raw)
    raw_f[4 * 100:4 * 101] += 16.0  # a needle block
    raw_f[4 * 4999:4 * 5000] += 16.0
    raw = synth.f32_to_bf16_bits_np(raw_f.astype(np.float32))
    keys = oracle.pool(raw, pw)[None]
    q = w.q_idx_np(np.arange(2))
    q[1] = 0  # all-zero query: every score is 0
    wh = w.w_head_np(np.arange(2))
    keys2 = np.concatenate([keys, keys])
    got = _score_case(spx, [nb * 4, nb * 4], nb, q, wh, keys2)
    ref = oracle.score(q[0], wh[0].astype(np.float64), keys[0])
    assert np.array_equal(got[0, :nb], ref.astype(np.float32))
    assert (got[1, :nb] == 0).all()


def test_index_score_general_data_close():
    # non-dyadic data: fp32 sums, compared with a bound on the rounding error
    spx = need_gpu()
    rng = np.random.default_rng(0)
    nb = 3000
    q = synth.f32_to_bf16_bits_np(rng.standard_normal((1, 32, 128)).astype(np.float32))
    keys = synth.f32_to_bf16_bits_np(rng.standard_normal((1, nb, 128)).astype(np.float32))
    wh = rng.standard_normal((1, 32)).astype(np.float32)
    got = _score_case(spx, [nb * 4], nb, q, wh, keys)
    ref = oracle.score(q[0], wh[0].astype(np.float64), keys[0])
    qd, kd = synth.bf16_bits_to_f64_np(q[0]), synth.bf16_bits_to_f64_np(keys[0])
    bound = (np.abs(kd) @ np.abs(qd).T) @ np.abs(wh[0].astype(np.float64)) * 300 * 2.0 ** -24
    assert (np.abs(got[0, :nb] - ref) <= bound + 1e-30).all()


# ----------------------------------------------------------------------------
# Top-k
# ----------------------------------------------------------------------------
def _topk_run(spx, scores_rows, n_vis):
    rows = len(n_vis)
    d = spx.dims(64)
    max_len = max(max(n_vis), 4)
    stride = max(1, max(len(s) for s in scores_rows))
    host = np.full((rows, stride), np.nan, np.float32)
    for r, s in enumerate(scores_rows):
        host[r, :len(s)] = s
    dev = torch.from_numpy(host).cuda()
    nv = torch.tensor(n_vis, dtype=torch.int64, device="cuda")
    idx = torch.full((rows, 512), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    ws = spx.workspace(spx.spx_topk_workspace_size(d, rows, max_len), "cuda")
    spx.spx_topk_blocks(d, rows, dev, stride, nv, max_len, idx, cnt, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy()


def _check_topk(spx, scores_rows, n_vis):
    idx, cnt = _topk_run(spx, scores_rows, n_vis)
    for r, s in enumerate(scores_rows):
        nb = n_vis[r] // 4
        ref = oracle.topk(np.asarray(s[:nb], np.float64), 512)
        assert cnt[r] == ref.size, f"row {r}"
        assert np.array_equal(idx[r, :cnt[r]], ref), f"row {r} nblk={nb}"
        assert (idx[r, cnt[r]:] == -1).all()


def test_topk_sizes_and_ties():
    spx = need_gpu()
    rng = np.random.default_rng(1)
    sizes = [0, 1, 7, 511, 512, 513, 2047, 2048, 2049, 8191, 8192, 8193, 30000, 33792]
    rows, nv = [], []
    for i, nb in enumerate(sizes):
        kind = i % 3
        if kind == 0:
            s = rng.integers(-3, 4, nb).astype(np.float32)  # heavy ties
        elif kind == 1:
            s = (rng.standard_normal(nb) * 100).astype(np.float32)
        else:
            s = np.zeros(nb, np.float32)
            s[rng.random(nb) < 0.5] = -0.0
        rows.append(s)
        nv.append(4 * nb + (i % 4))
    _check_topk(spx, rows, nv)


def test_topk_long_rows_multilevel():
    spx = need_gpu()
    rng = np.random.default_rng(2)
    rows, nv = [], []
    for nb in (262144, 1 << 21):
        s = rng.integers(0, 1000, nb).astype(np.float32)
        s[rng.choice(nb, 600, replace=False)] += 5000.0  # needles compete, with ties
        rows.append(s)
        nv.append(4 * nb)
    # an all-equal long row: the first 512 blocks win
    rows.append(np.full(262144, 2.5, np.float32))
    nv.append(4 * 262144)
    _check_topk(spx, rows, nv)


def test_topk_negative_and_mixed_signs():
    spx = need_gpu()
    rng = np.random.default_rng(3)
    s = (rng.standard_normal(20000) * 1e3).astype(np.float32)
    s[::7] = -np.abs(s[::7])
    s[5] = np.float32(-3.4e38)
    s[6] = np.float32(3.4e38)
    _check_topk(spx, [s, -np.abs(s)], [80000, 80000])


# ----------------------------------------------------------------------------
# Sparse MLA attention
# ----------------------------------------------------------------------------
def _attn_case(spx, H, n_vis, shared=False, bad_ids=False, seed=4):
    rng = np.random.default_rng(seed)
    w = synth.workload("mid")
    rows = len(n_vis)
    cap_tok = max(max(n_vis), 1)
    d = spx.dims(H, 1.0)
    q = w.q_np(np.arange(rows))[:, :H] if H <= w.heads else None
    nlat = 1 if shared else rows
    lat = np.stack([w.latent_np(r, np.arange(cap_tok)) for r in range(nlat)])
    idx = np.full((rows, 512), -1, np.int32)
    cnt = np.zeros(rows, np.int32)
    for r, n in enumerate(n_vis):
        nb = n // 4
        s = rng.standard_normal(nb)
        sel = oracle.topk(s, 512)
        if bad_ids and sel.size > 3:
            sel = sel.copy()
            sel[1] = nb + 5  # out of range: skipped
            sel[2] = -3
        idx[r, :sel.size] = sel
        cnt[r] = sel.size
    out = torch.empty(rows, H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(rows, H, device="cuda")
    max_len = cap_tok
    ws = spx.workspace(spx.spx_attn_workspace_size(d, rows, max_len), "cuda")
    seq_stride = 0 if shared else cap_tok * 512
    spx.spx_sparse_mla_attn(d, rows, to_dev_bf16(q), to_dev_bf16(lat), seq_stride, cap_tok,
                            torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                            torch.tensor(n_vis, dtype=torch.int64, device="cuda"), max_len, out,
                            lse, ws)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_attention_rows(q, lambda r, pos: lat[0 if shared else r][pos], idx, cnt,
                                         n_vis, 1.0)
    return f64_of(out), lse.cpu().numpy(), ref_o, ref_l


@pytest.mark.parametrize("H", [16, 64])
def test_attention_ragged_rows(H):
    spx = need_gpu()
    n_vis = [2051, 9000, 3, 40001, 2052, 8192]
    got, lse, ref, ref_l = _attn_case(spx, H, n_vis)
    assert_attention_close(got, ref, f"H={H}")
    assert np.allclose(lse, ref_l, atol=LSE_ATOL, rtol=0)


def test_attention_empty_and_shared_cache():
    spx = need_gpu()
    n_vis = [0, 1, 4, 7, 5000]
    got, lse, ref, ref_l = _attn_case(spx, 64, n_vis, shared=True)
    assert (got[0] == 0).all() and np.isneginf(lse[0]).all()
    assert_attention_close(got[1:], ref[1:], "shared")
    assert np.allclose(lse[1:], ref_l[1:], atol=LSE_ATOL, rtol=0)


def test_attention_skips_out_of_range_blocks():
    spx = need_gpu()
    got, lse, ref, ref_l = _attn_case(spx, 32, [20000, 6000], bad_ids=True)
    assert_attention_close(got, ref, "bad ids")
    assert np.allclose(lse, ref_l, atol=LSE_ATOL, rtol=0)
