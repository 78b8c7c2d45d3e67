"""INT8 pooled-key cache ([W1] section "양자화: W8A8와 혼합 캐시": far,
compressed indexer entries in INT8): the append, the scoring kernel and the
fused decode through the C ABI against the fp64 oracle's INT8 steps.
Codes, scales, scores and block ids bit-exact; attention within the bf16
tolerance; fused == composed bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import LSE_ATOL, assert_attention_close, f64_of, need_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


def _bf16_bits(values):
    """bf16 bits of values that are exactly representable in bf16."""
    t = torch.tensor(np.asarray(values, np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(values, np.float32)))
    return t.view(torch.int16).numpy().view(np.uint16)


def _bf16_bits_rounded(values):
    """bf16 bits of the nearest bf16 values (library rounding) of any data."""
    t = torch.tensor(np.asarray(values, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _append_i8(spx, lens, n_new, raw, pw, cap_blk):
    """spx_pool_append_i8 of raw[b][lens[b] : lens[b] + n_new] after lens[b] cached tokens."""
    d = spx.dims(64)
    B = len(lens)
    tail0 = np.zeros((B, 3, 128), np.uint16)
    for b, L0 in enumerate(lens):
        for p in range((L0 // 4) * 4, L0):
            tail0[b, p % 4] = raw[b][p]
    new = np.stack([raw[b][lens[b]:lens[b] + n_new] for b in range(B)])
    codes = torch.zeros(B, cap_blk, 128, dtype=torch.int8, device="cuda")
    scale = torch.zeros(B, cap_blk, dtype=torch.float32, device="cuda")
    tail = to_dev_bf16(tail0)
    len_dev = torch.tensor(lens, dtype=torch.int64, device="cuda")
    spx.spx_pool_append_i8(d, B, to_dev_bf16(new), n_new, pw.astype(np.float32), tail, codes,
                           scale, cap_blk, len_dev, max(lens) + n_new)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    return codes.cpu().numpy(), scale.cpu().numpy().astype(np.float64), tail


@pytest.mark.parametrize("lens,n_new", [([0, 5, 10, 3], 7), ([3, 0, 1, 2], 1),
                                        ([2, 9, 0, 4], 1003)])
def test_pool_append_i8_ragged(lens, n_new):
    spx = need_gpu()
    w = synth.workload("1m")  # dyadic 1/64 pool weights: codes round; needle blocks
    pw = w.pool_weights()
    total = max(lens) + n_new
    cap_blk = (total + 3) // 4 + 2
    raw = [w.raw_keys_np(b, 0, total) for b in range(len(lens))]
    got, gscale, tail = _append_i8(spx, lens, n_new, raw, pw, cap_blk)
    got_tail = tail.view(torch.int16).cpu().numpy().view(np.uint16)
    for b, L0 in enumerate(lens):
        end = L0 + n_new
        ref, rscale = oracle.pool_i8(raw[b][:end], pw)
        lo, hi = L0 // 4, end // 4
        assert np.array_equal(got[b, lo:hi], ref[lo:hi]), f"seq {b}"
        assert np.array_equal(gscale[b, lo:hi], rscale[lo:hi]), f"seq {b}"
        assert (got[b, :lo] == 0).all() and (got[b, hi:] == 0).all()
        for p in range((end // 4) * 4, end):
            assert np.array_equal(got_tail[b, p % 4], raw[b][p])


def test_pool_append_i8_magnitudes_zero_blocks_and_ties():
    spx = need_gpu()
    rng = np.random.default_rng(31)
    nblk = 64
    v = rng.integers(-8, 9, (nblk * 4, 128)).astype(np.float32)
    for j in range(nblk):
        v[4 * j:4 * j + 4] *= 2.0 ** (j - 40)  # exponents from 2^-40 to 2^23
    v[4 * 7:4 * 8] = 0.0                      # an all-zero block: scale 1, zero codes
    v[4 * 9:4 * 10] = 0.0
    v[4 * 9, 5] = -3.0                         # one nonzero element
    # a block whose codes land exactly half-way: x = (k + 1/2) 2^e
    v[4 * 11:4 * 12] = 0.0
    v[4 * 11, :4] = [127.0, 2.5, -2.5, 3.5]
    raw = _bf16_bits(v)
    pw = np.array([1.0, 0.0, 0.0, 0.0])
    got, gscale, _ = _append_i8(spx, [0], nblk * 4, [raw], pw, nblk)
    ref, rscale = oracle.pool_i8(raw, pw)
    assert np.array_equal(got[0], ref) and np.array_equal(gscale[0], rscale)
    assert rscale[7] == 1.0 and not ref[7].any()
    assert ref[11, :4].tolist() == [127, 2, -2, 4]


def _score_i8(spx, n_vis, cap_blk, q_bits, w_head, codes, scales, stride=None):
    B = len(n_vis)
    d = spx.dims(64)
    max_len = max(n_vis) if max(n_vis) > 0 else 4
    stride = stride or (cap_blk + 7) // 8 * 8
    scores = torch.full((B, stride), float("nan"), device="cuda")
    ws = spx.workspace(spx.spx_index_score_i8_workspace_size(d, B), "cuda")
    spx.spx_index_score_i8(d, B, to_dev_bf16(q_bits),
                           torch.from_numpy(w_head.astype(np.float32)).cuda(),
                           torch.from_numpy(codes).cuda(),
                           torch.from_numpy(scales.astype(np.float32)).cuda(), cap_blk,
                           torch.tensor(n_vis, dtype=torch.int64, device="cuda"), max_len, scores,
                           stride, ws)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    return scores.cpu().numpy()


def test_index_score_i8_exact_ragged():
    spx = need_gpu()
    w = synth.workload("1m")
    pw = w.pool_weights()
    n_vis = [10403, 517, 3, 4 * 128, 4 * 129 + 1]
    B = len(n_vis)
    cap_blk = 2601
    codes = np.zeros((B, cap_blk, 128), np.int8)
    scales = np.ones((B, cap_blk), np.float64)
    for b, n in enumerate(n_vis):
        nb = n // 4
        if nb:
            codes[b, :nb], scales[b, :nb] = oracle.pool_i8(w.raw_keys_np(b, 0, nb * 4), pw)
    q = w.q_idx_np(np.arange(B))
    wh = w.w_head_np(np.arange(B))
    got = _score_i8(spx, n_vis, cap_blk, q, wh, codes, scales)
    for b, n in enumerate(n_vis):
        nb = n // 4
        ref = oracle.score_i8(q[b], wh[b].astype(np.float64), codes[b, :nb], scales[b, :nb])
        assert np.array_equal(ref.astype(np.float32).astype(np.float64), ref)  # exact data
        assert np.array_equal(got[b, :nb], ref.astype(np.float32)), f"row {b}"
        assert np.isnan(got[b, nb:]).all()


def test_index_score_i8_zero_query_and_general_data():
    spx = need_gpu()
    rng = np.random.default_rng(32)
    B, nblk = 3, 700
    cap_blk = nblk
    raw = [_bf16_bits_rounded(rng.standard_normal((nblk * 4, 128))) for _ in range(B)]
    pw = np.array([0.4, 0.3, 0.2, 0.1])
    codes = np.zeros((B, cap_blk, 128), np.int8)
    scales = np.zeros((B, cap_blk))
    for b in range(B):
        codes[b], scales[b] = oracle.pool_i8(raw[b], pw)
    q = np.stack([_bf16_bits_rounded(rng.standard_normal((32, 128))) for _ in range(B)])
    q[1] = 0  # a zero query: every code 0, every score 0
    wh = rng.uniform(0.1, 1.0, (B, 32))
    got = _score_i8(spx, [nblk * 4] * B, cap_blk, q, wh, codes, scales)
    for b in range(B):
        ref = oracle.score_i8(q[b], wh[b], codes[b], scales[b])
        if b == 1:
            assert (got[b, :nblk] == 0).all() and (ref == 0).all()
            continue
        # general data: the fp32 head sum rounds; the integer dots stay exact
        assert np.allclose(got[b, :nblk], ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


# ----------------------------------------------------------------------------
# Fused decode with the INT8 cache
# ----------------------------------------------------------------------------
def _decode_state_i8(name, **kw):
    need_gpu()
    import bench
    return bench.DecodeState(synth.workload(name), torch.device("cuda", 0), keys="int8", **kw)


def _oracle_decode_i8(st, rows):
    """Oracle steps 1-4 on the INT8 cache; codes from the oracle's own pooling."""
    res = []
    nb = st.L // 4
    for b in rows:
        bg = st.b_offset + b
        codes, scale = oracle.pool_i8(st.raw_keys_host(b), st.w.pool_weights())
        s = oracle.score_i8(st.w.q_idx_np([bg])[0], st.w.w_head_np([bg])[0].astype(np.float64),
                            codes[:nb], scale[:nb])
        idx = oracle.topk(s)
        pos = oracle.token_set(idx, st.L)
        out, lse = oracle.attention(st.w.q_np([bg])[0], st.latent_rows_host(b, pos),
                                    st.w.sm_scale)
        res.append(dict(idx=idx, out=out, lse=lse, codes_last=codes[-1], scale_last=scale[-1]))
    return res


def _check_decode_i8(st, rows):
    spx = need_gpu()
    st.step()
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    idx = st.idx.cpu().numpy()
    cnt = st.count.cpu().numpy()
    out = f64_of(st.out)
    lse = st.lse.cpu().numpy()
    codes_last = st.pooled[:, -1].cpu().numpy()
    scale_last = st.k_scale[:, -1].cpu().numpy().astype(np.float64)
    ref = _oracle_decode_i8(st, rows)
    for i, b in enumerate(rows):
        r = ref[i]
        # the block completed by this step's append
        assert np.array_equal(codes_last[b], r["codes_last"]), f"pooled block of seq {b}"
        assert scale_last[b] == r["scale_last"]
        assert cnt[b] == r["idx"].size
        assert np.array_equal(idx[b, :cnt[b]], r["idx"]), f"seq {b}"
        assert (idx[b, cnt[b]:] == -1).all()
        assert np.allclose(lse[b], r["lse"], atol=LSE_ATOL, rtol=0)
    assert_attention_close(out[rows], np.stack([r["out"] for r in ref]), st.w.name + " int8")
    return ref


def test_mid_decode_i8_all_rows():
    st = _decode_state_i8("mid")
    _check_decode_i8(st, list(range(st.B)))


@pytest.mark.slow
def test_1m_decode_i8():
    """The benchmark's 1M-token workload with the INT8 cache, all four sequences."""
    st = _decode_state_i8("1m")
    ref = _check_decode_i8(st, list(range(st.B)))
    for b, r in enumerate(ref):
        nb = set(st.w.needle_blocks(b).tolist())
        assert len(nb & set(r["idx"].tolist())) >= 256


def test_fused_i8_equals_composed():
    spx = need_gpu()
    st = _decode_state_i8("mid", B=3)
    st.step()
    torch.cuda.synchronize()
    out_f, idx_f, cnt_f, lse_f = st.out.clone(), st.idx.clone(), st.count.clone(), st.lse.clone()
    d, B, L = st.d, st.B, st.L
    len_after = torch.full((B,), L, dtype=torch.int64, device="cuda")
    spx.spx_pool_append_i8(d, B, st.raw_new, 1, st.pool_w, st.tail, st.pooled, st.k_scale,
                           st.cap_blk, st.len_dev, L)
    stride = L // 4
    scores = torch.empty(B, stride, device="cuda")
    ws0 = spx.workspace(spx.spx_index_score_i8_workspace_size(d, B), "cuda")
    spx.spx_index_score_i8(d, B, st.q_idx, st.w_head, st.pooled, st.k_scale, st.cap_blk,
                           len_after, L, scores, stride, ws0)
    idx = torch.empty_like(st.idx)
    cnt = torch.empty_like(st.count)
    ws = spx.workspace(spx.spx_topk_workspace_size(d, B, L), "cuda")
    spx.spx_topk_blocks(d, B, scores, stride, len_after, L, idx, cnt, ws)
    out = torch.empty_like(st.out)
    lse = torch.empty_like(st.lse)
    ws2 = spx.workspace(spx.spx_attn_workspace_size(d, B, L), "cuda")
    spx.spx_sparse_mla_attn(d, B, st.q, st.latent, L * 512, L, idx, cnt, len_after, L, out, lse,
                            ws2)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_f) and torch.equal(cnt, cnt_f)
    assert torch.equal(out.view(torch.int16), out_f.view(torch.int16))
    assert torch.equal(lse, lse_f)
    # the INT8 selection keeps most of the bf16 cache's selection on this data
    st16 = __import__("bench").DecodeState(st.w, torch.device("cuda", 0), B=3)
    st16.step()
    torch.cuda.synchronize()
    for b in range(B):
        a = set(st16.idx[b].cpu().tolist())
        assert len(a & set(idx_f[b].cpu().tolist())) >= 400


# ---------------------------------------------------------------------------
# Chunked prefill on the INT8 cache (spx_prefill_chunk_i8)

def _prefill_state_i8(pos0, T):
    need_gpu()
    import bench
    return bench.PrefillState(synth.workload("prefill"), torch.device("cuda", 0), pos0=pos0, T=T,
                              keys="int8")


def _check_prefill_i8(st, queries, attn_queries=None):
    """Codes and scales of the chunk's blocks, the ids of `queries` bit-exact
    against the oracle's INT8 steps (pool_i8, score_i8 over the query's
    visible blocks, full-sort top-k), and attention of `attn_queries` (all of
    `queries` by default) within the bf16 tolerance."""
    from concurrent.futures import ThreadPoolExecutor
    spx = need_gpu()
    st.step()
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    codes, scale = oracle.pool_i8(st.raw_keys_host(), st.w.pool_weights())
    lo, hi = st.pos0 // 4, (st.pos0 + st.T) // 4
    assert np.array_equal(st.pooled[0, lo:hi].cpu().numpy(), codes[lo:hi]), "codes of the chunk"
    assert np.array_equal(st.k_scale[0, lo:hi].cpu().numpy().astype(np.float64), scale[lo:hi])
    idx, cnt = st.idx.cpu().numpy(), st.count.cpu().numpy()
    rows = st.pos0 + np.asarray(queries)
    q_idx = st.w.q_idx_np(rows)
    w_head = st.w.w_head_np(rows).astype(np.float64)

    def select(i):
        n = st.pos0 + queries[i] + 1
        s = oracle.score_i8(q_idx[i], w_head[i], codes[:n // 4], scale[:n // 4], nthreads=1)
        sel = oracle.topk(s)
        return sel, oracle.token_set(sel, n)

    with ThreadPoolExecutor(max_workers=oracle.threads(0)) as ex:
        ref = list(ex.map(select, range(len(queries))))
    bad = [t for t, (sel, _) in zip(queries, ref)
           if cnt[t] != sel.size or not np.array_equal(idx[t, :cnt[t]], sel)
           or not (idx[t, cnt[t]:] == -1).all()]
    assert not bad, f"{len(bad)} of {len(queries)} queries select other blocks, first {bad[:8]}"
    attn = list(queries) if attn_queries is None else list(attn_queries)
    pos_of = {t: pos for t, (_, pos) in zip(queries, ref)}
    q = st.w.q_np(st.pos0 + np.asarray(attn))
    out, lse = f64_of(st.out), st.lse.cpu().numpy()
    outs = []
    for i, t in enumerate(attn):
        o, l = oracle.attention(q[i], st.w.latent_np(0, pos_of[t]), st.w.sm_scale)
        assert np.allclose(lse[t], l, atol=LSE_ATOL, rtol=0), f"query {t}"
        outs.append(o)
    assert_attention_close(out[attn], np.stack(outs), "prefill int8")


def test_prefill_i8_small_all_queries():
    # 8190 cached tokens (a 2-token tail), 100 new ones: the 2048-token budget
    # boundary, several 128-block tiles and a partial group of 8 queries
    st = _prefill_state_i8(8190, 100)
    _check_prefill_i8(st, list(range(100)))


def test_prefill_i8_short_context_dense():
    st = _prefill_state_i8(1000, 64)
    _check_prefill_i8(st, list(range(64)))


def test_prefill_i8_full_chunk_stratified():
    """The prefill benchmark's shape (4096 new tokens on 131,072 cached ones)
    on the INT8 cache: ids of the 256-query stratified subset bit-exact, and
    the attention of 32 of them."""
    import bench
    st = _prefill_state_i8(None, None)
    sub = bench.stratified_prefill_queries(st.T)
    _check_prefill_i8(st, sub, attn_queries=sub[::8])
