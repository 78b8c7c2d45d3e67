"""Whole-layer parity: the fused decode and prefill entry points on the
workloads of the specification, in the configuration bench.py times,
against the fp64 oracle (block ids bit-exact, outputs within tolerance),
plus fused == composed bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import (LSE_ATOL, assert_attention_close, bits_of, f64_of, need_gpu,
                          oracle_attention_rows, to_dev_bf16)

pytestmark = pytest.mark.gpu


def _decode_state(name, **kw):
    need_gpu()
    import bench
    return bench.DecodeState(synth.workload(name), torch.device("cuda", 0), **kw)


def _oracle_decode(st, rows):
    """Oracle steps 2-4 of the given local rows; pooled keys from the oracle's own pooling."""
    res = []
    for b in rows:
        raw = st.raw_keys_host(b)
        pooled = oracle.pool(raw, st.w.pool_weights())
        r = oracle.decode_query(st.w.q_idx_np([st.b_offset + b])[0],
                                st.w.w_head_np([st.b_offset + b])[0].astype(np.float64), pooled,
                                st.L, st.w.q_np([st.b_offset + b])[0],
                                lambda pos, b=b: st.latent_rows_host(b, pos), st.w.sm_scale)
        r["pooled_last"] = pooled[-1]
        res.append(r)
    return res


def _check_decode(st, rows):
    st.step()
    torch.cuda.synchronize()
    spx = need_gpu()
    assert spx.spx_device_error() == 0
    idx = st.idx.cpu().numpy()
    cnt = st.count.cpu().numpy()
    out = f64_of(st.out)
    lse = st.lse.cpu().numpy()
    pooled_last = bits_of(st.pooled[:, -1])
    ref = _oracle_decode(st, rows)
    for i, b in enumerate(rows):
        r = ref[i]
        assert np.array_equal(pooled_last[b], r["pooled_last"]), f"pooled block of seq {b}"
        assert cnt[b] == r["idx"].size
        assert np.array_equal(idx[b, :cnt[b]], r["idx"]), f"seq {b}"
        assert (idx[b, cnt[b]:] == -1).all()
        assert np.allclose(lse[b], r["lse"], atol=LSE_ATOL, rtol=0)
    assert_attention_close(out[rows], np.stack([r["out"] for r in ref]), st.w.name)
    return ref


def test_tiny_decode():
    st = _decode_state("tiny")
    ref = _check_decode(st, [0])
    assert ref[0]["positions"].size == 2048  # 512 blocks x 4, no tail (L % 4 == 0)


def test_dense_fallback_equals_dense_attention():
    st = _decode_state("dense")
    ref = _check_decode(st, list(range(st.B)))
    for r in ref:
        assert r["idx"].tolist() == list(range(384))
        assert r["positions"].tolist() == list(range(1536))


def test_mid_decode_all_rows():
    st = _decode_state("mid")
    _check_decode(st, list(range(st.B)))


@pytest.mark.slow
def test_1m_decode_bench_configuration():
    """The benchmark's workload, all four sequences, in the bench's launch configuration."""
    st = _decode_state("1m")
    ref = _check_decode(st, list(range(st.B)))
    # the needles dominate the selection: most selected blocks are needles
    for b, r in enumerate(ref):
        nb = set(st.w.needle_blocks(b).tolist())
        assert len(nb & set(r["idx"].tolist())) >= 256


def test_fused_equals_composed_and_no_append_path():
    spx = need_gpu()
    st = _decode_state("mid", B=3)
    st.step()
    torch.cuda.synchronize()
    out_f, idx_f, cnt_f, lse_f = st.out.clone(), st.idx.clone(), st.count.clone(), st.lse.clone()
    d, B, L = st.d, st.B, st.L
    # composed: append, score, top-k, attention
    len_after = torch.full((B,), L, dtype=torch.int64, device="cuda")
    spx.spx_pool_append(d, B, st.raw_new, 1, st.pool_w, st.tail, st.pooled, st.cap_blk,
                        st.len_dev, L)
    stride = L // 4
    scores = torch.empty(B, stride, device="cuda")
    spx.spx_index_score(d, B, st.q_idx, st.w_head, st.pooled, st.cap_blk, len_after, L, scores,
                        stride)
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
    # raw_k = NULL: no append, the query sees len_dev tokens (here L after the append)
    spx.spx_decode_fused(d, B, None, None, st.tail, st.pooled, st.cap_blk, len_after, st.q_idx,
                         st.w_head, st.q, st.latent, st.cap_tok, L, out, lse, idx, cnt, st.ws)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_f)
    assert torch.equal(out.view(torch.int16), out_f.view(torch.int16))


@pytest.mark.parametrize("levels", [4, 256])
def test_fused_selection_heavy_ties(levels):
    """Rows whose scores take few distinct values: the 512th score is shared by
    thousands of blocks spread over every CTA of the row, so the fused
    selection must resolve ties at the cut inside CTAs and in the merge."""
    spx = need_gpu()
    rng = np.random.default_rng(levels)
    B, nblk = 3, 100003
    L = 4 * nblk + 1  # one tail token
    # pooled key b = c_b * e_0; query heads all e_0 with weight 1: s_b = 32 c_b
    c = rng.integers(0, levels, (B, nblk)).astype(np.float32)
    c[1, :] = 7.0  # a row of equal scores
    keys = np.zeros((B, nblk + 1, 128), np.float32)  # capacity for the tail token's block
    keys[:, :nblk, 0] = c
    pooled = torch.from_numpy(keys).to(torch.bfloat16).cuda()
    q_idx = torch.zeros(B, 32, 128, dtype=torch.bfloat16, device="cuda")
    q_idx[:, :, 0] = 1.0
    w_head = torch.ones(B, 32, device="cuda")
    d = spx.dims(16, 1.0)
    latent = torch.zeros(B, L, 512, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(B, 16, 512, dtype=torch.bfloat16, device="cuda")
    len_dev = torch.full((B,), L, dtype=torch.int64, device="cuda")
    out = torch.empty(B, 16, 512, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(B, 512, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    ws = spx.workspace(spx.spx_decode_workspace_size(d, B, L), "cuda")
    spx.spx_decode_fused(d, B, None, None, None, pooled, nblk + 1, len_dev, q_idx, w_head, q,
                         latent, L, L, out, None, idx, cnt, ws)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    idx = idx.cpu().numpy()
    cnt = cnt.cpu().numpy()
    for r in range(B):
        ref = oracle.topk(32.0 * c[r].astype(np.float64), 512)
        assert cnt[r] == 512 and np.array_equal(idx[r], ref), f"row {r}"
    assert idx[1].tolist() == list(range(512))


# ----------------------------------------------------------------------------
# Chunked prefill
# ----------------------------------------------------------------------------
def _prefill_state(pos0, T):
    need_gpu()
    import bench
    return bench.PrefillState(synth.workload("prefill"), torch.device("cuda", 0), pos0=pos0, T=T)


def _check_prefill(st, queries):
    spx = need_gpu()
    st.step()
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    raw = st.raw_keys_host()
    pw = st.w.pool_weights()
    pooled = oracle.pool(raw, pw)
    total = st.pos0 + st.T
    got_pooled = bits_of(st.pooled[0, : total // 4])
    lo = st.pos0 // 4
    assert np.array_equal(got_pooled[lo:], pooled[lo:]), "pooled blocks of the chunk"
    idx = st.idx.cpu().numpy()
    cnt = st.count.cpu().numpy()
    out = f64_of(st.out)
    lse = st.lse.cpu().numpy()
    rows = st.pos0 + np.asarray(queries)
    q_idx = st.w.q_idx_np(rows)
    w_head = st.w.w_head_np(rows).astype(np.float64)
    q = st.w.q_np(rows)
    outs = []
    for i, t in enumerate(queries):
        n = st.pos0 + t + 1
        s, sel, pos = oracle.select_query(q_idx[i], w_head[i], pooled, n)
        assert cnt[t] == sel.size, f"query {t}"
        assert np.array_equal(idx[t, :cnt[t]], sel), f"query {t}"
        o, l = oracle.attention(q[i], st.w.latent_np(0, pos), st.w.sm_scale)
        assert np.allclose(lse[t], l, atol=LSE_ATOL, rtol=0), f"query {t}"
        outs.append(o)
    assert_attention_close(out[list(queries)], np.stack(outs), "prefill")


def test_prefill_small_all_queries():
    # cache of 8190 tokens (a 2-token tail), 100 new tokens: crosses the
    # 2048-block budget boundary and several tiles of 128 blocks
    st = _prefill_state(8190, 100)
    _check_prefill(st, list(range(100)))


def test_prefill_short_context_dense():
    # every query sees fewer than 2052 tokens: all blocks selected
    st = _prefill_state(1000, 64)
    _check_prefill(st, list(range(64)))


@pytest.mark.parametrize("nblk0,levels", [(30000, 4), (30000, 256), (30000, 1), (40000, 256),
                                          (50001, 4)])
def test_prefill_selection_heavy_ties(nblk0, levels):
    """Prefill rows whose scores take few distinct values, so that the
    512th-best score is shared by thousands of blocks.  30,000 cached blocks
    go through the sampled one-CTA-per-row selection (4 and 1 levels overflow
    its survivor lists and fall back to the staged radix kernel, 256 levels
    do not), 40,000 (past the sampled path's stage) straight to the staged
    kernel, 50,001 (past that) through the key histograms and chunk lists;
    every path must return the oracle's ids (ties to the lower block) for
    every query of the chunk."""
    spx = need_gpu()
    rng = np.random.default_rng(nblk0 + levels)
    T = 8
    pos0 = 4 * nblk0
    total = pos0 + T
    cap_blk = total // 4 + 1
    # cached pooled key b = c_b e_0; query heads all e_0 with weight 1:
    # s_b = 32 c_b; the chunk's own tokens are zero keys (score 0)
    c = rng.integers(0, levels, nblk0).astype(np.float32)
    keys = np.zeros((1, cap_blk, 128), np.float32)
    keys[0, :nblk0, 0] = c
    pooled = torch.from_numpy(keys).to(torch.bfloat16).cuda()
    tail = torch.zeros(1, 3, 128, dtype=torch.bfloat16, device="cuda")
    raw = torch.zeros(T, 128, dtype=torch.bfloat16, device="cuda")
    pool_w = np.full(4, 0.25, np.float32)
    q_idx = torch.zeros(T, 32, 128, dtype=torch.bfloat16, device="cuda")
    q_idx[:, :, 0] = 1.0
    w_head = torch.ones(T, 32, device="cuda")
    d = spx.dims(16, 1.0)
    q = torch.zeros(T, 16, 512, dtype=torch.bfloat16, device="cuda")
    latent = torch.zeros(total, 512, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(T, 16, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(T, 16, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, 512, dtype=torch.int32, device="cuda")
    cnt = torch.empty(T, dtype=torch.int32, device="cuda")
    ws = spx.workspace(spx.spx_prefill_workspace_size(d, T, pos0), "cuda")
    spx.spx_prefill_chunk(d, T, raw, pool_w, tail, pooled, cap_blk, pos0, q_idx, w_head, q,
                          latent, total, out, lse, idx, cnt, ws)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    scores = np.zeros(cap_blk, np.float64)
    scores[:nblk0] = 32.0 * c
    for t in range(T):
        nb = (pos0 + t + 1) // 4
        ref = oracle.topk(scores[:nb], 512)
        assert cnt[t] == ref.size and np.array_equal(idx[t, :cnt[t]], ref), f"query {t}"
        assert (idx[t, cnt[t]:] == -1).all()


@pytest.mark.slow
def test_prefill_full_chunk_all_ids_stratified_attention():
    """The benchmark's prefill workload (4096 new tokens on a 131,072-token
    cache) in the bench's launch configuration: the selected block ids of
    every one of the 4096 queries bit-exact against the oracle, and the
    attention output and lse of a 256-query stratified subset within the
    specification's tolerance."""
    from concurrent.futures import ThreadPoolExecutor
    spx = need_gpu()
    st = _prefill_state(None, None)
    st.step()
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    pw = st.w.pool_weights()
    pooled = oracle.pool(st.raw_keys_host(), pw)
    lo = st.pos0 // 4
    assert np.array_equal(bits_of(st.pooled[0, lo:(st.pos0 + st.T) // 4]), pooled[lo:])
    idx, cnt = st.idx.cpu().numpy(), st.count.cpu().numpy()
    T = st.T
    rows = st.pos0 + np.arange(T)
    q_idx = st.w.q_idx_np(rows)
    w_head = st.w.w_head_np(rows).astype(np.float64)

    def ids(t):  # oracle steps 2-3 of query t (one thread per query)
        _, sel, _ = oracle.select_query(q_idx[t], w_head[t], pooled, st.pos0 + t + 1, nthreads=1)
        return sel

    with ThreadPoolExecutor(max_workers=oracle.threads(0)) as ex:
        sels = list(ex.map(ids, range(T)))
    bad = [t for t in range(T)
           if cnt[t] != sels[t].size or not np.array_equal(idx[t, :cnt[t]], sels[t])
           or not (idx[t, cnt[t]:] == -1).all()]
    assert not bad, f"{len(bad)} of {T} queries select other blocks, first {bad[:8]}"

    import bench
    sub = bench.stratified_prefill_queries(T)
    assert len(sub) == 256
    q = st.w.q_np(st.pos0 + np.asarray(sub))
    out, lse = f64_of(st.out), st.lse.cpu().numpy()

    def attend(i):
        t = sub[i]
        pos = oracle.token_set(sels[t], st.pos0 + t + 1)
        return oracle.attention(q[i], st.w.latent_np(0, pos), st.w.sm_scale)

    with ThreadPoolExecutor(max_workers=oracle.threads(0)) as ex:
        refs = list(ex.map(attend, range(len(sub))))
    for i, t in enumerate(sub):
        assert np.allclose(lse[t], refs[i][1], atol=LSE_ATOL, rtol=0), f"query {t}"
    assert_attention_close(out[sub], np.stack([r[0] for r in refs]), "prefill 4096")


def test_decode_ragged_lengths_one_call():
    """Rows of very different lengths in one fused call: dense rows (<= 2051
    tokens, one with a partial tail), a row whose 512th score is shared by
    many blocks, and longer rows spread over several selection chunks."""
    spx = need_gpu()
    rng = np.random.default_rng(7)
    lens = [9001, 2051, 1203, 20000, 36003, 4]  # tokens seen by each query
    B, max_len = len(lens), 36004
    cap_blk, cap_tok = max_len // 4 + 1, max_len
    pw = np.array([0.5, 0.25, 0.125, 0.125])
    keys = np.zeros((B, cap_blk, 128), np.uint16)
    pooled_ref = []
    for b, n in enumerate(lens):
        raw = rng.integers(-8, 9, (n - n % 4, 128)).astype(np.float32)
        if b == 3:
            raw[:, :] = np.sign(raw)  # few distinct scores: a crowded cut bin
        p = oracle.pool(synth.f32_to_bf16_bits_np(raw), pw)
        keys[b, :p.shape[0]] = p
        pooled_ref.append(p)
    q_idx = synth.f32_to_bf16_bits_np(rng.integers(-4, 5, (B, 32, 128)).astype(np.float32))
    w_head = np.array([0.25, 0.5, 1.0], np.float32)[rng.integers(0, 3, (B, 32))]
    H = 64
    q = synth.f32_to_bf16_bits_np((rng.standard_normal((B, H, 512)) / np.sqrt(512)).astype(np.float32))
    # latent rows: multiples of 1/16 in [-1/2, 1/2] (exact in bf16), made on the device
    g = torch.Generator(device="cuda").manual_seed(7)
    lat_dev = (torch.randint(-8, 9, (B, cap_tok, 512), generator=g, device="cuda",
                             dtype=torch.int16).to(torch.bfloat16) / 16)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    d = spx.dims(H, 1.0)
    len_dev = torch.tensor(lens, dtype=torch.int64, device="cuda")
    out = torch.empty(B, H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, 512, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    ws = spx.workspace(spx.spx_decode_workspace_size(d, B, max_len), "cuda")
    spx.spx_decode_fused(d, B, None, None, None, dev(keys), cap_blk, len_dev, dev(q_idx),
                         torch.from_numpy(w_head).cuda(), dev(q), lat_dev, cap_tok, max_len,
                         out, lse, idx, cnt, ws)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    got, lse = f64_of(out), lse.cpu().numpy()
    refs = []
    for b, n in enumerate(lens):
        r = oracle.decode_query(q_idx[b], w_head[b].astype(np.float64), pooled_ref[b], n, q[b],
                                lambda pos, b=b: bits_of(lat_dev[b, torch.from_numpy(pos).cuda()]),
                                1.0)
        assert cnt[b] == r["idx"].size, f"row {b}"
        assert np.array_equal(idx[b, :cnt[b]], r["idx"]), f"row {b}"
        assert (idx[b, cnt[b]:] == -1).all()
        assert np.allclose(lse[b], r["lse"], atol=LSE_ATOL, rtol=0), f"row {b}"
        refs.append(r["out"])
    assert_attention_close(got, np.stack(refs), "ragged")
    assert cnt[1] == 512 and cnt[2] == 300 and cnt[5] == 1


def test_indexshare_other_layer_on_shared_selection():
    """IndexShare: a second layer attends over the first layer's selection
    with its own query and latent cache (no indexer pass of its own)."""
    spx = need_gpu()
    st = _decode_state("tiny")
    st.step()
    torch.cuda.synchronize()
    B, L, H = st.B, st.L, st.H
    g = torch.Generator(device="cuda").manual_seed(11)
    lat2 = (torch.randint(-8, 9, (B, st.cap_tok, 512), generator=g, device="cuda",
                          dtype=torch.int16).to(torch.bfloat16) / 16)
    q2 = (torch.randn(B, H, 512, generator=g, device="cuda") / 512 ** 0.5).to(torch.bfloat16)
    n_vis = torch.full((B,), L, dtype=torch.int64, device="cuda")
    out2 = torch.empty_like(st.out)
    lse2 = torch.empty_like(st.lse)
    ws = spx.workspace(spx.spx_attn_workspace_size(st.d, B, L), "cuda")
    spx.spx_sparse_mla_attn(st.d, B, q2, lat2, st.cap_tok * 512, st.cap_tok, st.idx, st.count,
                            n_vis, L, out2, lse2, ws)
    torch.cuda.synchronize()
    idx, cnt = st.idx.cpu().numpy(), st.count.cpu().numpy()
    outs = []
    for b in range(B):
        pos = oracle.token_set(idx[b, :cnt[b]], L)
        o, l = oracle.attention(bits_of(q2[b]), bits_of(lat2[b, torch.from_numpy(pos).cuda()]),
                                st.w.sm_scale)
        assert np.allclose(lse2[b].cpu().numpy(), l, atol=LSE_ATOL, rtol=0)
        outs.append(o)
    assert_attention_close(f64_of(out2), np.stack(outs), "indexshare")


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_host_resident_latent_cache_matches_oracle(name):
    """HiSparse-style host-resident latent cache ([W3] "HiSparse는 전체 이력을
    GPU 밖으로 옮긴다"): the attention reads the selected rows straight from
    pinned host memory.  The block ids equal the oracle's bit for bit, the
    output and lse are within the specification's tolerance of the oracle's
    fp64 attention, and the result is the same, bit for bit, as with the
    cache in HBM."""
    spx = need_gpu()
    st = _decode_state(name)
    st.step()
    torch.cuda.synchronize()
    out_dev, lse_dev, idx_dev = st.out.clone(), st.lse.clone(), st.idx.clone()
    host_lat = st.latent.cpu().pin_memory()  # mapped into the device's address space (UVA)
    out = torch.empty_like(st.out)
    lse = torch.empty_like(st.lse)
    len_after = torch.full((st.B,), st.L, dtype=torch.int64, device="cuda")
    spx.spx_decode_fused(st.d, st.B, None, None, st.tail, st.pooled, st.cap_blk, len_after,
                         st.q_idx, st.w_head, st.q, host_lat.data_ptr(), st.cap_tok, st.L, out,
                         lse, st.idx, st.count, st.ws)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    rows = list(range(st.B))
    ref = _oracle_decode(st, rows)
    idx, cnt = st.idx.cpu().numpy(), st.count.cpu().numpy()
    lse_h = lse.cpu().numpy()
    for b in rows:
        assert cnt[b] == ref[b]["idx"].size
        assert np.array_equal(idx[b, :cnt[b]], ref[b]["idx"]), f"seq {b}"
        assert np.allclose(lse_h[b], ref[b]["lse"], atol=LSE_ATOL, rtol=0), f"seq {b}"
    assert_attention_close(f64_of(out), np.stack([r["out"] for r in ref]), f"host latent {name}")
    assert torch.equal(st.idx, idx_dev)
    assert torch.equal(out.view(torch.int16), out_dev.view(torch.int16))
    assert torch.equal(lse, lse_dev)


def test_decode_with_per_token_pool_weights():
    """A decode step whose IndexPool weights come with the tokens: the cache
    is built and the new token appended with spx_pool_append_tok, then the
    fused call runs steps 2-4 (raw_k = NULL).  Block ids bit-exact and
    attention within tolerance against the oracle's per-token pooling."""
    spx = need_gpu()
    w = synth.workload("mid")
    rng = np.random.default_rng(77)
    B, L, H = 3, 32768 + 4, 64
    cap_blk, cap_tok = L // 4, L
    d = spx.dims(H, w.sm_scale)
    dev = torch.device("cuda", 0)
    raw = [w.raw_keys_np(b, 0, L) for b in range(B)]
    g = rng.standard_normal((B, L))
    wt = np.exp(g.reshape(B, L // 4, 4))
    wt = (wt / wt.sum(axis=2, keepdims=True)).astype(np.float32).reshape(B, L)
    pooled = torch.zeros(B, cap_blk, 128, dtype=torch.bfloat16, device=dev)
    tail = torch.zeros(B, 3, 128, dtype=torch.bfloat16, device=dev)
    tail_w = torch.zeros(B, 3, device=dev)
    zero = torch.zeros(B, dtype=torch.int64, device=dev)
    # the cache as earlier steps left it: L - 1 tokens, then the new token
    spx.spx_pool_append_tok(d, B, to_dev_bf16(np.stack([r[:L - 1] for r in raw])),
                            torch.from_numpy(wt[:, :L - 1].copy()).to(dev), L - 1, tail, tail_w,
                            pooled, cap_blk, zero, L - 1)
    len_dev = torch.full((B,), L - 1, dtype=torch.int64, device=dev)
    spx.spx_pool_append_tok(d, B, to_dev_bf16(np.stack([r[L - 1:] for r in raw])),
                            torch.from_numpy(wt[:, L - 1:].copy()).to(dev), 1, tail, tail_w,
                            pooled, cap_blk, len_dev, L)
    n_vis = torch.full((B,), L, dtype=torch.int64, device=dev)
    rows = np.arange(B)
    q_idx = w.q_idx_np(rows)
    w_head = w.w_head_np(rows)
    q = w.q_np(rows)
    g2 = torch.Generator(device=dev).manual_seed(5)
    lat = (torch.randint(-8, 9, (B, cap_tok, 512), generator=g2, device=dev,
                         dtype=torch.int16).to(torch.bfloat16) / 16)
    out = torch.empty(B, H, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, device=dev)
    idx = torch.empty(B, 512, dtype=torch.int32, device=dev)
    cnt = torch.empty(B, dtype=torch.int32, device=dev)
    ws = spx.workspace(spx.spx_decode_workspace_size(d, B, L), dev)
    spx.spx_decode_fused(d, B, None, None, None, pooled, cap_blk, n_vis, to_dev_bf16(q_idx),
                         torch.from_numpy(w_head).to(dev), to_dev_bf16(q), lat, cap_tok, L, out,
                         lse, idx, cnt, ws)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    idx, cnt, lse = idx.cpu().numpy(), cnt.cpu().numpy(), lse.cpu().numpy()
    refs = []
    for b in range(B):
        pk = oracle.pool_tok(raw[b], wt[b].astype(np.float64))
        assert np.array_equal(bits_of(pooled[b]), pk), f"pooled cache of seq {b}"
        r = oracle.decode_query(q_idx[b], w_head[b].astype(np.float64), pk, L, q[b],
                                lambda pos, b=b: bits_of(lat[b, torch.from_numpy(pos).to(dev)]),
                                w.sm_scale)
        assert cnt[b] == r["idx"].size and np.array_equal(idx[b, :cnt[b]], r["idx"]), f"seq {b}"
        assert np.allclose(lse[b], r["lse"], atol=LSE_ATOL, rtol=0)
        refs.append(r["out"])
    assert_attention_close(f64_of(out), np.stack(refs), "per-token pooling")
