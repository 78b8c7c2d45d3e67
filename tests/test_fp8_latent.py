"""FP8 (E4M3) latent cache ([W1] section "양자화: W8A8와 혼합 캐시": recent,
important entries in FP8): the quantising cache write against the oracle's
codes and row exponents bit for bit, and attention over the FP8 cache against
the oracle's attention over the dequantised rows, through the C ABI, on
ragged rows (skipped ids, partial tails, a shared cache) and the mid and 1M
decode workloads."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import (LSE_ATOL, assert_attention_close, bits_of, f64_of, need_gpu,
                          to_dev_bf16)

pytestmark = pytest.mark.gpu


def _quant(spx, lat_bits):
    n = lat_bits.shape[0]
    codes = torch.zeros(n, 512, dtype=torch.uint8, device="cuda")
    exps = torch.zeros(n, dtype=torch.int32, device="cuda")
    spx.spx_latent_quant_fp8(to_dev_bf16(lat_bits), n, codes, exps)
    torch.cuda.synchronize()
    return codes, exps


def test_latent_quant_fp8_matches_oracle():
    spx = need_gpu()
    rng = np.random.default_rng(8)
    n = 600
    x = rng.standard_normal((n, 512)) * np.exp2(rng.integers(-60, 60, (n, 1)))
    x[3] = 0.0                       # an all-zero row: exponent 0, zero codes
    x[4] = -0.0
    x[5, :7] = [448.0, 3.0, -1.0, 0.5, 416.0, 432.0, 440.0]  # grid points and ties
    x[5, 7:] = 0.0
    x[6, 0] = 448.0 * 2.0 ** -40     # the 448 boundary at a small scale
    x[6, 1:] = -1e-14
    bits = synth.f32_to_bf16_bits_np(x.astype(np.float32))
    codes, exps = _quant(spx, bits)
    ref_c, ref_e = oracle.latent_fp8(bits)
    assert np.array_equal(exps.cpu().numpy().astype(np.int64), ref_e)
    assert np.array_equal(codes.cpu().numpy(), ref_c)
    assert ref_e[3] == 0 and not ref_c[3].any()


def _fp8_attn(spx, d, rows, q_bits, codes, exps, seq_stride, cap_tok, idx, cnt, n_vis, max_len):
    H = d.heads
    out = torch.empty(rows, H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(rows, H, device="cuda")
    ws = spx.workspace(spx.spx_attn_fp8_workspace_size(d, rows, max_len), "cuda")
    spx.spx_sparse_mla_attn_fp8(d, rows, q_bits, codes, exps, seq_stride, cap_tok, idx, cnt,
                                n_vis, max_len, out, lse, ws)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    return f64_of(out), lse.cpu().numpy()


@pytest.mark.parametrize("shared", [False, True])
def test_attention_fp8_ragged_rows(shared):
    spx = need_gpu()
    rng = np.random.default_rng(9)
    w = synth.workload("mid")
    n_vis = [2051, 9001, 3, 40002, 0, 4]
    rows, H = len(n_vis), 64
    cap_tok = max(n_vis)
    d = spx.dims(H, 1.0)
    nlat = 1 if shared else rows
    lat = np.stack([w.latent_np(r, np.arange(cap_tok)) for r in range(nlat)])
    codes, exps = _quant(spx, lat.reshape(-1, 512))
    idx = np.full((rows, 512), -1, np.int32)
    cnt = np.zeros(rows, np.int32)
    for r, n in enumerate(n_vis):
        sel = oracle.topk(rng.standard_normal(n // 4), 512)
        if sel.size > 3:
            sel = sel.copy()
            sel[1] = n // 4 + 5  # out of range: skipped
            sel[2] = -3
        idx[r, :sel.size] = sel
        cnt[r] = sel.size
    q = w.q_np(np.arange(rows))
    got, lse = _fp8_attn(spx, d, rows, to_dev_bf16(q), codes, exps, 0 if shared else cap_tok * 512,
                         cap_tok, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                         torch.tensor(n_vis, dtype=torch.int64, device="cuda"), cap_tok)
    refs, ref_l = [], []
    for r, n in enumerate(n_vis):
        sel = [int(b) for b in idx[r, :cnt[r]] if 0 <= b < n // 4]
        pos = oracle.token_set(np.array(sel, np.int32), n)
        o, l = oracle.attention_fp8(q[r], lat[0 if shared else r][pos], 1.0) if pos.size else \
            (np.zeros((H, 512)), np.full(H, -np.inf))
        refs.append(o)
        ref_l.append(l)
    assert (got[4] == 0).all() and np.isneginf(lse[4]).all()  # the empty row
    keep = [r for r in range(rows) if r != 4]
    assert_attention_close(got[keep], np.stack(refs)[keep], "fp8 ragged")
    assert np.allclose(lse[keep], np.stack(ref_l)[keep], atol=LSE_ATOL, rtol=0)


def _decode_fp8_check(name, sample_rows=64):
    """The decode workload: the selection of the bf16 fused step, then
    attention over the FP8 copy of the whole latent cache, against the
    oracle's FP8 attention of every row; codes of the selected rows checked
    against the oracle's quantisation."""
    spx = need_gpu()
    import bench
    st = bench.DecodeState(synth.workload(name), torch.device("cuda", 0))
    st.step()
    torch.cuda.synchronize()
    B, L = st.B, st.L
    codes = torch.empty(B * L, 512, dtype=torch.uint8, device="cuda")
    exps = torch.empty(B * L, dtype=torch.int32, device="cuda")
    spx.spx_latent_quant_fp8(st.latent.view(-1, 512), B * L, codes, exps)
    n_vis = torch.full((B,), L, dtype=torch.int64, device="cuda")
    got, lse = _fp8_attn(spx, st.d, B, st.q, codes, exps, L * 512, L, st.idx, st.count, n_vis, L)
    idx, cnt = st.idx.cpu().numpy(), st.count.cpu().numpy()
    refs = []
    for b in range(B):
        pos = oracle.token_set(idx[b, :cnt[b]], L)
        rows = st.latent_rows_host(b, pos)
        rc, re = oracle.latent_fp8(rows[:sample_rows])
        gpos = torch.from_numpy(b * L + pos[:sample_rows]).cuda()
        assert np.array_equal(codes[gpos].cpu().numpy(), rc), f"codes of seq {b}"
        assert np.array_equal(exps[gpos].cpu().numpy().astype(np.int64), re)
        o, l = oracle.attention_fp8(st.w.q_np([st.b_offset + b])[0], rows, st.w.sm_scale)
        assert np.allclose(lse[b], l, atol=LSE_ATOL, rtol=0), f"seq {b}"
        refs.append(o)
    assert_attention_close(got, np.stack(refs), f"fp8 {name}")


def test_decode_fp8_latent_mid():
    _decode_fp8_check("mid")


@pytest.mark.slow
def test_decode_fp8_latent_1m():
    _decode_fp8_check("1m")
