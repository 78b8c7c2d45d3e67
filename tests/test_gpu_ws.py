"""HiSparse-style device working set ([W3] "HiSparse는 전체 이력을 GPU 밖으로
옮긴다"): the latent history in pinned host memory, a fixed pool of block
slots on the device, and per step a fetch of only the selected blocks that
are not resident.  Over several steps with different queries, every step's
output must equal, bit for bit, the attention over the same cache in device
memory, and be within the specification's tolerance of the oracle; the
hit/fetch counters and the slot maps must stay consistent."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import LSE_ATOL, assert_attention_close, bits_of, f64_of, need_gpu

pytestmark = pytest.mark.gpu


def test_working_set_steps_match_device_cache_and_oracle():
    spx = need_gpu()
    import bench
    w = synth.workload("mid")
    dev = torch.device("cuda", 0)
    st = bench.DecodeState(w, dev, B=4)
    B, L, H = st.B, st.L, st.H
    cap_blk = L // 4
    nslots = 1024  # 4,096 tokens of the 131,072 per sequence stay on the device
    host_lat = st.latent.cpu().pin_memory()
    pool = torch.zeros(B, nslots + 1, 4, 512, dtype=torch.bfloat16, device=dev)
    slot_blk = torch.full((B, nslots), -1, dtype=torch.int32, device=dev)
    blk_slot = torch.full((B, cap_blk), -1, dtype=torch.int32, device=dev)
    stamp = torch.full((B, nslots), -1, dtype=torch.int32, device=dev)
    hand = torch.zeros(B, dtype=torch.int32, device=dev)
    stats = torch.zeros(B, 2, dtype=torch.int64, device=dev)
    ws = spx.workspace(spx.spx_ws_workspace_size(st.d, B, nslots), dev)
    ws_a = spx.workspace(spx.spx_attn_workspace_size(st.d, B, L), dev)
    n_vis = torch.full((B,), L, dtype=torch.int64, device=dev)
    rng = np.random.default_rng(3)
    g = torch.Generator(device=dev).manual_seed(3)
    total_sel = 0
    prev = None
    for step in range(5):
        # a new indexer query each step (the previous one half the time, so
        # that blocks stay selected across steps)
        q_idx = st.q_idx if step % 2 == 0 else (
            torch.randint(-4, 5, st.q_idx.shape, generator=g, device=dev).to(torch.bfloat16))
        st.step(q_idx=q_idx)
        torch.cuda.synchronize()
        idx, cnt = st.idx.clone(), st.count.clone()
        out_ws = torch.empty_like(st.out)
        lse_ws = torch.empty_like(st.lse)
        spx.spx_sparse_mla_attn_ws(st.d, B, st.q, host_lat.data_ptr(), L * 512, L, idx, cnt, n_vis,
                                   L, pool, nslots, slot_blk, blk_slot, stamp, hand, step, stats,
                                   out_ws, lse_ws, ws)
        out_dev = torch.empty_like(st.out)
        lse_dev = torch.empty_like(st.lse)
        spx.spx_sparse_mla_attn(st.d, B, st.q, st.latent, L * 512, L, idx, cnt, n_vis, L, out_dev,
                                lse_dev, ws_a)
        torch.cuda.synchronize()
        assert spx.spx_device_error() == 0
        assert torch.equal(out_ws.view(torch.int16), out_dev.view(torch.int16)), f"step {step}"
        assert torch.equal(lse_ws, lse_dev), f"step {step}"
        total_sel += int(cnt.sum())
        # maps: every selected block is resident in the slot that holds it
        sb, bs = slot_blk.cpu().numpy(), blk_slot.cpu().numpy()
        idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        for b in range(B):
            for blk in idx_h[b, :cnt_h[b]]:
                assert bs[b, blk] >= 0 and sb[b, bs[b, blk]] == blk
            res = np.nonzero(bs[b] >= 0)[0]
            assert np.array_equal(np.sort(sb[b][bs[b, res]]), res)  # bijective
        if step == 4:
            # the oracle for the last step
            qi = q_idx.view(torch.int16).cpu().numpy().view(np.uint16)
            refs = []
            for b in range(B):
                pos = oracle.token_set(idx_h[b, :cnt_h[b]], L)
                o, l = oracle.attention(w.q_np([b])[0], st.latent_rows_host(b, pos), w.sm_scale)
                assert np.allclose(lse_ws[b].cpu().numpy(), l, atol=LSE_ATOL, rtol=0)
                refs.append(o)
            assert_attention_close(f64_of(out_ws), np.stack(refs), "working set")
        prev = idx_h
    hits, fetched = stats.cpu().numpy().sum(axis=0)
    assert hits + fetched == total_sel
    assert hits > 0 and fetched > 0  # repeated queries hit, new ones fetch
