"""spx_topk_blocks_noalloc: the top-k selection for callers that cannot give
the library scratch memory (its candidate lists live in an array built into
the library).  Its results must equal spx_topk_blocks' on the same inputs,
call after call, since both run the same kernels; only the scratch differs.

This file is collected last so that a failure here cannot hide another
test's result in a run that stops at the first failure."""
import numpy as np
import pytest
import torch


def _spx():
    from conftest import build_lib
    build_lib()
    import long_context_decode_indexpool_b200 as spx
    return spx


def test_noalloc_rejects_requests_above_its_scratch():
    # host-side check, nothing is launched: 4096 rows of 33,792 blocks need
    # far more candidate scratch than the built-in array holds
    spx = _spx()
    d = spx.dims(64, 1.0)
    need = spx.spx_topk_workspace_size(d, 4096, 135168)
    assert need > spx.NOALLOC_SCRATCH_BYTES
    fake = 1 << 20
    with pytest.raises(spx.SpxError) as e:
        spx.spx_topk_blocks_noalloc(d, 4096, fake, 33792, fake, 135168, fake, fake, stream=0)
    assert e.value.status == 4


def _scores(rng, rows, nblk):
    s = rng.integers(0, 2000, (rows, nblk)).astype(np.float32)
    for r in range(rows):
        s[r, rng.choice(nblk, 600, replace=False)] += 10000.0  # competing needles, with ties
    return s


@pytest.mark.gpu
def test_noalloc_matches_workspace_version_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spx = _spx()
    d = spx.dims(64, 1.0)
    rng = np.random.default_rng(11)
    # two calls in a row with different inputs and plans: one merge level,
    # then two merge levels (the larger one reuses the same built-in array)
    for rows, nblk in ((4, 262144), (2, 1 << 21)):
        max_len = 4 * nblk
        assert spx.spx_topk_workspace_size(d, rows, max_len) <= spx.NOALLOC_SCRATCH_BYTES
        scores = torch.from_numpy(_scores(rng, rows, nblk)).cuda()
        n_vis = torch.tensor([max_len - 4 * r for r in range(rows)], dtype=torch.int64,
                             device="cuda")
        ws = spx.workspace(spx.spx_topk_workspace_size(d, rows, max_len), "cuda")
        idx_ref = torch.empty(rows, 512, dtype=torch.int32, device="cuda")
        cnt_ref = torch.empty(rows, dtype=torch.int32, device="cuda")
        spx.spx_topk_blocks(d, rows, scores, nblk, n_vis, max_len, idx_ref, cnt_ref, ws)
        idx = torch.full((rows, 512), -5, dtype=torch.int32, device="cuda")
        cnt = torch.full((rows,), -5, dtype=torch.int32, device="cuda")
        spx.spx_topk_blocks_noalloc(d, rows, scores, nblk, n_vis, max_len, idx, cnt)
        torch.cuda.synchronize()
        assert torch.equal(cnt, cnt_ref)
        assert torch.equal(idx, idx_ref)
        assert (cnt.cpu().numpy() == 512).all()
