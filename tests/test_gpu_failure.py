"""Failure detection on the GPU without a fault: a kernel's bounded wait is
made to run out on purpose (mbarriers that nothing completes, through the
library's self-test call), and the host must learn of it through the device
error word while the context stays usable for the next, correct, step."""
import numpy as np
import pytest
import torch

import oracle
import synth
from _gpu_helpers import assert_attention_close, f64_of, need_gpu

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000  # 1 ms


def test_bounded_wait_gives_up_drains_and_reports():
    spx = need_gpu()
    assert spx.spx_device_error() == 0
    res = torch.full((6,), -1, dtype=torch.int64, device="cuda")
    spx.spx_selftest_wait_timeout(LIMIT_NS, res)
    torch.cuda.synchronize()
    first_ok, second_ok, drained, t_first, t_second, copy_ok = res.cpu().tolist()
    assert first_ok == 0, "the wait on a barrier nothing completes must give up"
    assert LIMIT_NS <= t_first < 200 * LIMIT_NS, t_first
    # the second role gives up on the abort flag, far before its own limit
    assert second_ok == 0
    assert t_second < 200 * LIMIT_NS, t_second
    # the bulk copy in flight at the timeout was waited for and is intact
    assert drained == 1 and copy_ok == 1
    assert spx.spx_device_error() == 1  # kErrWaitTimeout
    assert spx.spx_device_error() == 0  # reading clears it


def test_context_usable_after_a_timeout():
    """After a wait gave up, the next decode step on the same context runs
    without error and matches the oracle."""
    spx = need_gpu()
    res = torch.zeros(6, dtype=torch.int64, device="cuda")
    spx.spx_selftest_wait_timeout(LIMIT_NS, res)
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 1
    import bench
    w = synth.workload("tiny")
    st = bench.DecodeState(w, torch.device("cuda", 0))
    st.step()
    torch.cuda.synchronize()
    assert spx.spx_device_error() == 0
    pooled = oracle.pool(st.raw_keys_host(0), w.pool_weights())
    ref = oracle.decode_query(w.q_idx_np([0])[0], w.w_head_np([0])[0].astype(np.float64), pooled,
                              w.L, w.q_np([0])[0], lambda pos: st.latent_rows_host(0, pos),
                              w.sm_scale)
    cnt = int(st.count[0].item())
    assert np.array_equal(st.idx[0, :cnt].cpu().numpy(), ref["idx"])
    assert_attention_close(f64_of(st.out[0]), ref["out"], "after timeout")
