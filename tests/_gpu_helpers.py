"""Helpers shared by the GPU parity tests: device/host conversions, the
attention tolerance of the workload specification, oracle references."""
import numpy as np
import pytest
import torch

import oracle

# Attention tolerance fixed by the workload specification: bf16 outputs
# against the fp64 oracle.
MAX_ABS = 1e-2
REL_L2 = 5e-3
LSE_ATOL = 2e-3  # lse is fp32 from fp32 logits of the same bf16 inputs


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_lib
    build_lib()
    import long_context_decode_indexpool_b200 as spx
    return spx


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_attention_close(got: np.ndarray, ref: np.ndarray, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / denom) if denom > 0 else float(np.linalg.norm(got))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def oracle_attention_rows(q_bits, latent_rows_fn, idx_rows, count_rows, n_vis_rows, sm_scale):
    """Oracle out/lse for each row given its selected blocks."""
    outs, lses = [], []
    for r in range(len(n_vis_rows)):
        n = int(n_vis_rows[r])
        nblk = n // 4
        sel = [int(b) for b in idx_rows[r][: int(count_rows[r])] if 0 <= int(b) < nblk]
        pos = oracle.token_set(np.array(sel, dtype=np.int32), n)
        rows = latent_rows_fn(r, pos)
        o, l = oracle.attention(q_bits[r], rows, sm_scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)
