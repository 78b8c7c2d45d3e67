"""Seeded synthetic inputs for the sparse-attention layer (IndexPool -> indexer
-> top-k -> sparse MLA attention).

This module is shared by the fp64 oracle tests and the CUDA path: it holds no
arithmetic of the method itself, only the recipe that draws inputs.  Every
value is a pure function of (seed, tensor tag, flat element index), so any
slice of a tensor can be regenerated on its own, on the host (numpy) or on a
CUDA device (torch integer ops), and both produce identical bits.

Generator: the splitmix64 finaliser (Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) applied to a Weyl counter.

Value recipes (readings of the workload descriptions; the pages print none):
  * integer keys in [lo, hi]: lo + (top 31 bits of the draw) mod (hi - lo + 1)
  * "~N(0,1)" values: Irwin-Hall sum of the four 16-bit lanes of one draw,
    centred and scaled by sqrt(3) in fp32, so the result is bit-identical on
    every IEEE machine (no transcendental functions), then rounded to bf16
    with round-to-nearest-even done in integer arithmetic.
  * indexer head weights w_h in {1/4, 1/2, 1}.
  * pool weights: either fixed (1/2, 1/4, 1/8, 1/8) or the softmax of four
    seeded N(0,1) logits rounded to multiples of 1/64 with the rounding
    residual added to the largest so that they sum to exactly 1.

bf16 tensors are returned as raw uint16 bit patterns (numpy) or int16 tensors
(torch) that callers view as bfloat16.
"""
from __future__ import annotations

import math

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1

# Tensor tags: each logical tensor of a workload draws from its own stream.
TAG_RAW_K = 1
TAG_Q_IDX = 2
TAG_W_HEAD = 3
TAG_Q = 4
TAG_LATENT = 5
TAG_POOL_W = 6
TAG_NEEDLE = 7
TAG_MISC = 8

SQRT3_F32 = np.float32(math.sqrt(3.0))


def _mix64_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tag: int) -> int:
    """64-bit key of one tensor's stream."""
    return _mix64_int((seed * 0x1000193) ^ (tag << 40) ^ 0x5DEECE66D)


# --------------------------------------------------------------------------
# numpy (host) implementation
# --------------------------------------------------------------------------
def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * np.uint64(M1)
    z = z ^ (z >> np.uint64(27))
    z = z * np.uint64(M2)
    return z ^ (z >> np.uint64(31))


def draws_np(seed: int, tag: int, index) -> np.ndarray:
    """uint64 draw for each flat element index (any int array)."""
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(stream_key(seed, tag)) + (idx + np.uint64(1)) * np.uint64(GOLDEN)
        return _mix64_np(z)


def ints_np(seed, tag, index, lo, hi) -> np.ndarray:
    d = draws_np(seed, tag, index)
    top = (d >> np.uint64(33)).astype(np.int64)
    return lo + top % (hi - lo + 1)


def _normal_f32_np(d: np.ndarray, scale_f32: np.float32) -> np.ndarray:
    s = np.zeros(d.shape, dtype=np.int64)
    for lane in range(4):
        s += ((d >> np.uint64(16 * lane)) & np.uint64(0xFFFF)).astype(np.int64)
    x = ((s + 2).astype(np.float32) / np.float32(65536.0)) - np.float32(2.0)  # exact
    return (x * scale_f32).astype(np.float32)  # one IEEE fp32 rounding


def f32_to_bf16_bits_np(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, nearest-even, as integer arithmetic on the bits."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64_np(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16_np(seed, tag, index, scale=1.0) -> np.ndarray:
    """bf16 bits of an approximately N(0, scale^2) value per index."""
    sc = np.float32(np.float32(scale) * SQRT3_F32) if scale != 1.0 else SQRT3_F32
    return f32_to_bf16_bits_np(_normal_f32_np(draws_np(seed, tag, index), sc))


def int_bf16_np(seed, tag, index, lo, hi) -> np.ndarray:
    """bf16 bits of an integer value in [lo, hi] (exact in bf16 for |v| <= 256)."""
    v = ints_np(seed, tag, index, lo, hi).astype(np.float32)
    return f32_to_bf16_bits_np(v)


# --------------------------------------------------------------------------
# torch implementation (host or device); identical bits to the numpy one
# --------------------------------------------------------------------------
def _s64(v: int) -> int:
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr(torch, z, k):
    """Logical right shift of int64 tensors."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix64_t(torch, z):
    z = z ^ _lsr(torch, z, 30)
    z = z * _s64(M1)
    z = z ^ _lsr(torch, z, 27)
    z = z * _s64(M2)
    return z ^ _lsr(torch, z, 31)


def draws_t(seed, tag, index):
    """int64 (two's complement of the uint64 draw) for an int64 index tensor."""
    import torch
    z = (index + 1) * _s64(GOLDEN) + _s64(stream_key(seed, tag))
    return _mix64_t(torch, z)


def ints_t(seed, tag, index, lo, hi):
    import torch
    d = draws_t(seed, tag, index)
    top = _lsr(torch, d, 33)
    return lo + torch.remainder(top, hi - lo + 1)


def f32_to_bf16_bits_t(x):
    import torch
    u = x.to(torch.float32).contiguous().view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    r = torch.where(r >= 0x8000, r - 0x10000, r)
    return r.to(torch.int16)


def normal_bf16_t(seed, tag, index, scale=1.0):
    import torch
    d = draws_t(seed, tag, index)
    s = torch.zeros_like(d)
    for lane in range(4):
        s = s + (_lsr(torch, d, 16 * lane) & 0xFFFF if lane else d & 0xFFFF)
    x = ((s + 2).to(torch.float32) / 65536.0) - 2.0
    sc = float(np.float32(np.float32(scale) * SQRT3_F32)) if scale != 1.0 else float(SQRT3_F32)
    x = x * torch.tensor(sc, dtype=torch.float32, device=x.device)
    return f32_to_bf16_bits_t(x)


def int_bf16_t(seed, tag, index, lo, hi):
    import torch
    return f32_to_bf16_bits_t(ints_t(seed, tag, index, lo, hi).to(torch.float32))


# --------------------------------------------------------------------------
# Workload descriptions
# --------------------------------------------------------------------------
IDX_HEADS = 32
IDX_DIM = 128
POOL = 4
TOPK_BLOCKS = 512
LATENT = 512

MLA_Q_SCALE = 1.0 / math.sqrt(512.0)


class Workload:
    """One synthetic workload: shapes plus the value recipe.

    Decode: B sequences, query at position L-1 sees n = L tokens; the step
    appends the raw indexer key of token L-1, so the cache before the step
    holds L-1 tokens.  Prefill: batch 1, a cache of `pos0` tokens and T new
    query tokens; query t sees pos0 + t + 1 tokens.
    """

    def __init__(self, name, kind, B, L, heads, seed, pool_w_mode, needles=0,
                 T=0, sm_scale=1.0):
        self.name = name
        self.kind = kind  # "decode" | "prefill"
        self.B = B
        self.L = L  # decode: visible tokens per sequence; prefill: pos0
        self.heads = heads
        self.seed = seed
        self.pool_w_mode = pool_w_mode  # "fixed" | "dyadic64"
        self.needles = needles
        self.T = T
        self.sm_scale = sm_scale

    # ---- sizes ----
    @property
    def total_tokens(self):
        return self.L if self.kind == "decode" else self.L + self.T

    @property
    def nblk(self):
        return self.total_tokens // POOL

    # ---- pool weights (host, 4 doubles summing exactly to 1) ----
    def pool_weights(self) -> np.ndarray:
        if self.pool_w_mode == "fixed":
            return np.array([0.5, 0.25, 0.125, 0.125], dtype=np.float64)
        d = draws_np(self.seed, TAG_POOL_W, np.arange(4))
        logits = _normal_f32_np(d, SQRT3_F32).astype(np.float64)
        e = np.exp(logits - logits.max())
        p = e / e.sum()
        w = np.round(p * 64.0) / 64.0
        w[int(np.argmax(w))] += 1.0 - w.sum()
        assert abs(w.sum() - 1.0) == 0.0 and (w >= 0).all()
        return w

    # ---- needles: sorted distinct block ids per sequence ----
    def needle_blocks(self, b: int) -> np.ndarray:
        if self.needles == 0:
            return np.zeros(0, dtype=np.int64)
        nb = self.nblk
        chosen = []
        seen = set()
        i = 0
        while len(chosen) < self.needles:
            cand = int(ints_np(self.seed, TAG_NEEDLE, np.array([b * 1_000_003 + i]), 0, nb - 1)[0])
            i += 1
            if cand not in seen:
                seen.add(cand)
                chosen.append(cand)
        return np.array(sorted(chosen), dtype=np.int64)

    # ---- raw indexer keys [B, tokens, 128] int-valued bf16 ----
    def raw_key_index(self, b, tok, d):
        return (np.asarray(b, np.int64) * self.total_tokens + np.asarray(tok, np.int64)) * IDX_DIM + np.asarray(d, np.int64)

    def raw_keys_np(self, b, tok0, tok1) -> np.ndarray:
        """bf16 bits [tok1-tok0, 128] of sequence b."""
        tok = np.arange(tok0, tok1, dtype=np.int64)
        idx = self.raw_key_index(b, tok[:, None], np.arange(IDX_DIM)[None, :])
        v = ints_np(self.seed, TAG_RAW_K, idx, -8, 8)
        if self.needles:
            nb = self.needle_blocks(b)
            hit = np.isin(tok // POOL, nb)
            v = v + 16 * hit[:, None]
        return f32_to_bf16_bits_np(v.astype(np.float32))

    def raw_keys_t(self, b, tok0, tok1, device, needle_t=None):
        import torch
        tok = torch.arange(tok0, tok1, dtype=torch.int64, device=device)
        d = torch.arange(IDX_DIM, dtype=torch.int64, device=device)
        idx = (b * self.total_tokens + tok[:, None]) * IDX_DIM + d[None, :]
        v = ints_t(self.seed, TAG_RAW_K, idx, -8, 8)
        if self.needles:
            if needle_t is None:
                needle_t = torch.as_tensor(self.needle_blocks(b), device=device)
            hit = torch.isin(tok // POOL, needle_t)
            v = v + 16 * hit[:, None].to(torch.int64)
        return f32_to_bf16_bits_t(v.to(torch.float32))

    # ---- indexer query [rows, 32, 128] ints in [-4,4]; head weights ----
    def q_idx_np(self, rows) -> np.ndarray:
        rows = np.asarray(rows, np.int64)
        idx = (rows[:, None, None] * IDX_HEADS + np.arange(IDX_HEADS)[None, :, None]) * IDX_DIM + np.arange(IDX_DIM)[None, None, :]
        return int_bf16_np(self.seed, TAG_Q_IDX, idx, -4, 4)

    def w_head_np(self, rows) -> np.ndarray:
        rows = np.asarray(rows, np.int64)
        idx = rows[:, None] * IDX_HEADS + np.arange(IDX_HEADS)[None, :]
        k = ints_np(self.seed, TAG_W_HEAD, idx, 0, 2)
        return np.array([0.25, 0.5, 1.0], dtype=np.float32)[k]

    # ---- MLA query [rows, H, 512] ~ N(0,1)/sqrt(512) ----
    def q_np(self, rows) -> np.ndarray:
        rows = np.asarray(rows, np.int64)
        H = self.heads
        idx = (rows[:, None, None] * H + np.arange(H)[None, :, None]) * LATENT + np.arange(LATENT)[None, None, :]
        return normal_bf16_np(self.seed, TAG_Q, idx, scale=MLA_Q_SCALE)

    # ---- MLA latent rows [B, tokens, 512] ~ N(0,1) ----
    def latent_np(self, b, tok) -> np.ndarray:
        tok = np.asarray(tok, np.int64)
        idx = (b * self.total_tokens + tok[:, None]) * LATENT + np.arange(LATENT)[None, :]
        return normal_bf16_np(self.seed, TAG_LATENT, idx)

    def latent_t(self, b, tok0, tok1, device):
        import torch
        tok = torch.arange(tok0, tok1, dtype=torch.int64, device=device)
        d = torch.arange(LATENT, dtype=torch.int64, device=device)
        idx = (b * self.total_tokens + tok[:, None]) * LATENT + d[None, :]
        return normal_bf16_t(self.seed, TAG_LATENT, idx)


def _cfg(name):
    if name == "tiny":
        return Workload("tiny_decode_B1_L8192_H16", "decode", B=1, L=8192, heads=16, seed=1, pool_w_mode="fixed")
    if name == "dense":
        return Workload("dense_fallback_B64_L1536_H64", "decode", B=64, L=1536, heads=64, seed=2, pool_w_mode="fixed")
    if name == "mid":
        return Workload("mid_decode_B16_L131072_H64", "decode", B=16, L=131072, heads=64, seed=3, pool_w_mode="dyadic64")
    if name == "1m":
        return Workload("decode_B4_L1048576_H64_needles600", "decode", B=4, L=1 << 20, heads=64, seed=4,
                        pool_w_mode="dyadic64", needles=600)
    if name == "prefill":
        return Workload("prefill_T4096_pos131072_H64", "prefill", B=1, L=131072, heads=64, seed=5,
                        pool_w_mode="dyadic64", T=4096)
    raise KeyError(name)


WORKLOADS = ("tiny", "dense", "mid", "1m", "prefill")


def workload(name: str) -> Workload:
    return _cfg(name)
