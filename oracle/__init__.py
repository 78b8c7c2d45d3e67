"""fp64 CPU oracle of the sparse-attention layer (test infrastructure).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import
this package.  The product library never does; it shares no code with it.

The arithmetic lives in ``spx_oracle.cpp`` (plain fp64 loops, std::sort for
top-k); this module builds it with g++ on first use and wraps each function
with numpy marshalling.  ``decode_query`` and ``prefill_query`` compose the
four steps exactly as the pages order them: pooled-key cache -> indexer
scores -> top-k blocks -> attention over the gathered latent rows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spx_oracle.cpp")
_LIB = os.path.join(_HERE, "libspx_oracle.so")
_lock = threading.Lock()
_lib = None

POOL = 4
TOPK_BLOCKS = 512


def build(force: bool = False) -> str:
    """Compile the oracle shared library (g++, -O2, strict fp64 semantics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
               "-ffp-contract=off", "-fno-fast-math", "-o", _LIB + ".tmp", _SRC]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64 = ctypes.c_int64
            lib.orc_threads.argtypes = [ctypes.c_int]
            lib.orc_threads.restype = ctypes.c_int
            lib.orc_bf16_rne.argtypes = [ctypes.c_double]
            lib.orc_bf16_rne.restype = ctypes.c_uint16
            lib.orc_pool.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P, P]
            lib.orc_pool.restype = None
            lib.orc_pool_tok.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P, P]
            lib.orc_pool_tok.restype = None
            lib.orc_score.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P, i64, P, ctypes.c_int]
            lib.orc_score.restype = None
            lib.orc_quant_i8.argtypes = [P, ctypes.c_int, P]
            lib.orc_quant_i8.restype = ctypes.c_int
            lib.orc_pool_i8.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P, P, P]
            lib.orc_pool_i8.restype = None
            lib.orc_score_i8.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P, P, i64, P, ctypes.c_int]
            lib.orc_score_i8.restype = None
            lib.orc_e4m3_bits.argtypes = [ctypes.c_double]
            lib.orc_e4m3_bits.restype = ctypes.c_uint8
            lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_value.restype = ctypes.c_double
            lib.orc_quant_e4m3.argtypes = [P, ctypes.c_int, P]
            lib.orc_quant_e4m3.restype = ctypes.c_int
            lib.orc_topk.argtypes = [P, i64, i64, P]
            lib.orc_topk.restype = i64
            lib.orc_token_set.argtypes = [P, i64, i64, ctypes.c_int, P]
            lib.orc_token_set.restype = i64
            lib.orc_attention.argtypes = [P, ctypes.c_int, ctypes.c_int, P, i64, ctypes.c_double, P, P]
            lib.orc_attention.restype = None
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def threads(requested: int = 0) -> int:
    return _load().orc_threads(requested)


def bf16_rne(v: float) -> int:
    """bf16 bit pattern of the nearest-even rounding of a double."""
    return int(_load().orc_bf16_rne(float(v)))


def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def pool(raw_bits: np.ndarray, w, pool_size: int = POOL) -> np.ndarray:
    """IndexPool: [n_tok, dim] raw bf16 keys -> [n_tok // pool, dim] bf16 bits."""
    raw = np.ascontiguousarray(raw_bits, dtype=np.uint16)
    n_tok, dim = raw.shape
    w = np.ascontiguousarray(w, dtype=np.float64)
    assert w.shape == (pool_size,)
    out = np.zeros((n_tok // pool_size, dim), dtype=np.uint16)
    _load().orc_pool(_p(raw), n_tok, dim, pool_size, _p(w), _p(out))
    return out


def pool_tok(raw_bits: np.ndarray, wt, pool_size: int = POOL) -> np.ndarray:
    """IndexPool with a weight per token: [n_tok, dim] raw bf16 keys and
    [n_tok] weights (each block's four summing to 1) -> [n_tok // pool, dim]
    bf16 bits."""
    raw = np.ascontiguousarray(raw_bits, dtype=np.uint16)
    n_tok, dim = raw.shape
    wt = np.ascontiguousarray(wt, dtype=np.float64)
    assert wt.shape == (n_tok,)
    out = np.zeros((n_tok // pool_size, dim), dtype=np.uint16)
    _load().orc_pool_tok(_p(raw), n_tok, dim, pool_size, _p(wt), _p(out))
    return out


def score(q_bits: np.ndarray, w_head, keys_bits: np.ndarray, nthreads: int = 0) -> np.ndarray:
    """Indexer scores [nblk] (fp64) of one query [heads, dim] against pooled keys."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    heads, dim = q.shape
    w = np.ascontiguousarray(w_head, dtype=np.float64)
    assert w.shape == (heads,)
    keys = np.ascontiguousarray(keys_bits, dtype=np.uint16)
    nblk = keys.shape[0] if keys.size else 0
    assert nblk == 0 or keys.shape[1] == dim
    out = np.zeros(nblk, dtype=np.float64)
    if nblk:
        _load().orc_score(_p(q), _p(w), heads, dim, _p(keys), nblk, _p(out), nthreads)
    return out


def quant_i8(x) -> tuple[np.ndarray, int]:
    """INT8 code of one vector: (int8 codes, e) with x ~= 2^e * codes."""
    v = np.ascontiguousarray(x, dtype=np.float64).reshape(-1)
    codes = np.zeros(v.size, dtype=np.int8)
    e = _load().orc_quant_i8(_p(v), v.size, _p(codes))
    return codes, int(e)


def pool_i8(raw_bits: np.ndarray, w, pool_size: int = POOL):
    """IndexPool into the INT8 cache: [n_tok, dim] raw bf16 keys ->
    (codes [n_tok // pool, dim] int8, scale [n_tok // pool] fp64)."""
    raw = np.ascontiguousarray(raw_bits, dtype=np.uint16)
    n_tok, dim = raw.shape
    w = np.ascontiguousarray(w, dtype=np.float64)
    assert w.shape == (pool_size,)
    nblk = n_tok // pool_size
    codes = np.zeros((nblk, dim), dtype=np.int8)
    scale = np.zeros(nblk, dtype=np.float64)
    _load().orc_pool_i8(_p(raw), n_tok, dim, pool_size, _p(w), _p(codes), _p(scale))
    return codes, scale


def score_i8(q_bits: np.ndarray, w_head, codes: np.ndarray, scale, nthreads: int = 0) -> np.ndarray:
    """Indexer scores [nblk] (fp64) of one query [heads, dim] against the INT8 cache."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    heads, dim = q.shape
    w = np.ascontiguousarray(w_head, dtype=np.float64)
    assert w.shape == (heads,)
    c = np.ascontiguousarray(codes, dtype=np.int8)
    sc = np.ascontiguousarray(scale, dtype=np.float64)
    nblk = c.shape[0] if c.size else 0
    assert nblk == 0 or (c.shape[1] == dim and sc.shape == (nblk,))
    out = np.zeros(nblk, dtype=np.float64)
    if nblk:
        _load().orc_score_i8(_p(q), _p(w), heads, dim, _p(c), _p(sc), nblk, _p(out), nthreads)
    return out


def e4m3_bits(v: float) -> int:
    """E4M3 bit pattern of the nearest-even E4M3 value of v (|v| <= 448)."""
    return int(_load().orc_e4m3_bits(float(v)))


def e4m3_value(bits) -> np.ndarray:
    """Values (fp64) of E4M3 bit patterns."""
    lib = _load()
    table = np.array([lib.orc_e4m3_value(b) for b in range(256)], dtype=np.float64)
    return table[np.asarray(bits, dtype=np.uint8)]


def quant_e4m3(x) -> tuple[np.ndarray, int]:
    """FP8 (E4M3) code of one vector: (uint8 codes, e) with x ~= 2^e * value(codes)."""
    v = np.ascontiguousarray(x, dtype=np.float64).reshape(-1)
    codes = np.zeros(v.size, dtype=np.uint8)
    e = _load().orc_quant_e4m3(_p(v), v.size, _p(codes))
    return codes, int(e)


def latent_fp8(rows_bits: np.ndarray):
    """FP8 latent cache of bf16 latent rows [S, D]: (codes [S, D] uint8, e [S])."""
    rows = bf16_to_f64(np.asarray(rows_bits, dtype=np.uint16)).reshape(-1, np.shape(rows_bits)[-1])
    out = [quant_e4m3(r) for r in rows]
    codes = np.stack([c for c, _ in out]) if out else np.zeros((0, rows.shape[1]), np.uint8)
    return codes, np.array([e for _, e in out], dtype=np.int64)


def dequant_fp8_bits(codes: np.ndarray, e) -> np.ndarray:
    """bf16 bits of the dequantised FP8 rows (exact: 4 significant bits times 2^k)."""
    vals = e4m3_value(codes) * np.ldexp(1.0, np.asarray(e))[:, None]
    bits = np.array([bf16_rne(v) for v in vals.reshape(-1)], dtype=np.uint16).reshape(vals.shape)
    assert np.array_equal(bf16_to_f64(bits), vals)
    return bits


def topk(scores, K: int = TOPK_BLOCKS) -> np.ndarray:
    """Selected block ids (int32, ascending) of the top min(K, n) scores."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    out = np.zeros(max(1, min(K, s.size)), dtype=np.int32)
    cnt = _load().orc_topk(_p(s), s.size, K, _p(out)) if s.size else 0
    return out[:cnt].copy()


def token_set(idx, n_vis: int, pool_size: int = POOL) -> np.ndarray:
    """Token positions a query attends to: selected blocks, then the tail."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.zeros(idx.size * pool_size + pool_size, dtype=np.int64)
    m = _load().orc_token_set(_p(idx), idx.size, n_vis, pool_size, _p(out))
    return out[:m].copy()


def attention(q_bits: np.ndarray, rows_bits: np.ndarray, sm_scale: float):
    """Softmax attention (fp64) of q [H, D] over latent rows [S, D] -> (out [H, D], lse [H])."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    H, D = q.shape
    rows = np.ascontiguousarray(rows_bits, dtype=np.uint16).reshape(-1, D)
    out = np.zeros((H, D), dtype=np.float64)
    lse = np.zeros(H, dtype=np.float64)
    _load().orc_attention(_p(q), H, D, _p(rows), rows.shape[0], float(sm_scale), _p(out), _p(lse))
    return out, lse


def select_query(q_idx_bits, w_head, pooled_bits, n_vis: int, K: int = TOPK_BLOCKS, nthreads: int = 0):
    """Steps 2-3 for one query that sees n_vis tokens: (scores, idx, positions)."""
    nblk = n_vis // POOL
    s = score(q_idx_bits, w_head, pooled_bits[:nblk], nthreads)
    idx = topk(s, K)
    return s, idx, token_set(idx, n_vis)


def attention_fp8(q_bits: np.ndarray, rows_bits: np.ndarray, sm_scale: float):
    """Attention over an FP8 latent cache: the rows are stored as E4M3 codes
    with one power-of-two scale each, and attended in their dequantised form."""
    codes, e = latent_fp8(rows_bits)
    return attention(q_bits, dequant_fp8_bits(codes, e), sm_scale)


def decode_query(q_idx_bits, w_head, pooled_bits, n_vis, q_bits, latent_rows_fn, sm_scale,
                 K: int = TOPK_BLOCKS, nthreads: int = 0):
    """Steps 2-4 for one decode query.

    ``latent_rows_fn(positions) -> [S, D] bf16 bits`` returns the latent rows
    of the given token positions (the caller's cache).
    Returns dict(scores, idx, positions, out, lse).
    """
    s, idx, pos = select_query(q_idx_bits, w_head, pooled_bits, n_vis, K, nthreads)
    rows = latent_rows_fn(pos)
    out, lse = attention(q_bits, rows, sm_scale)
    return dict(scores=s, idx=idx, positions=pos, out=out, lse=lse)
