"""Python binding of libspx, the B200 (sm_100a) sparse-attention layer.

A thin ctypes layer over the C ABI declared in ``include/spx.h``: every
function here has the C function's name and arguments, takes torch tensors
where the C call takes device pointers, passes ``tensor.data_ptr()`` and the
current CUDA stream, and raises ``SpxError`` on a non-zero status.  All
computation happens in the library's CUDA kernels; torch only provides device
memory and streams.  There is no fallback: if ``libspx.so`` is missing the
import fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspx.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libspx.so not found at {LIB_PATH}; build it with "
        "`python long_context_decode_indexpool_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

IDX_HEADS = 32
IDX_DIM = 128
POOL = 4
TOPK_BLOCKS = 512
LATENT = 512

STATUS = {0: "SPX_OK", 1: "SPX_ERR_INVALID_ARG", 2: "SPX_ERR_SHAPE", 3: "SPX_ERR_UNSUPPORTED",
          4: "SPX_ERR_WORKSPACE", 5: "SPX_ERR_CUDA", 6: "SPX_ERR_DEVICE"}


class SpxError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class spx_dims(ctypes.Structure):
    _fields_ = [("idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
                ("pool", ctypes.c_int32), ("topk_blocks", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("latent", ctypes.c_int32),
                ("sm_scale", ctypes.c_float)]


class spx_timing(ctypes.Structure):
    _fields_ = [("score_begin", ctypes.c_void_p), ("score_end", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_DIMS = ctypes.POINTER(spx_dims)

_SIGS = {
    "spx_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "spx_version": ([], ctypes.c_char_p),
    "spx_launch_count": ([], ctypes.c_uint64),
    "spx_dims_init": ([_DIMS, _I32, ctypes.c_float], ctypes.c_int),
    "spx_device_error": ([ctypes.POINTER(_I32), _P], ctypes.c_int),
    "spx_selftest_wait_timeout": ([_I64, _P, _P], ctypes.c_int),
    "spx_pool_append": ([_DIMS, _I32, _P, _I32, _P, _P, _P, _I64, _P, _I64, _P], ctypes.c_int),
    "spx_pool_append_tok": ([_DIMS, _I32, _P, _P, _I32, _P, _P, _P, _I64, _P, _I64, _P], ctypes.c_int),
    "spx_index_score": ([_DIMS, _I32, _P, _P, _P, _I64, _P, _I64, _P, _I64, _P], ctypes.c_int),
    "spx_topk_workspace_size": ([_DIMS, _I32, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
    "spx_topk_blocks": ([_DIMS, _I32, _P, _I64, _P, _I64, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "spx_topk_blocks_noalloc": ([_DIMS, _I32, _P, _I64, _P, _I64, _P, _P, _P], ctypes.c_int),
    "spx_attn_workspace_size": ([_DIMS, _I32, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
    "spx_sparse_mla_attn": ([_DIMS, _I32, _P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P, _SZ, _P],
                            ctypes.c_int),
    "spx_latent_quant_fp8": ([_P, _I64, _P, _P, _P], ctypes.c_int),
    "spx_attn_fp8_workspace_size": ([_DIMS, _I32, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
    "spx_sparse_mla_attn_fp8": ([_DIMS, _I32, _P, _P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P,
                                 _SZ, _P], ctypes.c_int),
    "spx_ws_workspace_size": ([_DIMS, _I32, _I32, ctypes.POINTER(_SZ)], ctypes.c_int),
    "spx_sparse_mla_attn_ws": ([_DIMS, _I32, _P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _I32, _P, _P,
                                _P, _P, _I32, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "spx_decode_workspace_size": ([_DIMS, _I32, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
    "spx_decode_fused": ([_DIMS, _I32, _P, _P, _P, _P, _I64, _P, _P, _P, _P, _P, _I64, _I64, _P,
                          _P, _P, _P, _P, _SZ, ctypes.POINTER(spx_timing), _P], ctypes.c_int),
    "spx_pool_append_i8": ([_DIMS, _I32, _P, _I32, _P, _P, _P, _P, _I64, _P, _I64, _P],
                           ctypes.c_int),
    "spx_index_score_i8_workspace_size": ([_DIMS, _I32, ctypes.POINTER(_SZ)], ctypes.c_int),
    "spx_index_score_i8": ([_DIMS, _I32, _P, _P, _P, _P, _I64, _P, _I64, _P, _I64, _P, _SZ, _P],
                           ctypes.c_int),
    "spx_decode_fused_i8": ([_DIMS, _I32, _P, _P, _P, _P, _P, _I64, _P, _P, _P, _P, _P, _I64, _I64,
                             _P, _P, _P, _P, _P, _SZ, ctypes.POINTER(spx_timing), _P],
                            ctypes.c_int),
    "spx_prefill_workspace_size": ([_DIMS, _I32, _I64, ctypes.POINTER(_SZ)], ctypes.c_int),
    "spx_prefill_chunk": ([_DIMS, _I32, _P, _P, _P, _P, _I64, _I64, _P, _P, _P, _P, _I64, _P, _P,
                           _P, _P, _P, _SZ, ctypes.POINTER(spx_timing), _P], ctypes.c_int),
    "spx_prefill_chunk_i8": ([_DIMS, _I32, _P, _P, _P, _P, _P, _I64, _I64, _P, _P, _P, _P, _I64,
                              _P, _P, _P, _P, _P, _SZ, ctypes.POINTER(spx_timing), _P],
                             ctypes.c_int),
}

for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res

EXPORTED = tuple(_SIGS)


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != 0:
        raise SpxError(st, where)


def dims(heads: int, sm_scale: float = 1.0) -> spx_dims:
    d = spx_dims()
    _check(_lib.spx_dims_init(ctypes.byref(d), heads, sm_scale), "spx_dims_init")
    return d


def status_string(status: int) -> str:
    return _lib.spx_status_string(status).decode()


def version() -> str:
    return _lib.spx_version().decode()


def _host_f32(arr):
    if isinstance(arr, ctypes.Array):
        return arr
    return (ctypes.c_float * 4)(*[float(x) for x in arr])


def pool_weights(w):
    """The 4 pooling weights as the host array the calls take (convert once, reuse)."""
    return _host_f32(w)


def _event_handle(ev):
    """cudaEvent_t of a torch.cuda.Event (torch creates it on first record)."""
    if ev is None:
        return None
    if not ev.cuda_event:
        ev.record()
    return ev.cuda_event


def _timing(events):
    if events is None:
        return None
    t = spx_timing()
    t.score_begin = _event_handle(events[0])
    t.score_end = _event_handle(events[1])
    return ctypes.byref(t)


# ---------------------------------------------------------------------------
# the C ABI, one function each
# ---------------------------------------------------------------------------
def spx_launch_count() -> int:
    return int(_lib.spx_launch_count())


def spx_device_error(stream=None) -> int:
    code = _I32(0)
    _check(_lib.spx_device_error(ctypes.byref(code), _stream(stream)), "spx_device_error")
    return code.value


def spx_selftest_wait_timeout(limit_ns, result, stream=None):
    """Launches the bounded-wait self-test kernel; result: int64 [6] on the device."""
    _check(_lib.spx_selftest_wait_timeout(int(limit_ns), _ptr(result), _stream(stream)),
           "spx_selftest_wait_timeout")


def spx_pool_append(d, B, raw_k, n_new, pool_w, tail, pooled_k, cap_blk, len_dev, max_len,
                    stream=None):
    _check(_lib.spx_pool_append(ctypes.byref(d), B, _ptr(raw_k), n_new, _host_f32(pool_w),
                                _ptr(tail), _ptr(pooled_k), cap_blk, _ptr(len_dev), max_len,
                                _stream(stream)), "spx_pool_append")


def spx_pool_append_tok(d, B, raw_k, raw_w, n_new, tail, tail_w, pooled_k, cap_blk, len_dev,
                        max_len, stream=None):
    _check(_lib.spx_pool_append_tok(ctypes.byref(d), B, _ptr(raw_k), _ptr(raw_w), n_new, _ptr(tail),
                                    _ptr(tail_w), _ptr(pooled_k), cap_blk, _ptr(len_dev), max_len,
                                    _stream(stream)), "spx_pool_append_tok")


def spx_index_score(d, B, q_idx, w_head, pooled_k, cap_blk, n_vis, max_len, scores, score_stride,
                    stream=None):
    _check(_lib.spx_index_score(ctypes.byref(d), B, _ptr(q_idx), _ptr(w_head), _ptr(pooled_k),
                                cap_blk, _ptr(n_vis), max_len, _ptr(scores), score_stride,
                                _stream(stream)), "spx_index_score")


def spx_topk_workspace_size(d, rows, max_len) -> int:
    n = _SZ(0)
    _check(_lib.spx_topk_workspace_size(ctypes.byref(d), rows, max_len, ctypes.byref(n)),
           "spx_topk_workspace_size")
    return n.value


def spx_topk_blocks(d, rows, scores, score_stride, n_vis, max_len, idx, count, ws, ws_bytes=None,
                    stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.spx_topk_blocks(ctypes.byref(d), rows, _ptr(scores), score_stride, _ptr(n_vis),
                                max_len, _ptr(idx), _ptr(count), _ptr(ws), ws_bytes,
                                _stream(stream)), "spx_topk_blocks")


def spx_topk_blocks_noalloc(d, rows, scores, score_stride, n_vis, max_len, idx, count,
                            stream=None):
    """spx_topk_blocks without a caller workspace: the library's built-in
    scratch array is used (see include/spx.h for its size and rules)."""
    _check(_lib.spx_topk_blocks_noalloc(ctypes.byref(d), rows, _ptr(scores), score_stride,
                                        _ptr(n_vis), max_len, _ptr(idx), _ptr(count),
                                        _stream(stream)), "spx_topk_blocks_noalloc")


NOALLOC_SCRATCH_BYTES = 4 << 20


def spx_attn_workspace_size(d, rows, max_len) -> int:
    n = _SZ(0)
    _check(_lib.spx_attn_workspace_size(ctypes.byref(d), rows, max_len, ctypes.byref(n)),
           "spx_attn_workspace_size")
    return n.value


def spx_sparse_mla_attn(d, rows, q, latent, seq_stride, cap_tok, idx, count, n_vis, max_len, out,
                        lse=None, ws=None, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.spx_sparse_mla_attn(ctypes.byref(d), rows, _ptr(q), _ptr(latent), seq_stride,
                                    cap_tok, _ptr(idx), _ptr(count), _ptr(n_vis), max_len,
                                    _ptr(out), _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
           "spx_sparse_mla_attn")


def spx_latent_quant_fp8(latent, n, codes, exps, stream=None):
    _check(_lib.spx_latent_quant_fp8(_ptr(latent), n, _ptr(codes), _ptr(exps), _stream(stream)),
           "spx_latent_quant_fp8")


def spx_attn_fp8_workspace_size(d, rows, max_len) -> int:
    n = _SZ(0)
    _check(_lib.spx_attn_fp8_workspace_size(ctypes.byref(d), rows, max_len, ctypes.byref(n)),
           "spx_attn_fp8_workspace_size")
    return n.value


def spx_sparse_mla_attn_fp8(d, rows, q, codes, exps, seq_stride, cap_tok, idx, count, n_vis,
                            max_len, out, lse=None, ws=None, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.spx_sparse_mla_attn_fp8(ctypes.byref(d), rows, _ptr(q), _ptr(codes), _ptr(exps),
                                        seq_stride, cap_tok, _ptr(idx), _ptr(count), _ptr(n_vis),
                                        max_len, _ptr(out), _ptr(lse), _ptr(ws), ws_bytes,
                                        _stream(stream)), "spx_sparse_mla_attn_fp8")


def spx_ws_workspace_size(d, rows, nslots) -> int:
    n = _SZ(0)
    _check(_lib.spx_ws_workspace_size(ctypes.byref(d), rows, nslots, ctypes.byref(n)),
           "spx_ws_workspace_size")
    return n.value


def spx_sparse_mla_attn_ws(d, rows, q, host_latent, seq_stride, cap_tok, idx, count, n_vis,
                           max_len, pool, nslots, slot_blk, blk_slot, slot_stamp, hand, step,
                           stats, out, lse=None, ws=None, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.spx_sparse_mla_attn_ws(ctypes.byref(d), rows, _ptr(q), _ptr(host_latent),
                                       seq_stride, cap_tok, _ptr(idx), _ptr(count), _ptr(n_vis),
                                       max_len, _ptr(pool), nslots, _ptr(slot_blk),
                                       _ptr(blk_slot), _ptr(slot_stamp), _ptr(hand), step,
                                       _ptr(stats), _ptr(out), _ptr(lse), _ptr(ws), ws_bytes,
                                       _stream(stream)), "spx_sparse_mla_attn_ws")


def spx_decode_workspace_size(d, B, max_len) -> int:
    n = _SZ(0)
    _check(_lib.spx_decode_workspace_size(ctypes.byref(d), B, max_len, ctypes.byref(n)),
           "spx_decode_workspace_size")
    return n.value


def spx_decode_fused(d, B, raw_k, pool_w, tail, pooled_k, cap_blk, len_dev, q_idx, w_head, q,
                     latent, cap_tok, max_len, out, lse=None, idx_out=None, count_out=None,
                     ws=None, ws_bytes=None, timing=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    pw = _host_f32(pool_w) if pool_w is not None else None
    _check(_lib.spx_decode_fused(ctypes.byref(d), B, _ptr(raw_k), pw, _ptr(tail), _ptr(pooled_k),
                                 cap_blk, _ptr(len_dev), _ptr(q_idx), _ptr(w_head), _ptr(q),
                                 _ptr(latent), cap_tok, max_len, _ptr(out), _ptr(lse),
                                 _ptr(idx_out), _ptr(count_out), _ptr(ws), ws_bytes,
                                 _timing(timing), _stream(stream)), "spx_decode_fused")


def spx_pool_append_i8(d, B, raw_k, n_new, pool_w, tail, pooled_k8, k_scale, cap_blk, len_dev,
                       max_len, stream=None):
    _check(_lib.spx_pool_append_i8(ctypes.byref(d), B, _ptr(raw_k), n_new, _host_f32(pool_w),
                                   _ptr(tail), _ptr(pooled_k8), _ptr(k_scale), cap_blk,
                                   _ptr(len_dev), max_len, _stream(stream)), "spx_pool_append_i8")


def spx_index_score_i8_workspace_size(d, B) -> int:
    n = _SZ(0)
    _check(_lib.spx_index_score_i8_workspace_size(ctypes.byref(d), B, ctypes.byref(n)),
           "spx_index_score_i8_workspace_size")
    return n.value


def spx_index_score_i8(d, B, q_idx, w_head, pooled_k8, k_scale, cap_blk, n_vis, max_len, scores,
                       score_stride, ws, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.spx_index_score_i8(ctypes.byref(d), B, _ptr(q_idx), _ptr(w_head), _ptr(pooled_k8),
                                   _ptr(k_scale), cap_blk, _ptr(n_vis), max_len, _ptr(scores),
                                   score_stride, _ptr(ws), ws_bytes, _stream(stream)),
           "spx_index_score_i8")


def spx_decode_fused_i8(d, B, raw_k, pool_w, tail, pooled_k8, k_scale, cap_blk, len_dev, q_idx,
                        w_head, q, latent, cap_tok, max_len, out, lse=None, idx_out=None,
                        count_out=None, ws=None, ws_bytes=None, timing=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    pw = _host_f32(pool_w) if pool_w is not None else None
    _check(_lib.spx_decode_fused_i8(ctypes.byref(d), B, _ptr(raw_k), pw, _ptr(tail),
                                    _ptr(pooled_k8), _ptr(k_scale), cap_blk, _ptr(len_dev),
                                    _ptr(q_idx), _ptr(w_head), _ptr(q), _ptr(latent), cap_tok,
                                    max_len, _ptr(out), _ptr(lse), _ptr(idx_out),
                                    _ptr(count_out), _ptr(ws), ws_bytes, _timing(timing),
                                    _stream(stream)), "spx_decode_fused_i8")


def spx_prefill_workspace_size(d, T, pos0) -> int:
    n = _SZ(0)
    _check(_lib.spx_prefill_workspace_size(ctypes.byref(d), T, pos0, ctypes.byref(n)),
           "spx_prefill_workspace_size")
    return n.value


def spx_prefill_chunk(d, T, raw_k, pool_w, tail, pooled_k, cap_blk, pos0, q_idx, w_head, q,
                      latent, cap_tok, out, lse=None, idx_out=None, count_out=None, ws=None,
                      ws_bytes=None, timing=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.spx_prefill_chunk(ctypes.byref(d), T, _ptr(raw_k), _host_f32(pool_w), _ptr(tail),
                                  _ptr(pooled_k), cap_blk, pos0, _ptr(q_idx), _ptr(w_head),
                                  _ptr(q), _ptr(latent), cap_tok, _ptr(out), _ptr(lse),
                                  _ptr(idx_out), _ptr(count_out), _ptr(ws), ws_bytes,
                                  _timing(timing), _stream(stream)), "spx_prefill_chunk")


def spx_prefill_chunk_i8(d, T, raw_k, pool_w, tail, pooled_k8, k_scale, cap_blk, pos0, q_idx,
                         w_head, q, latent, cap_tok, out, lse=None, idx_out=None, count_out=None,
                         ws=None, ws_bytes=None, timing=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(_lib.spx_prefill_chunk_i8(ctypes.byref(d), T, _ptr(raw_k), _host_f32(pool_w),
                                     _ptr(tail), _ptr(pooled_k8), _ptr(k_scale), cap_blk, pos0,
                                     _ptr(q_idx), _ptr(w_head), _ptr(q), _ptr(latent), cap_tok,
                                     _ptr(out), _ptr(lse), _ptr(idx_out), _ptr(count_out),
                                     _ptr(ws), ws_bytes, _timing(timing), _stream(stream)),
           "spx_prefill_chunk_i8")


def workspace(nbytes: int, device) -> torch.Tensor:
    """A caller-owned scratch buffer of at least nbytes (256-byte aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
