"""Python binding of libcsa: hybrid compressed attention (CSA + HCA) on B200 (sm_100a).

Argument marshalling only.  Every step of the hot path runs in the CUDA kernels of ``libcsa.so``
through its C ABI (``include/csa.h``); there is no CPU or PyTorch fallback -- if the library is
missing or fails to load, every call raises.  Tensors are torch CUDA tensors (passed by data
pointer); bf16 data may be ``torch.bfloat16`` or ``torch.int16``/``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os

from . import _build

_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_DIR, "libcsa.so")

CSA_OK = 0
CSA_ERR_ARG = -1
CSA_ERR_UNSUPPORTED = -2
CSA_ERR_CUDA = -3
CSA_ERR_TIMEOUT = -4
CSA_ERR_INDEX = -5

CSA_OP_INDEX_TOPK = 1
CSA_OP_SPARSE_ATTN = 2
CSA_OP_HCA_ATTN = 3
CSA_OP_DECODE = 4
CSA_OP_PREFILL = 5

EXPORTS = ("csa_compress", "csa_compress_all", "csa_index_topk", "csa_sparse_attn", "hca_dense_attn", "hybrid_attn_decode",
           "hybrid_attn_prefill", "csa_workspace_size", "csa_last_error", "csa_sync_status", "csa_version",
           "csa_set_stage_events", "csa_index_topk_noalloc", "csa_debug_inject", "csa_quantize_keys",
           "csa_index_topk_mx8", "csa_quantize_entries", "csa_sparse_attn_fp4", "hca_dense_attn_fp4")
CSA_DECODE_MARKS = 5

_i32, _i64, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class csa_dims(ctypes.Structure):
    _fields_ = [("d", _i32), ("H", _i32), ("d_I", _i32), ("H_I", _i32), ("m", _i32), ("m_hca", _i32),
                ("k", _i32), ("W", _i32)]


class csa_ws_query(ctypes.Structure):
    _fields_ = [("dims", csa_dims), ("Q", _i32), ("reserved", _i32), ("max_len", _i64)]


class csa_norms(ctypes.Structure):
    _fields_ = [("q_norm", _vp), ("entry_norm_c", _vp), ("entry_norm_h", _vp), ("sink", _vp), ("eps", _f32),
                ("reserved", _i32)]


class csa_decode_args(ctypes.Structure):
    _fields_ = [("dims", csa_dims), ("B", _i32), ("append", _i32), ("max_len", _i64), ("scale", _f32),
                ("seqs", _vp), ("x", _vp), ("logit_c", _vp), ("logit_h", _vp), ("idx_key", _vp),
                ("bias_c", _vp), ("bias_h", _vp), ("entries", _vp), ("entry_keys", _vp), ("hca_entries", _vp),
                ("q", _vp), ("q_idx", _vp), ("w", _vp), ("out", _vp), ("lse", _vp), ("idx_out", _vp),
                ("new_rows", _vp), ("keys_q", _vp), ("key_scales", _vp), ("idx_in", _vp),
                ("norms", ctypes.POINTER(csa_norms)), ("entries_q", _vp), ("entry_scales", _vp), ("hca_q", _vp),
                ("hca_scales", _vp)]


class csa_prefill_args(ctypes.Structure):
    _fields_ = [("dims", csa_dims), ("compress", _i32), ("reserved", _i32), ("len", _i64), ("q_begin", _i64),
                ("q_end", _i64), ("scale", _f32), ("seq", _vp), ("x", _vp), ("logit_c", _vp), ("logit_h", _vp),
                ("idx_key", _vp), ("bias_c", _vp), ("bias_h", _vp), ("entries", _vp), ("entry_keys", _vp),
                ("hca_entries", _vp), ("q", _vp), ("q_idx", _vp), ("w", _vp), ("out", _vp), ("lse", _vp),
                ("idx_out", _vp), ("idx_in", _vp), ("norms", ctypes.POINTER(csa_norms))]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libcsa.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        L.csa_compress.argtypes = [P(csa_dims), ctypes.c_int, _vp, _vp, ctypes.c_int, _i64, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _vp]
        L.csa_compress_all.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _vp, _vp, P(csa_norms), _vp]
        L.csa_index_topk.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                     _vp]
        L.csa_sparse_attn.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _vp,
                                      _sz, _vp]
        L.hca_dense_attn.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _i64, _vp, _vp, _vp, ctypes.c_int, _f32,
                                     _vp, _vp, _vp, _sz, _vp]
        L.hybrid_attn_decode.argtypes = [P(csa_decode_args), _vp, _sz, _vp]
        L.hybrid_attn_prefill.argtypes = [P(csa_prefill_args), _vp, _sz, _vp]
        L.csa_workspace_size.argtypes = [ctypes.c_int, _vp]
        L.csa_workspace_size.restype = _sz
        L.csa_last_error.restype = ctypes.c_char_p
        L.csa_sync_status.argtypes = [_vp]
        L.csa_set_stage_events.argtypes = [_vp, ctypes.c_int]
        L.csa_debug_inject.argtypes = [ctypes.c_int, _i64]
        L.csa_quantize_keys.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _i64, _vp, _vp, _vp, _vp]
        L.csa_index_topk_mx8.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                         _vp, _sz, _vp]
        L.csa_index_topk_noalloc.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _i64, _vp, _vp, _vp, _vp, _vp, _vp]
        L.csa_quantize_entries.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _i64, ctypes.c_int, _vp, _vp, _vp,
                                           _vp]
        L.csa_sparse_attn_fp4.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _f32, _vp,
                                          _vp, _vp, _sz, _vp]
        L.hca_dense_attn_fp4.argtypes = [P(csa_dims), _vp, _vp, ctypes.c_int, _i64, _vp, _vp, _vp, _vp, ctypes.c_int,
                                         _f32, _vp, _vp, _vp, _sz, _vp]
        for n in ("csa_compress", "csa_compress_all", "csa_index_topk", "csa_sparse_attn", "hca_dense_attn", "hybrid_attn_decode",
                  "hybrid_attn_prefill", "csa_sync_status", "csa_version", "csa_set_stage_events",
                  "csa_index_topk_noalloc", "csa_debug_inject", "csa_quantize_keys", "csa_index_topk_mx8",
                  "csa_quantize_entries", "csa_sparse_attn_fp4", "hca_dense_attn_fp4"):
            getattr(L, n).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, name: str) -> None:
    if rc != CSA_OK:
        msg = lib().csa_last_error().decode()
        raise RuntimeError(f"{name} failed ({rc}): {msg}")


def make_dims(d=512, H=64, d_I=64, H_I=4, m=4, m_hca=128, k=1024, W=128) -> csa_dims:
    return csa_dims(d, H, d_I, H_I, m, m_hca, k, W)


def csa_version() -> int:
    return lib().csa_version()


def csa_last_error() -> str:
    return lib().csa_last_error().decode()


def csa_sync_status(stream=None) -> int:
    return lib().csa_sync_status(_vp(_stream(stream)))


def csa_set_stage_events(events) -> None:
    """events: list of torch.cuda.Event (a multiple of CSA_DECODE_MARKS), or None to turn off."""
    global _stage_array
    if not events:
        _stage_array = None
        _check(lib().csa_set_stage_events(None, 0), "csa_set_stage_events")
        return
    handles = [e.cuda_event for e in events]
    _stage_array = (_vp * len(handles))(*handles)
    _check(lib().csa_set_stage_events(_stage_array, len(handles)), "csa_set_stage_events")


_stage_array = None


def csa_workspace_size(op: int, args) -> int:
    return int(lib().csa_workspace_size(op, ctypes.byref(args)))


def csa_compress(dims, which, seqs, ranges, B, max_entries, x, logit, bias, idx_key, entries, entry_keys,
                 stream=None) -> None:
    rc = lib().csa_compress(ctypes.byref(dims), which, _ptr(seqs), _ptr(ranges), B, max_entries, _ptr(x),
                            _ptr(logit), _ptr(bias), _ptr(idx_key), _ptr(entries), _ptr(entry_keys),
                            _vp(_stream(stream)))
    _check(rc, "csa_compress")


def csa_debug_inject(fault: int, wait_limit_ns: int = 0) -> None:
    """Fault injection for the bounded-wait tests (see csa.h); csa_debug_inject(0) turns it off."""
    _check(lib().csa_debug_inject(fault, wait_limit_ns), "csa_debug_inject")


def make_norms(q_norm=None, entry_norm_c=None, entry_norm_h=None, sink=None, eps=1e-6) -> csa_norms:
    """csa_norms from device tensors (or None for the parts that are off)."""
    n = csa_norms()
    n.q_norm, n.entry_norm_c, n.entry_norm_h, n.sink = (_ptr(q_norm), _ptr(entry_norm_c), _ptr(entry_norm_h),
                                                        _ptr(sink))
    n.eps = float(eps)
    n.reserved = 0
    return n


def csa_compress_all(dims, seqs, tok_ranges, B, max_tokens, x, logit_c, logit_h, bias_c, bias_h, idx_key, entries,
                     entry_keys, hca_entries, stream=None, norms=None) -> None:
    rc = lib().csa_compress_all(ctypes.byref(dims), _ptr(seqs), _ptr(tok_ranges), B, max_tokens, _ptr(x),
                                _ptr(logit_c), _ptr(logit_h), _ptr(bias_c), _ptr(bias_h), _ptr(idx_key),
                                _ptr(entries), _ptr(entry_keys), _ptr(hca_entries),
                                None if norms is None else ctypes.byref(norms), _vp(_stream(stream)))
    _check(rc, "csa_compress_all")


def csa_index_topk(dims, seqs, queries, Q, max_len, q_idx, w, entry_keys, idx_out, score_out, ws, stream=None):
    rc = lib().csa_index_topk(ctypes.byref(dims), _ptr(seqs), _ptr(queries), Q, max_len, _ptr(q_idx), _ptr(w),
                              _ptr(entry_keys), _ptr(idx_out), _ptr(score_out), _ptr(ws),
                              0 if ws is None else ws.numel() * ws.element_size(), _vp(_stream(stream)))
    _check(rc, "csa_index_topk")


def csa_index_topk_noalloc(dims, seqs, queries, Q, max_len, q_idx, w, entry_keys, idx_out, score_out,
                           stream=None):
    """csa_index_topk with the library's built-in scratch instead of a workspace (see csa.h)."""
    rc = lib().csa_index_topk_noalloc(ctypes.byref(dims), _ptr(seqs), _ptr(queries), Q, max_len, _ptr(q_idx),
                                      _ptr(w), _ptr(entry_keys), _ptr(idx_out), _ptr(score_out),
                                      _vp(_stream(stream)))
    _check(rc, "csa_index_topk_noalloc")


def csa_quantize_keys(dims, seqs, ranges, B, max_entries, entry_keys, keys_q, key_scales, stream=None) -> None:
    rc = lib().csa_quantize_keys(ctypes.byref(dims), _ptr(seqs), _ptr(ranges), B, max_entries, _ptr(entry_keys),
                                 _ptr(keys_q), _ptr(key_scales), _vp(_stream(stream)))
    _check(rc, "csa_quantize_keys")


def csa_index_topk_mx8(dims, seqs, queries, Q, max_len, q_idx, w, keys_q, key_scales, idx_out, score_out, ws,
                       stream=None):
    rc = lib().csa_index_topk_mx8(ctypes.byref(dims), _ptr(seqs), _ptr(queries), Q, max_len, _ptr(q_idx), _ptr(w),
                                  _ptr(keys_q), _ptr(key_scales), _ptr(idx_out), _ptr(score_out), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(), _vp(_stream(stream)))
    _check(rc, "csa_index_topk_mx8")


def csa_sparse_attn(dims, seqs, queries, Q, q, entries, idx, x, scale, out, lse, ws, stream=None):
    rc = lib().csa_sparse_attn(ctypes.byref(dims), _ptr(seqs), _ptr(queries), Q, _ptr(q), _ptr(entries), _ptr(idx),
                               _ptr(x), scale, _ptr(out), _ptr(lse), _ptr(ws),
                               0 if ws is None else ws.numel() * ws.element_size(), _vp(_stream(stream)))
    _check(rc, "csa_sparse_attn")


def hca_dense_attn(dims, seqs, queries, Q, max_len, q, hca_entries, x, W, scale, out, lse, ws, stream=None):
    rc = lib().hca_dense_attn(ctypes.byref(dims), _ptr(seqs), _ptr(queries), Q, max_len, _ptr(q),
                              _ptr(hca_entries), _ptr(x), W, scale, _ptr(out), _ptr(lse), _ptr(ws),
                              0 if ws is None else ws.numel() * ws.element_size(), _vp(_stream(stream)))
    _check(rc, "hca_dense_attn")


def csa_quantize_entries(dims, seqs, ranges, B, max_entries, which, entries, entries_q, entry_scales,
                         stream=None) -> None:
    """FP4 copies of the stored bf16 entries of the CSA cache (which = 0) or the HCA cache (which = 1)."""
    rc = lib().csa_quantize_entries(ctypes.byref(dims), _ptr(seqs), _ptr(ranges), B, max_entries, which,
                                    _ptr(entries), _ptr(entries_q), _ptr(entry_scales), _vp(_stream(stream)))
    _check(rc, "csa_quantize_entries")


def csa_sparse_attn_fp4(dims, seqs, queries, Q, q, entries_q, entry_scales, idx, x, scale, out, lse, ws, stream=None):
    rc = lib().csa_sparse_attn_fp4(ctypes.byref(dims), _ptr(seqs), _ptr(queries), Q, _ptr(q), _ptr(entries_q),
                                   _ptr(entry_scales), _ptr(idx), _ptr(x), scale, _ptr(out), _ptr(lse), _ptr(ws),
                                   0 if ws is None else ws.numel() * ws.element_size(), _vp(_stream(stream)))
    _check(rc, "csa_sparse_attn_fp4")


def hca_dense_attn_fp4(dims, seqs, queries, Q, max_len, q, hca_q, hca_scales, x, W, scale, out, lse, ws,
                       stream=None):
    rc = lib().hca_dense_attn_fp4(ctypes.byref(dims), _ptr(seqs), _ptr(queries), Q, max_len, _ptr(q), _ptr(hca_q),
                                  _ptr(hca_scales), _ptr(x), W, scale, _ptr(out), _ptr(lse), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(), _vp(_stream(stream)))
    _check(rc, "hca_dense_attn_fp4")


def hybrid_attn_decode(args: csa_decode_args, ws, stream=None) -> None:
    rc = lib().hybrid_attn_decode(ctypes.byref(args), _ptr(ws), ws.numel() * ws.element_size(),
                                  _vp(_stream(stream)))
    _check(rc, "hybrid_attn_decode")


def hybrid_attn_prefill(args: csa_prefill_args, ws, stream=None) -> None:
    rc = lib().hybrid_attn_prefill(ctypes.byref(args), _ptr(ws), ws.numel() * ws.element_size(),
                                   _vp(_stream(stream)))
    _check(rc, "hybrid_attn_prefill")


def build() -> str:
    return _build.build()


from .layer import HybridLayer  # noqa: E402  (torch-side cache allocation; imports torch lazily)
