"""fp64 CPU oracle of the hybrid compressed attention hot path (CSA + HCA).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this package.  It shares no code with the CUDA library: the arithmetic
lives in ``oracle/oracle.c`` (plain loops in double precision); this module only marshals numpy
arrays through ctypes and composes the per-stage routines in the order the method applies them.

Every stage cites its source passage in ``oracle.c``.  Parity status of each routine:

* compress, index_scores, topk, csa_attn, hca_attn, lse_merge: pinned by the invariant and
  special-case tests in ``tests/test_oracle_pins.py`` (window mean, weights summing to one,
  locality, identity at m=1, each indexer-key channel weighted by its own channel's softmax,
  brute-force selection, dense attention against a library softmax, partition invariance of the
  merge).
* e2m1_code, quantize_entries_mx4, dequantize_entries_mx4 (FP4 entries, R15): pinned by the E2M1
  grid (every value maps to itself, every midpoint to its even neighbour, saturation), the block
  scale's definition at its boundary, exact round trips of on-grid rows, and a brute-force nearest
  search on random rows.
* hybrid_query (the composition): pinned at q = 0, q^I = 0, where the merged softmax is uniform
  over exactly the keys the method attends (lse = log of their count, O = their mean), at lengths
  below and above the window and the HCA ratio.  Beyond that the pages print no worked numeric
  example of the composed method.
"""
from __future__ import annotations

import ctypes
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

from . import _build

_DIR = os.path.dirname(os.path.abspath(__file__))
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = os.path.join(_DIR, "liboracle.so")
        if not os.path.exists(path):
            _build.build()
        L = ctypes.CDLL(path)
        vp, i64, ci, cd = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.oracle_round_bf16.argtypes = [vp, i64, vp]
        L.oracle_bf16_to_double.argtypes = [vp, i64, vp]
        L.oracle_compress.argtypes = [vp, vp, vp, vp, i64, ci, ci, ci, ci, vp, i64, vp, vp]
        L.oracle_compress.restype = ci
        L.oracle_compress_weights.argtypes = [vp, vp, i64, ci, ci, ci, vp, i64, vp]
        L.oracle_compress_weights.restype = ci
        L.oracle_index_scores.argtypes = [vp, vp, ci, ci, vp, i64, vp]
        L.oracle_topk.argtypes = [vp, i64, ci, vp]
        L.oracle_topk.restype = ci
        L.oracle_csa_attn.argtypes = [vp, ci, ci, vp, vp, ci, ci, vp, i64, ci, cd, vp, vp]
        L.oracle_csa_attn.restype = ci
        L.oracle_hca_attn.argtypes = [vp, ci, ci, vp, ci, vp, i64, ci, cd, vp, vp]
        L.oracle_hca_attn.restype = ci
        L.oracle_lse_merge.argtypes = [vp, vp, vp, vp, ci, ci, vp, vp]
        L.oracle_rms_norm.argtypes = [vp, i64, ci, vp, cd, vp]
        L.oracle_e4m3_round.argtypes = [vp, i64, vp]
        L.oracle_e4m3_value.argtypes = [vp, i64, vp]
        L.oracle_quantize_keys_mx8.argtypes = [vp, i64, ci, vp, vp]
        L.oracle_quantize_keys_mx8.restype = ci
        L.oracle_index_scores_mx8.argtypes = [vp, vp, ci, ci, vp, vp, i64, vp]
        L.oracle_e2m1_round.argtypes = [vp, i64, vp]
        L.oracle_quantize_entries_mx4.argtypes = [vp, i64, ci, vp, vp]
        L.oracle_quantize_entries_mx4.restype = ci
        L.oracle_dequantize_entries_mx4.argtypes = [vp, vp, i64, ci, vp]
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest-even); returns the uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_round_bf16(_p(a), a.size, _p(out))
    return out


def bf16_to_f64(u: np.ndarray) -> np.ndarray:
    u = _u16(u)
    out = np.empty(u.shape, dtype=np.float64)
    lib().oracle_bf16_to_double(_p(u), u.size, _p(out))
    return out


def compress(x, logit, bias, kI, L: int, m: int, win: int, js, d_I: int = 0):
    """Compressor entries js of one sequence: (E [n,d] fp64, KI [n,d_I] fp64 or None).

    x, logit: uint16 [>=L, d]; bias: float32 [win, d]; kI: uint16 [>=L, d_I] or None.
    """
    x, logit = _u16(x), _u16(logit)
    bias = np.ascontiguousarray(bias, dtype=np.float32)
    js = np.ascontiguousarray(js, dtype=np.int64)
    d = x.shape[1]
    E = np.empty((len(js), d), dtype=np.float64)
    KI = None
    if kI is not None:
        kI = _u16(kI)
        d_I = kI.shape[1]
        KI = np.empty((len(js), d_I), dtype=np.float64)
    rc = lib().oracle_compress(_p(x), _p(logit), _p(bias), _p(kI), L, d, d_I, m, win, _p(js), len(js), _p(E), _p(KI))
    if rc != 0:
        raise ValueError(f"oracle_compress failed ({rc})")
    return E, KI


def compress_parallel(x, logit, bias, kI, L, m, win, js, threads: int = 0, chunk: int = 4096):
    """compress() split over a thread pool (ctypes releases the GIL); same results."""
    js = np.ascontiguousarray(js, dtype=np.int64)
    threads = threads or os.cpu_count() or 1
    parts = [js[i:i + chunk] for i in range(0, len(js), chunk)]
    if len(parts) <= 1 or threads == 1:
        return compress(x, logit, bias, kI, L, m, win, js)
    x, logit = _u16(x), _u16(logit)
    kI = None if kI is None else _u16(kI)
    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(lambda p: compress(x, logit, bias, kI, L, m, win, p), parts))
    E = np.concatenate([r[0] for r in res])
    KI = None if kI is None else np.concatenate([r[1] for r in res])
    return E, KI


def compress_weights(logit, bias, L, m, win, js):
    logit = _u16(logit)
    bias = np.ascontiguousarray(bias, dtype=np.float32)
    js = np.ascontiguousarray(js, dtype=np.int64)
    d = logit.shape[1]
    W = np.empty((len(js), win, d), dtype=np.float64)
    if lib().oracle_compress_weights(_p(logit), _p(bias), L, d, m, win, _p(js), len(js), _p(W)) != 0:
        raise ValueError("oracle_compress_weights failed")
    return W


def index_scores(qI, w, KI) -> np.ndarray:
    """s_j = sum_h w_h relu(qI_h . KI_j) for every row of KI (uint16 [n, d_I])."""
    qI, KI = _u16(qI), _u16(KI)
    w = np.ascontiguousarray(w, dtype=np.float32)
    H_I, d_I = qI.shape
    s = np.empty(KI.shape[0], dtype=np.float64)
    lib().oracle_index_scores(_p(qI), _p(w), H_I, d_I, _p(KI), KI.shape[0], _p(s))
    return s


def e4m3_round(v) -> np.ndarray:
    """Doubles with |v| <= 448 to the nearest FP8 E4M3 value (ties to even), as bit patterns."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_round(_p(v), v.size, _p(out))
    return out


def e4m3_value(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(b.shape, dtype=np.float64)
    lib().oracle_e4m3_value(_p(b), b.size, _p(out))
    return out


def quantize_keys_mx8(KI):
    """bf16 key rows [n, d_I] -> (E4M3 bytes [n, d_I], biased power-of-two scales [n, d_I / 32])."""
    KI = _u16(KI)
    n, d_I = KI.shape
    Kq = np.empty((n, d_I), dtype=np.uint8)
    sc = np.empty((n, d_I // 32), dtype=np.uint8)
    if lib().oracle_quantize_keys_mx8(_p(KI), n, d_I, _p(Kq), _p(sc)) != 0:
        raise ValueError("d_I must be a multiple of 32")
    return Kq, sc


def e2m1_code(v) -> np.ndarray:
    """fp64 values -> the 4-bit E2M1 code of the nearest value (ties to the even code, |v| > 6 -> 6)."""
    v = np.ascontiguousarray(v, dtype=np.float64).ravel()
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e2m1_round(_p(v), v.size, _p(out))
    return out


def quantize_entries_mx4(E):
    """bf16 entry rows [n, d] -> (packed E2M1 codes [n, d / 2], biased power-of-two scales [n, d / 32])."""
    E = _u16(E)
    n, d = E.shape
    Eq = np.empty((n, d // 2), dtype=np.uint8)
    sc = np.empty((n, d // 32), dtype=np.uint8)
    if lib().oracle_quantize_entries_mx4(_p(E), n, d, _p(Eq), _p(sc)) != 0:
        raise ValueError("d must be a multiple of 32")
    return Eq, sc


def dequantize_entries_mx4(Eq, scales) -> np.ndarray:
    """packed E2M1 codes [n, d / 2] + scales [n, d / 32] -> dequantized values [n, d] (fp64)."""
    Eq = np.ascontiguousarray(Eq, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    n, d = Eq.shape[0], Eq.shape[1] * 2
    out = np.empty((n, d), dtype=np.float64)
    lib().oracle_dequantize_entries_mx4(_p(Eq), _p(scales), n, d, _p(out))
    return out


def mx4_entries_as_bf16(E) -> np.ndarray:
    """The entry rows the attention sees when the cache holds them in FP4 (R15): quantized, then
    dequantized.  Every dequantized value (at most two significant bits times a power of two) is a
    bf16 value, so it is returned as bf16 bit patterns for the bf16 attention routines."""
    Eq, sc = quantize_entries_mx4(E)
    v = dequantize_entries_mx4(Eq, sc)
    b = round_bf16(v)
    assert np.array_equal(bf16_to_f64(b), v), "a dequantized FP4 value is not a bf16 value"
    return b


def index_scores_mx8(qI, w, Kq, scales) -> np.ndarray:
    """Indexer scores of the dequantized 8-bit keys (fp64)."""
    qI = _u16(qI)
    w = np.ascontiguousarray(w, dtype=np.float32)
    Kq = np.ascontiguousarray(Kq, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    H_I, d_I = qI.shape
    s = np.empty(Kq.shape[0], dtype=np.float64)
    lib().oracle_index_scores_mx8(_p(qI), _p(w), H_I, d_I, _p(Kq), _p(scales), Kq.shape[0], _p(s))
    return s


def topk(s, k: int) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float64)
    idx = np.empty(k, dtype=np.int32)
    if lib().oracle_topk(_p(s), len(s), k, _p(idx)) != 0:
        raise MemoryError("oracle_topk")
    return idx


def csa_attn(q, entries, idx, m, raw, L, W, scale):
    q, entries, raw = _u16(q), _u16(entries), _u16(raw)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    H, d = q.shape
    O = np.empty((H, d), dtype=np.float64)
    lse = np.empty(H, dtype=np.float64)
    rc = lib().oracle_csa_attn(_p(q), H, d, _p(entries), _p(idx), len(idx), m, _p(raw), L, W, scale, _p(O), _p(lse))
    if rc != 0:
        raise ValueError(f"oracle_csa_attn failed ({rc})")
    return O, lse


def hca_attn(q, hca, m_hca, raw, L, W, scale):
    q, hca, raw = _u16(q), _u16(hca), _u16(raw)
    H, d = q.shape
    O = np.empty((H, d), dtype=np.float64)
    lse = np.empty(H, dtype=np.float64)
    rc = lib().oracle_hca_attn(_p(q), H, d, _p(hca), m_hca, _p(raw), L, W, scale, _p(O), _p(lse))
    if rc != 0:
        raise ValueError(f"oracle_hca_attn failed ({rc})")
    return O, lse


def rms_norm(x, gain, eps: float) -> np.ndarray:
    """Rows of x (fp64 [rows, d]) RMS-normalized with gain [d] (fp64 out)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    gain = np.ascontiguousarray(gain, dtype=np.float32)
    rows, d = x.reshape(-1, x.shape[-1]).shape
    out = np.empty(x.shape, dtype=np.float64)
    lib().oracle_rms_norm(_p(x), rows, d, _p(gain), float(eps), _p(out))
    return out


def sink_merge(O, lse, sink):
    """The attention-sink logit z_h of every head as one more softmax term whose value is zero
    ("DeepSeek V4 comprimeix el context", "CSA: buscar primer i atendre despres", last paragraph):
    exactly an LSE merge with a partial of output 0 and log-sum-exp z."""
    z = np.ascontiguousarray(sink, dtype=np.float64)
    return lse_merge(O, lse, np.zeros_like(np.asarray(O, dtype=np.float64)), z)


def lse_merge(O1, lse1, O2, lse2):
    O1, O2 = np.ascontiguousarray(O1, np.float64), np.ascontiguousarray(O2, np.float64)
    lse1, lse2 = np.ascontiguousarray(lse1, np.float64), np.ascontiguousarray(lse2, np.float64)
    H, d = O1.shape
    O = np.empty((H, d), dtype=np.float64)
    lse = np.empty(H, dtype=np.float64)
    lib().oracle_lse_merge(_p(O1), _p(lse1), _p(O2), _p(lse2), H, d, _p(O), _p(lse))
    return O, lse


@dataclass(frozen=True)
class Shape:
    """Widths of one hybrid attention layer (names follow the pages' notation)."""
    d: int = 512        # shared KV latent width
    H: int = 64         # query heads (MQA over the latent)
    d_I: int = 64       # indexer key width
    H_I: int = 4        # indexer heads
    m: int = 4          # CSA compression ratio (window 2m, overlapping)
    m_hca: int = 128    # HCA compression ratio (window m', non-overlapping)
    k: int = 1024       # entries kept by the indexer
    W: int = 128        # raw sliding window

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


def hybrid_query(shape: Shape, L: int, q, qI, w, raw, entries, KI, hca, sink=None, q_gain=None, eps=1e-6,
                 keys_mx8=None, entries_mx4=False):
    """One query of the hybrid layer at visible length L, composed from the stages above.

    raw: uint16 [>=L, d] raw latents of the sequence; entries: uint16 [>=L//m, d] CSA cache;
    KI: uint16 [>=L//m, d_I] indexer-key cache; hca: uint16 [>=L//m', d] HCA cache.
    Optional: sink [H] attention-sink logits; q_gain [d]: the query heads are RMS-normalized with
    this gain (and rounded to bf16, the attention's operand type) before attending; keys_mx8 =
    (Kq, scales): the indexer scores these 8-bit keys instead of KI; entries_mx4: the CSA and HCA
    caches hold FP4 entries with block scales (R15), so the attention sees their dequantized values.
    Returns a dict with the selected indices, the two partials and the merged output.
    """
    if entries_mx4:
        entries = mx4_entries_as_bf16(entries[:L // shape.m]) if L // shape.m > 0 else entries
        hca = mx4_entries_as_bf16(hca[:L // shape.m_hca]) if L // shape.m_hca > 0 else hca
    n_c = L // shape.m
    if keys_mx8 is not None:
        s = index_scores_mx8(qI, w, keys_mx8[0][:n_c], keys_mx8[1][:n_c])
    else:
        s = index_scores(qI, w, KI[:n_c])
    idx = topk(s, shape.k)
    if q_gain is not None:
        q = round_bf16(rms_norm(bf16_to_f64(q), q_gain, eps))
    O_c, lse_c = csa_attn(q, entries, idx, shape.m, raw, L, shape.W, shape.scale)
    O_h, lse_h = hca_attn(q, hca, shape.m_hca, raw, L, 0, shape.scale)
    O, lse = lse_merge(O_c, lse_c, O_h, lse_h)
    if sink is not None:
        O, lse = sink_merge(O, lse, sink)
    return {"idx": idx, "scores": s, "O_csa": O_c, "lse_csa": lse_c, "O_hca": O_h, "lse_hca": lse_h,
            "O": O, "lse": lse}


def parallel_map(fn, items, threads: int = 0):
    threads = threads or os.cpu_count() or 1
    items = list(items)
    if threads == 1 or len(items) <= 1:
        return [fn(i) for i in items]
    with ThreadPoolExecutor(threads) as ex:
        return list(ex.map(fn, items))
