"""Seeded, counter-based synthetic inputs for the hybrid compressed-attention workloads.

The generator is defined in ``synth/synth.h`` (SplitMix64 in counter mode, Box-Muller with
series-evaluated log and cos, direct round-to-nearest-even to bfloat16).  It has a host build
(``libsynth.so``, used by the fp64 oracle's side of every test) and a device build
(``libsynth_cuda.so``, used to fill multi-gigabyte inputs in HBM); the two agree bit for bit.
This module holds none of the attention method's arithmetic: it only produces input bytes.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import _build

_DIR = os.path.dirname(os.path.abspath(__file__))

X, A, B, KI, Q, QI, W, BIAS_C, BIAS_H, LEN = range(10)

_host = None
_dev = None


def host_lib() -> ctypes.CDLL:
    global _host
    if _host is None:
        path = os.path.join(_DIR, "libsynth.so")
        if not os.path.exists(path):
            _build.build_host()
        lib = ctypes.CDLL(path)
        i64, u64, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p
        for name in ("synth_fill_bf16_normal", "synth_fill_f32_normal", "synth_fill_f32_uniform"):
            fn = getattr(lib, name)
            fn.argtypes = [u64, ctypes.c_int, i64, i64, i64, i64, i64, i64, ctypes.c_double, vp]
            fn.restype = ctypes.c_int
        lib.synth_lengths.argtypes = [u64, i64, i64, i64, vp]
        lib.synth_lengths.restype = ctypes.c_int
        lib.synth_raw_bits.argtypes = [u64, ctypes.c_int, i64, i64, i64, vp]
        lib.synth_raw_bits.restype = ctypes.c_int
        lib.synth_log_host.argtypes = [ctypes.c_double]
        lib.synth_log_host.restype = ctypes.c_double
        lib.synth_cos2pi_host.argtypes = [ctypes.c_double]
        lib.synth_cos2pi_host.restype = ctypes.c_double
        lib.synth_bf16_host.argtypes = [ctypes.c_double]
        lib.synth_bf16_host.restype = ctypes.c_uint16
        _host = lib
    return _host


def dev_lib() -> ctypes.CDLL:
    global _dev
    if _dev is None:
        path = os.path.join(_DIR, "libsynth_cuda.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        i64, u64, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p
        for name in ("synth_dev_fill_bf16_normal", "synth_dev_fill_f32_normal", "synth_dev_fill_f32_uniform"):
            fn = getattr(lib, name)
            fn.argtypes = [u64, ctypes.c_int, i64, i64, i64, i64, i64, i64, ctypes.c_double, vp, vp]
            fn.restype = ctypes.c_int
        _dev = lib
    return _dev


def _cols(ncols, c0, c1):
    return (0 if c0 is None else c0), (ncols if c1 is None else c1)


def bf16_normal(seed: int, tensor: int, seq: int, ncols: int, r0: int, r1: int, c0=None, c1=None,
                scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of scale*N(0,1) for rows [r0,r1) x cols [c0,c1) of a [*, ncols] tensor."""
    c0, c1 = _cols(ncols, c0, c1)
    out = np.empty((r1 - r0, c1 - c0), dtype=np.uint16)
    rc = host_lib().synth_fill_bf16_normal(seed, tensor, seq, ncols, r0, r1, c0, c1, scale,
                                           out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("synth_fill_bf16_normal: bad arguments")
    return out


def f32_normal(seed, tensor, seq, ncols, r0, r1, c0=None, c1=None, scale=1.0) -> np.ndarray:
    c0, c1 = _cols(ncols, c0, c1)
    out = np.empty((r1 - r0, c1 - c0), dtype=np.float32)
    rc = host_lib().synth_fill_f32_normal(seed, tensor, seq, ncols, r0, r1, c0, c1, scale,
                                          out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("synth_fill_f32_normal: bad arguments")
    return out


def f32_uniform(seed, tensor, seq, ncols, r0, r1, c0=None, c1=None, scale=1.0) -> np.ndarray:
    c0, c1 = _cols(ncols, c0, c1)
    out = np.empty((r1 - r0, c1 - c0), dtype=np.float32)
    rc = host_lib().synth_fill_f32_uniform(seed, tensor, seq, ncols, r0, r1, c0, c1, scale,
                                           out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise ValueError("synth_fill_f32_uniform: bad arguments")
    return out


def lengths(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    if host_lib().synth_lengths(seed, n, lo, hi, out.ctypes.data_as(ctypes.c_void_p)) != 0:
        raise ValueError("synth_lengths: bad arguments")
    return out


def raw_bits(seed, tensor, seq, i0, n) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    host_lib().synth_raw_bits(seed, tensor, seq, i0, n, out.ctypes.data_as(ctypes.c_void_p))
    return out


def dev_fill(kind: str, seed: int, tensor: int, seq: int, ncols: int, r0: int, r1: int, out_ptr: int,
             stream_ptr: int = 0, c0=None, c1=None, scale: float = 1.0) -> None:
    """Fill a device buffer (raw pointer) with the same values the host routines produce."""
    c0, c1 = _cols(ncols, c0, c1)
    fn = {"bf16_normal": dev_lib().synth_dev_fill_bf16_normal,
          "f32_normal": dev_lib().synth_dev_fill_f32_normal,
          "f32_uniform": dev_lib().synth_dev_fill_f32_uniform}[kind]
    rc = fn(seed, tensor, seq, ncols, r0, r1, c0, c1, scale, ctypes.c_void_p(out_ptr), ctypes.c_void_p(stream_ptr))
    if rc != 0:
        raise RuntimeError(f"synth device fill failed ({rc})")


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
