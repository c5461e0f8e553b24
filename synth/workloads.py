"""The synthetic workloads: shapes, lengths, seeds and the per-tensor input recipe.

Every input is drawn from the counter-based generator (``synth.h``) at a coordinate
(seed, tensor, sequence, flat index), so the oracle's harness and the CUDA harness obtain the same
bytes, and any sub-block can be regenerated on its own.  Recipe (all N(0,1) draws rounded to bf16
unless stated):

* raw latent x_t [d], CSA logits a_t [d], HCA logits b_t [d], raw indexer key k^I_t [d_I]:
  tensor X / A / B / KI, sequence b, flat index t*width + c;
* CSA bias [2m, d] and HCA bias [m', d]: fp32 N(0, 0.5^2), sequence 0 (shared by all sequences);
* decode query of sequence b at step s: q [H, d], q^I [H_I, d_I] (bf16 N(0,1)), w [H_I]
  (fp32 U(0,1)), tensor Q / QI / W, sequence b, row s;
* prefill query at position i: the same tensors, sequence 0, row i;
* ragged lengths: uniform integers on [32768, 131072] (tensor LEN).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import A, B, BIAS_C, BIAS_H, KI, Q, QI, W, X, bf16_normal, f32_normal, f32_uniform, lengths


@dataclass(frozen=True)
class Dims:
    d: int = 512
    H: int = 64
    d_I: int = 64
    H_I: int = 4
    m: int = 4
    m_hca: int = 128
    k: int = 1024
    W: int = 128

    @property
    def win(self) -> int:
        return 2 * self.m


TINY_DIMS = Dims(d=128, H=8, d_I=32, H_I=4, m=4, m_hca=16, k=32, W=16)
PROD_DIMS = Dims()


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dims: Dims
    n0: tuple            # initial raw tokens per sequence (decode) / sequence length (prefill)
    steps: int           # decode steps (one appended token + one query per sequence each)
    mode: str = "decode"
    note: str = ""

    @property
    def B(self) -> int:
        return len(self.n0)

    def capacity(self, b: int) -> int:
        return self.n0[b] + (self.steps if self.mode == "decode" else 0)


def tiny() -> Workload:
    return Workload("tiny_decode_N1024", 1000, TINY_DIMS, (1023,), 1,
                    note="B=1, L=1024 at the query (1023 cached + 1 appended), d=128, H=8, k=32, W=16, m'=16")


def long_decode() -> Workload:
    return Workload("long_decode_N65536", 1001, PROD_DIMS, (65536,), 256,
                    note="B=1, N0=65536, 256 decode steps")


def ragged_decode() -> Workload:
    ls = lengths(1002, 32, 32768, 131072)
    return Workload("ragged_decode_B32", 1002, PROD_DIMS, tuple(int(v) for v in ls), 64,
                    note="B=32, lengths U[32768,131072], 64 decode steps")


def ctx1m_decode() -> Workload:
    return Workload("ctx1m_decode_B4_N1048576", 1003, PROD_DIMS, (1 << 20,) * 4, 128,
                    note="B=4, N0=2^20, 128 decode steps")


def prefill() -> Workload:
    return Workload("prefill_N131072", 1004, PROD_DIMS, (131072,), 0, mode="prefill",
                    note="B=1, N=131072 causal queries")


ALL = {"tiny": tiny, "long": long_decode, "ragged": ragged_decode, "ctx1m": ctx1m_decode, "prefill": prefill}


# ---- host generation (numpy, uint16 bf16 bit patterns / float32) -------------------------------

def raw_tokens(wl: Workload, b: int, t0: int, t1: int, which: str) -> np.ndarray:
    d = wl.dims
    tensor, width = {"x": (X, d.d), "a": (A, d.d), "b": (B, d.d), "kI": (KI, d.d_I)}[which]
    return bf16_normal(wl.seed, tensor, b, width, t0, t1)


def raw_tokens_cols(wl: Workload, b: int, t0: int, t1: int, which: str, c0: int, c1: int) -> np.ndarray:
    d = wl.dims
    tensor, width = {"x": (X, d.d), "a": (A, d.d), "b": (B, d.d), "kI": (KI, d.d_I)}[which]
    return bf16_normal(wl.seed, tensor, b, width, t0, t1, c0, c1)


def bias_c(wl: Workload) -> np.ndarray:
    return f32_normal(wl.seed, BIAS_C, 0, wl.dims.d, 0, wl.dims.win, scale=0.5)


def bias_h(wl: Workload) -> np.ndarray:
    return f32_normal(wl.seed, BIAS_H, 0, wl.dims.d, 0, wl.dims.m_hca, scale=0.5)


def queries(wl: Workload, b: int, r0: int, r1: int):
    """(q [n,H,d] u16, qI [n,H_I,d_I] u16, w [n,H_I] f32) for rows [r0, r1) of sequence b."""
    d = wl.dims
    q = bf16_normal(wl.seed, Q, b, d.H * d.d, r0, r1).reshape(r1 - r0, d.H, d.d)
    qi = bf16_normal(wl.seed, QI, b, d.H_I * d.d_I, r0, r1).reshape(r1 - r0, d.H_I, d.d_I)
    w = f32_uniform(wl.seed, W, b, d.H_I, r0, r1)
    return q, qi, w


def query_len(wl: Workload, b: int, row: int) -> int:
    """Visible length L of query `row`: decode step s sees n0+s+1 tokens; prefill position i sees i+1."""
    return wl.n0[b] + row + 1 if wl.mode == "decode" else row + 1
