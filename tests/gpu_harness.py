"""Shared helpers of the GPU parity tests: device layers filled from the generator, the oracle's
view of the same sequences, and the comparison rules.

Comparison rules (the tolerances are the ones the parity bar states for bf16 inputs with fp32
accumulation):
* attention outputs: max |gpu - oracle| <= 1e-2 and ||gpu - oracle||_2 / ||oracle||_2 <= 5e-3;
* selected index sets, when both sides score the same bf16 keys: identical, except that where the
  oracle's k-th and (k+1)-th scores lie within 1e-5 relative of each other either choice is
  accepted (``sets_match``);
* selected index sets in the end-to-end pipeline, where each side builds its own bf16 caches (a
  GPU fp32 compressor and the fp64 oracle may round a stored element to neighbouring bf16 values):
  every entry in the symmetric difference must lie within the score change that one-ulp key
  differences can cause (``sets_explained``).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import compressed_sparse_kv_overlapped_b200 as csa
import oracle
import synth
from synth import device as sdev
from synth import workloads

ATOL = 1e-2
RTOL_L2 = 5e-3
TIE_REL = 1e-5


def dims_of(wd: workloads.Dims):
    return csa.make_dims(d=wd.d, H=wd.H, d_I=wd.d_I, H_I=wd.H_I, m=wd.m, m_hca=wd.m_hca, k=wd.k, W=wd.W)


def oshape(wd: workloads.Dims) -> oracle.Shape:
    return oracle.Shape(d=wd.d, H=wd.H, d_I=wd.d_I, H_I=wd.H_I, m=wd.m, m_hca=wd.m_hca, k=wd.k, W=wd.W)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def new_layer(wl: workloads.Workload, lens=None) -> csa.HybridLayer:
    layer = csa.HybridLayer(dims_of(wl.dims), [wl.capacity(b) for b in range(wl.B)])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths(list(wl.n0) if lens is None else lens)
    layer.compress()
    torch.cuda.synchronize()
    return layer


def query_table(pairs) -> torch.Tensor:
    """csa_query rows (seq, len) as an int64 [Q, 2] device tensor."""
    return torch.tensor([[s, n] for s, n in pairs], dtype=torch.int64, device="cuda")


def check_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    assert np.isfinite(gpu).all(), f"{what}: non-finite GPU values"
    mx = float(err.max()) if err.size else 0.0
    rl2 = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30))
    assert mx <= ATOL and rl2 <= RTOL_L2, f"{what}: max abs {mx:.3e}, rel L2 {rl2:.3e}"
    return mx, rl2


def sets_match(gpu_idx, oracle_idx, scores, k):
    """Selected sets when both sides scored the same keys (near-tie rule at the k-th score)."""
    g = set(int(v) for v in gpu_idx if v >= 0)
    o = set(int(v) for v in oracle_idx if v >= 0)
    if g == o:
        return True
    assert len(g) == len(o), (len(g), len(o))
    order = sorted(o, key=lambda j: (-scores[j], j))
    sk = scores[order[-1]]
    band = {j for j in range(len(scores)) if abs(scores[j] - sk) <= TIE_REL * max(abs(sk), 1e-30)}
    assert (o - band) <= g and g <= (o | band), (sorted(g - o)[:10], sorted(o - g)[:10])
    return True


def score_slack(qI, w, KI_rows):
    """Largest change of s_j = sum_h w_h relu(q_h . K_j) when every key element moves by one bf16 ulp
    (at most 2^-7 of its magnitude), plus fp32 accumulation slack."""
    q = synth.bf16_to_f64(qI)
    K = synth.bf16_to_f64(KI_rows)
    mag = np.abs(K) @ np.abs(q).T  # [n, H_I]
    return (mag * np.abs(w)[None, :]).sum(axis=1) * (2.0 ** -7) + 1e-5 * (np.abs(K @ q.T) * np.abs(w)).sum(axis=1)


def sets_explained(gpu_idx, oracle_idx, scores, slack):
    """End-to-end selection check: entries that differ must be within their own cache-rounding slack
    of the oracle's selection threshold."""
    g = set(int(v) for v in gpu_idx if v >= 0)
    o = set(int(v) for v in oracle_idx if v >= 0)
    assert len(g) == len(o)
    if g == o:
        return 0
    sk = min(scores[j] for j in o)
    worst = 0.0
    for j in g ^ o:
        gap = abs(scores[j] - sk)
        assert gap <= slack[j] + slack[min(o, key=lambda i: scores[i])] + 1e-9, (j, gap, slack[j])
        worst = max(worst, gap)
    return len(g ^ o)


class OracleSeq:
    """The oracle's view of one sequence of a workload: host inputs and oracle-built caches."""

    def __init__(self, wl: workloads.Workload, b: int, T: int, with_mass: bool = False):
        self.wl, self.b, self.T = wl, b, T
        d = wl.dims
        self.x = workloads.raw_tokens(wl, b, 0, T, "x")
        self.a = workloads.raw_tokens(wl, b, 0, T, "a")
        self.bl = workloads.raw_tokens(wl, b, 0, T, "b")
        self.kI = workloads.raw_tokens(wl, b, 0, T, "kI")
        self.bias_c = workloads.bias_c(wl)
        self.bias_h = workloads.bias_h(wl)
        n_c, n_h = T // d.m, T // d.m_hca
        E, KI = oracle.compress_parallel(self.x, self.a, self.bias_c, self.kI, T, d.m, 2 * d.m, np.arange(n_c))
        self.E = oracle.round_bf16(E)
        self.KI = oracle.round_bf16(KI)
        self.E64, self.KI64 = E, KI
        if with_mass:  # sum_t w_t |x_t|: the scale of the fp32 accumulation error of each element
            ax = oracle.round_bf16(np.abs(synth.bf16_to_f64(self.x)))
            akI = oracle.round_bf16(np.abs(synth.bf16_to_f64(self.kI)))
            self.E_mass, self.KI_mass = oracle.compress_parallel(ax, self.a, self.bias_c, akI, T, d.m, 2 * d.m,
                                                                 np.arange(n_c))
        if n_h:
            H, _ = oracle.compress_parallel(self.x, self.bl, self.bias_h, None, T, d.m_hca, d.m_hca, np.arange(n_h))
            self.H = oracle.round_bf16(H)
            self.H64 = H
            if with_mass:
                self.H_mass, _ = oracle.compress_parallel(ax, self.bl, self.bias_h, None, T, d.m_hca, d.m_hca,
                                                          np.arange(n_h))
        else:
            self.H = np.zeros((1, d.d), np.uint16)
            self.H64 = np.zeros((0, d.d))
            self.H_mass = np.zeros((0, d.d))

    def query(self, L, q, qI, w):
        return oracle.hybrid_query(oshape(self.wl.dims), L, q, qI, w, self.x, self.E, self.KI, self.H)


def ulp_compare(gpu_u16: np.ndarray, ref64: np.ndarray, abs_mass: np.ndarray | None = None):
    """Compare bf16 GPU values with fp64 reference values: returns (#elements off by more than one
    bf16 ulp of the reference plus the fp32 accumulation bound, #elements that differ from the
    reference's own rounding).

    abs_mass = sum_t w_t |x_t| per element (the oracle's compressor applied to |x|).  A weighted sum
    accumulated in fp32 carries an absolute error of a few fp32 ulps of that mass; where terms
    cancel, this exceeds one bf16 ulp of the (small) result.  2^-18 is 32 fp32 ulps."""
    g = synth.bf16_to_f64(gpu_u16)
    r_round = synth.bf16_to_f64(oracle.round_bf16(ref64))
    ulp = np.maximum(np.abs(r_round) * 2.0 ** -7, 2.0 ** -133)
    if abs_mass is not None:
        ulp = ulp + abs_mass * 2.0 ** -18
    far = int((np.abs(g - ref64) > ulp).sum())
    diff = int((gpu_u16 != oracle.round_bf16(ref64)).sum())
    return far, diff


def scale_of(wd) -> float:
    return 1.0 / math.sqrt(wd.d)


class OracleSeqLazy:
    """The oracle's view of one long sequence (e.g. 2^20 tokens) for sampled queries: indexer keys and
    HCA entries are built for the whole sequence, CSA entries only where a sampled query needs them."""

    def __init__(self, wl: workloads.Workload, b: int, T: int):
        self.wl, self.b, self.T = wl, b, T
        d = wl.dims
        self.x = workloads.raw_tokens(wl, b, 0, T, "x")
        self.a = workloads.raw_tokens(wl, b, 0, T, "a")
        kI = workloads.raw_tokens(wl, b, 0, T, "kI")
        self.bias_c = workloads.bias_c(wl)
        n_c, n_h = T // d.m, T // d.m_hca
        # indexer keys = the compressor on channels 0..d_I-1 with the raw indexer keys as values
        KI, _ = oracle.compress_parallel(kI, np.ascontiguousarray(self.a[:, :d.d_I]),
                                         np.ascontiguousarray(self.bias_c[:, :d.d_I]), None, T, d.m, 2 * d.m,
                                         np.arange(n_c))
        self.KI = oracle.round_bf16(KI)
        bl = workloads.raw_tokens(wl, b, 0, T, "b")
        H, _ = oracle.compress_parallel(self.x, bl, workloads.bias_h(wl), None, T, d.m_hca, d.m_hca, np.arange(n_h))
        self.H = oracle.round_bf16(H)
        self.E = np.zeros((max(n_c, 1), d.d), np.uint16)
        self.have = np.zeros(max(n_c, 1), bool)

    def query(self, L, q, qI, w):
        d = self.wl.dims
        n_c = L // d.m
        s = oracle.index_scores(qI, w, self.KI[:n_c])
        idx = oracle.topk(s, d.k)
        need = np.array([j for j in idx if j >= 0 and not self.have[j]], dtype=np.int64)
        if len(need):
            E, _ = oracle.compress_parallel(self.x, self.a, self.bias_c, None, self.T, d.m, 2 * d.m, need)
            self.E[need] = oracle.round_bf16(E)
            self.have[need] = True
        return oracle.hybrid_query(oshape(d), L, q, qI, w, self.x, self.E, self.KI, self.H)
