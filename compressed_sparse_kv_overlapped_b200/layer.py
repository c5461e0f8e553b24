"""Device-resident state of one hybrid attention layer: ragged, packed per-sequence caches.

Memory layout in HBM (row-major, every tensor 256-byte aligned by the allocator):

  raw tokens   x, logit_c, logit_h : [sum_b cap_b, d]   bf16   (sequence b at rows tok_off[b]..)
               idx_key             : [sum_b cap_b, d_I] bf16
  CSA cache    entries             : [sum_b cap_b // m, d]   bf16   (rows csa_off[b]..)
               entry_keys          : [sum_b cap_b // m, d_I] bf16
  HCA cache    hca_entries         : [sum_b cap_b // m', d]  bf16   (rows hca_off[b]..)
  optional     keys_q / key_scales  (key_format "mx8"): 8-bit indexer keys [*, d_I] + [*, d_I / 32]
               entries_q / entry_scales, hca_q / hca_scales (kv_format "fp4"): FP4 entries
               [*, d / 2] + [*, d / 32] beside the bf16 caches
  parameters   bias_c [2m, d], bias_h [m', d] fp32
  table        seqs                : [B, 4] int64 = (tok_off, csa_off, hca_off, len) = csa_seq

The caller fills the raw-token rows (and the parameters); ``compress`` builds the caches and
``decode`` runs one step through ``hybrid_attn_decode``.  Torch is used for allocation only.
"""
from __future__ import annotations

import ctypes

from . import (CSA_OP_DECODE, CSA_OP_PREFILL, csa_compress, csa_compress_all, csa_decode_args, csa_norms,
               csa_prefill_args, csa_quantize_entries, csa_quantize_keys, csa_workspace_size, hybrid_attn_decode,
               hybrid_attn_prefill)


class HybridLayer:
    """key_format "mx8" adds 8-bit block-scaled copies of the indexer keys (keys_q [*, d_I] E4M3,
    key_scales [*, d_I / 32]) that the decode's indexer scores instead of the bf16 keys.  kv_format
    "fp4" adds FP4 copies of the CSA and HCA entries (E2M1 codes [*, d / 2], scales [*, d / 32]) that
    the decode's attention reads instead of the bf16 entries."""

    def __init__(self, dims, capacity, device="cuda", key_format="bf16", kv_format="bf16"):
        import torch

        self.dims = dims
        self.B = len(capacity)
        self.capacity = [int(c) for c in capacity]
        d, dI, m, mh = dims.d, dims.d_I, dims.m, dims.m_hca
        tok, csa, hca = [], [], []
        t = c = h = 0
        for cap in self.capacity:
            tok.append(t)
            csa.append(c)
            hca.append(h)
            t += cap
            c += cap // m
            h += cap // mh
        self.tok_off, self.csa_off, self.hca_off = tok, csa, hca
        bf = torch.bfloat16
        self.x = torch.empty(max(t, 1), d, dtype=bf, device=device)
        self.logit_c = torch.empty(max(t, 1), d, dtype=bf, device=device)
        self.logit_h = torch.empty(max(t, 1), d, dtype=bf, device=device)
        self.idx_key = torch.empty(max(t, 1), dI, dtype=bf, device=device)
        self.entries = torch.zeros(max(c, 1), d, dtype=bf, device=device)
        self.entry_keys = torch.zeros(max(c, 1), dI, dtype=bf, device=device)
        self.hca_entries = torch.zeros(max(h, 1), d, dtype=bf, device=device)
        if key_format not in ("bf16", "mx8"):
            raise ValueError(f"key_format {key_format!r}")
        self.key_format = key_format
        self.keys_q = self.key_scales = None
        if key_format == "mx8":
            self.keys_q = torch.zeros(max(c, 1), dI, dtype=torch.uint8, device=device)
            self.key_scales = torch.zeros(max(c, 1), dI // 32, dtype=torch.uint8, device=device)
        if kv_format not in ("bf16", "fp4"):
            raise ValueError(f"kv_format {kv_format!r}")
        self.kv_format = kv_format
        self.entries_q = self.entry_scales = self.hca_q = self.hca_scales = None
        if kv_format == "fp4":
            u8 = torch.uint8
            self.entries_q = torch.zeros(max(c, 1), d // 2, dtype=u8, device=device)
            self.entry_scales = torch.zeros(max(c, 1), d // 32, dtype=u8, device=device)
            self.hca_q = torch.zeros(max(h, 1), d // 2, dtype=u8, device=device)
            self.hca_scales = torch.zeros(max(h, 1), d // 32, dtype=u8, device=device)
        self.bias_c = torch.zeros(2 * m, d, dtype=torch.float32, device=device)
        self.bias_h = torch.zeros(mh, d, dtype=torch.float32, device=device)
        self.seqs = torch.tensor([[tok[b], csa[b], hca[b], 0] for b in range(self.B)], dtype=torch.int64,
                                 device=device)
        self.lens = [0] * self.B
        self.device = device
        self.norms = None  # optional csa_norms (set_norms)

    # ---- normalization and sinks ----------------------------------------------------------------
    def set_norms(self, q_norm=None, entry_norm_c=None, entry_norm_h=None, sink=None, eps=1e-6) -> None:
        """Optional query / entry RMS-normalization gains ([d] fp32) and sink logits ([H] fp32), device
        tensors kept by the layer; every later compress, decode and prefill uses them."""
        from . import make_norms
        self._norm_tensors = (q_norm, entry_norm_c, entry_norm_h, sink)
        self.norms = make_norms(q_norm, entry_norm_c, entry_norm_h, sink, eps)

    # ---- lengths ------------------------------------------------------------------------------
    def set_lengths(self, lens) -> None:
        import torch
        assert len(lens) == self.B and all(0 <= n <= c for n, c in zip(lens, self.capacity))
        self.lens = [int(n) for n in lens]
        self.seqs[:, 3] = torch.tensor(self.lens, dtype=torch.int64, device=self.device)

    # ---- compressor full pass -----------------------------------------------------------------
    def compress(self, stream=None) -> None:
        """(Re)build every complete CSA and HCA entry of every sequence from the raw tokens (one pass
        over the raw rows for both caches, csa_compress_all)."""
        import torch
        rt = torch.tensor([[0, n] for n in self.lens], dtype=torch.int64, device=self.device)
        if max(self.lens) > 0:
            csa_compress_all(self.dims, self.seqs, rt, self.B, max(self.lens), self.x, self.logit_c, self.logit_h,
                             self.bias_c, self.bias_h, self.idx_key, self.entries, self.entry_keys,
                             self.hca_entries, stream, norms=self.norms)
        if self.keys_q is not None:
            self.quantize_keys(stream)
        if self.entries_q is not None:
            self.quantize_entries(stream)
        self._keep = rt  # the kernels read the range table asynchronously

    def quantize_entries(self, stream=None) -> None:
        """The FP4 copies of every complete CSA and HCA entry (kv_format "fp4")."""
        import torch
        d = self.dims
        ec = [n // d.m for n in self.lens]
        eh = [n // d.m_hca for n in self.lens]
        rc = torch.tensor([[0, n] for n in ec], dtype=torch.int64, device=self.device)
        rh = torch.tensor([[0, n] for n in eh], dtype=torch.int64, device=self.device)
        if max(ec) > 0:
            csa_quantize_entries(d, self.seqs, rc, self.B, max(ec), 0, self.entries, self.entries_q, self.entry_scales,
                                 stream)
        if max(eh) > 0:
            csa_quantize_entries(d, self.seqs, rh, self.B, max(eh), 1, self.hca_entries, self.hca_q, self.hca_scales,
                                 stream)
        self._keep_e = (rc, rh)

    def quantize_keys(self, stream=None) -> None:
        """The 8-bit copies of every complete entry's indexer key (key_format "mx8")."""
        import torch
        d = self.dims
        rq = torch.tensor([[0, n // d.m] for n in self.lens], dtype=torch.int64, device=self.device)
        if max(n // d.m for n in self.lens) > 0:
            csa_quantize_keys(d, self.seqs, rq, self.B, max(n // d.m for n in self.lens), self.entry_keys, self.keys_q,
                              self.key_scales, stream)
        self._keep_q = rq

    def compress_separately(self, stream=None) -> None:
        """The same caches through two csa_compress calls (CSA entries with their keys, then HCA)."""
        import torch
        d = self.dims
        rc = torch.tensor([[0, n // d.m] for n in self.lens], dtype=torch.int64, device=self.device)
        rh = torch.tensor([[0, n // d.m_hca] for n in self.lens], dtype=torch.int64, device=self.device)
        csa_compress(d, 0, self.seqs, rc, self.B, max(n // d.m for n in self.lens), self.x, self.logit_c,
                     self.bias_c, self.idx_key, self.entries, self.entry_keys, stream)
        if max(n // d.m_hca for n in self.lens) > 0:
            csa_compress(d, 1, self.seqs, rh, self.B, max(n // d.m_hca for n in self.lens), self.x, self.logit_h,
                         self.bias_h, None, self.hca_entries, None, stream)
        self._keep2 = (rc, rh)

    # ---- decode -------------------------------------------------------------------------------
    def decode_args(self, q, q_idx, w, out, append=True, lse=None, idx_out=None, max_len=None,
                    scale=None, new_rows=None, idx_in=None) -> csa_decode_args:
        """Arguments of one decode step.  With append, the new token's raw rows either are already in
        the caches at row tok_off + len (new_rows None) or come as new_rows [B, 3d + d_I] bf16
        (x | logit_c | logit_h | idx_key per sequence) and the call writes them there."""
        d = self.dims
        a = csa_decode_args()
        a.dims = d
        a.B = self.B
        a.append = 1 if append else 0
        a.max_len = int(max_len if max_len is not None else max(self.capacity))
        a.scale = float(scale if scale is not None else d.d ** -0.5)
        for name, t in (("seqs", self.seqs), ("x", self.x), ("logit_c", self.logit_c), ("logit_h", self.logit_h),
                        ("idx_key", self.idx_key), ("bias_c", self.bias_c), ("bias_h", self.bias_h),
                        ("entries", self.entries), ("entry_keys", self.entry_keys),
                        ("hca_entries", self.hca_entries), ("q", q), ("q_idx", q_idx), ("w", w), ("out", out),
                        ("lse", lse), ("idx_out", idx_out), ("new_rows", new_rows), ("keys_q", self.keys_q),
                        ("key_scales", self.key_scales), ("idx_in", idx_in), ("entries_q", self.entries_q),
                        ("entry_scales", self.entry_scales), ("hca_q", self.hca_q), ("hca_scales", self.hca_scales)):
            setattr(a, name, None if t is None else t.data_ptr())
        if self.norms is not None:
            a.norms = ctypes.pointer(self.norms)
        return a

    def decode_workspace(self, max_len=None):
        import torch
        a = csa_decode_args()
        a.dims = self.dims
        a.B = self.B
        a.max_len = int(max_len if max_len is not None else max(self.capacity))
        n = csa_workspace_size(CSA_OP_DECODE, a)
        return torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)

    def decode(self, args: csa_decode_args, ws, stream=None) -> None:
        hybrid_attn_decode(args, ws, stream)
        if args.append:
            self.lens = [n + 1 for n in self.lens]

    # ---- prefill (sequence 0) -----------------------------------------------------------------
    def prefill_args(self, q, q_idx, w, out, q_begin, q_end, compress=True, lse=None, idx_out=None,
                     scale=None, idx_in=None) -> csa_prefill_args:
        d = self.dims
        a = csa_prefill_args()
        a.dims = d
        a.compress = 1 if compress else 0
        a.len = int(self.lens[0])
        a.q_begin, a.q_end = int(q_begin), int(q_end)
        a.scale = float(scale if scale is not None else d.d ** -0.5)
        a.seq = self.seqs.data_ptr()
        for name, t in (("x", self.x), ("logit_c", self.logit_c), ("logit_h", self.logit_h),
                        ("idx_key", self.idx_key), ("bias_c", self.bias_c), ("bias_h", self.bias_h),
                        ("entries", self.entries), ("entry_keys", self.entry_keys),
                        ("hca_entries", self.hca_entries), ("q", q), ("q_idx", q_idx), ("w", w), ("out", out),
                        ("lse", lse), ("idx_out", idx_out), ("idx_in", idx_in)):
            setattr(a, name, None if t is None else t.data_ptr())
        if self.norms is not None:
            a.norms = ctypes.pointer(self.norms)
        return a

    def prefill_workspace(self, q_end):
        import torch
        a = csa_prefill_args()
        a.dims = self.dims
        a.q_end = int(q_end)
        n = csa_workspace_size(CSA_OP_PREFILL, a)
        return torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)

    def prefill(self, args: csa_prefill_args, ws, stream=None) -> None:
        hybrid_attn_prefill(args, ws, stream)
