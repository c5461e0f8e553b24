"""Fill device tensors with a workload's synthetic inputs (same bytes as the host generator).

Works on any object that carries the raw-token tensors of a hybrid layer (``x``, ``logit_c``,
``logit_h``, ``idx_key``, ``bias_c``, ``bias_h``) and the per-sequence ``tok_off``/``capacity``
lists; holds none of the attention method's arithmetic.
"""
from __future__ import annotations

from . import A, B, BIAS_C, BIAS_H, KI, Q, QI, W, X, dev_fill


def fill_layer_inputs(layer, wl, stream_ptr: int = 0) -> None:
    d = wl.dims
    for b in range(layer.B):
        cap = layer.capacity[b]
        t0 = layer.tok_off[b]
        for t, tensor, width in ((layer.x, X, d.d), (layer.logit_c, A, d.d), (layer.logit_h, B, d.d),
                                 (layer.idx_key, KI, d.d_I)):
            ptr = t.data_ptr() + t0 * width * t.element_size()
            dev_fill("bf16_normal", wl.seed, tensor, b, width, 0, cap, ptr, stream_ptr)
    dev_fill("f32_normal", wl.seed, BIAS_C, 0, d.d, 0, 2 * d.m, layer.bias_c.data_ptr(), stream_ptr, scale=0.5)
    dev_fill("f32_normal", wl.seed, BIAS_H, 0, d.d, 0, d.m_hca, layer.bias_h.data_ptr(), stream_ptr, scale=0.5)


def fill_queries(wl, b: int, r0: int, r1: int, q, q_idx, w, stream_ptr: int = 0) -> None:
    """Rows [r0, r1) of sequence b's query tensors into q [n,H,d], q_idx [n,H_I,d_I], w [n,H_I]."""
    d = wl.dims
    for t in (q, q_idx, w):  # the fill writes rows back to back from data_ptr()
        if not t.is_contiguous():
            raise ValueError("fill_queries needs contiguous tensors")
    dev_fill("bf16_normal", wl.seed, Q, b, d.H * d.d, r0, r1, q.data_ptr(), stream_ptr)
    dev_fill("bf16_normal", wl.seed, QI, b, d.H_I * d.d_I, r0, r1, q_idx.data_ptr(), stream_ptr)
    dev_fill("f32_uniform", wl.seed, W, b, d.H_I, r0, r1, w.data_ptr(), stream_ptr)
