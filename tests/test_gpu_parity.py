"""GPU parity: every stage of the CUDA path, called through the C ABI, against the fp64 oracle on
the same seeded inputs.  Stage tests feed both sides identical input bytes (the oracle's caches);
end-to-end tests let each side build its own caches from the raw tokens."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import compressed_sparse_kv_overlapped_b200 as csa
import oracle
import synth
from synth import device as sdev
from synth import workloads
from tests import gpu_harness as gh

pytestmark = pytest.mark.gpu

SMALL_PROD = workloads.Dims()  # production widths, used with short sequences


def wl_small(n0, steps=3, B=1, seed=2001, dims=SMALL_PROD, mode="decode"):
    return workloads.Workload(f"small_{n0}", seed, dims, tuple(n0) if isinstance(n0, (list, tuple)) else (n0,) * B,
                              steps, mode=mode)


# --------------------------------------------------------------------------------- generator

def test_device_generator_matches_host():
    for tensor, ncols, r0, r1 in [(synth.X, 512, 5, 300), (synth.KI, 64, 0, 1000), (synth.Q, 64 * 512, 2, 4),
                                  (synth.QI, 4 * 64, 0, 37)]:
        host = synth.bf16_normal(1234, tensor, 2, ncols, r0, r1)
        dev = torch.empty(r1 - r0, ncols, dtype=torch.int16, device="cuda")
        synth.dev_fill("bf16_normal", 1234, tensor, 2, ncols, r0, r1, dev.data_ptr())
        np.testing.assert_array_equal(dev.cpu().numpy().view(np.uint16), host)
    host = synth.f32_normal(9, synth.BIAS_C, 0, 512, 0, 8, scale=0.5)
    dev = torch.empty(8, 512, dtype=torch.float32, device="cuda")
    synth.dev_fill("f32_normal", 9, synth.BIAS_C, 0, 512, 0, 8, dev.data_ptr(), scale=0.5)
    np.testing.assert_array_equal(dev.cpu().numpy(), host)
    host = synth.f32_uniform(9, synth.W, 3, 4, 0, 100)
    dev = torch.empty(100, 4, dtype=torch.float32, device="cuda")
    synth.dev_fill("f32_uniform", 9, synth.W, 3, 4, 0, 100, dev.data_ptr())
    np.testing.assert_array_equal(dev.cpu().numpy(), host)


# --------------------------------------------------------------------------------- a1/a2

@pytest.mark.parametrize("wl", [workloads.tiny(), wl_small(5003), wl_small([700, 2600, 130], B=3)],
                         ids=["tiny", "prod5003", "ragged3"])
def test_compressor_within_one_ulp(wl):
    layer = gh.new_layer(wl)
    d = wl.dims
    for b in range(wl.B):
        n = wl.n0[b]
        ref = gh.OracleSeq(wl, b, n, with_mass=True)
        n_c, n_h = n // d.m, n // d.m_hca
        E = gh.u16(layer.entries[layer.csa_off[b]:layer.csa_off[b] + n_c])
        K = gh.u16(layer.entry_keys[layer.csa_off[b]:layer.csa_off[b] + n_c])
        checks = [(E, ref.E64, ref.E_mass, "entries"), (K, ref.KI64, ref.KI_mass, "entry_keys")]
        if n_h:
            Hh = gh.u16(layer.hca_entries[layer.hca_off[b]:layer.hca_off[b] + n_h])
            checks.append((Hh, ref.H64, ref.H_mass, "hca_entries"))
        for got, want, mass, name in checks:
            far, diff = gh.ulp_compare(got, want, mass)
            print(f"seq {b} {name}: {diff} of {want.size} elements rounded differently, {far} beyond bound")
            assert far == 0, f"{name}: {far} elements beyond one bf16 ulp + fp32 accumulation bound"
            assert diff <= max(2, 2e-3 * want.size), f"{name}: {diff} of {want.size} rounded differently"


def test_incremental_append_equals_full_pass():
    """Decode appends (compressor called per completed 4- and 128-token block) leave the caches
    bit-identical to one full compressor pass over the same tokens."""
    wl = wl_small([1000, 515], steps=260, B=2)
    layer = gh.new_layer(wl)
    d = wl.dims
    q = torch.empty(wl.B, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(wl.B, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(wl.B, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(wl.B, d.H, d.d, dtype=torch.float32, device="cuda")
    ws = layer.decode_workspace()
    for s in range(wl.steps):
        for b in range(wl.B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
        layer.decode(layer.decode_args(q, qi, w, out), ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    full = gh.new_layer(wl, lens=[n + wl.steps for n in wl.n0])
    for name in ("entries", "entry_keys", "hca_entries"):
        assert torch.equal(getattr(layer, name).view(torch.int16), getattr(full, name).view(torch.int16)), name
    assert layer.seqs[:, 3].tolist() == [n + wl.steps for n in wl.n0]


# Ratios on both sides of the block form (CSA m = 4, HCA m' a power of two from 4 to 128) and of the
# per-entry serial form used otherwise.
_SHAPES = {
    "m4_h128": workloads.Dims(d=512, H=64, d_I=64, H_I=4, m=4, m_hca=128, k=64, W=16),
    "m4_h8_d128": workloads.Dims(d=128, H=8, d_I=32, H_I=4, m=4, m_hca=8, k=32, W=16),
    "m4_h64_d128": workloads.Dims(d=128, H=8, d_I=64, H_I=4, m=4, m_hca=64, k=32, W=16),
    "m4_h256": workloads.Dims(d=128, H=8, d_I=32, H_I=4, m=4, m_hca=256, k=32, W=16),
    "m2_h32": workloads.Dims(d=128, H=8, d_I=32, H_I=4, m=2, m_hca=32, k=32, W=16),
    "m8_h100": workloads.Dims(d=128, H=8, d_I=32, H_I=4, m=8, m_hca=100, k=32, W=16),
}


@pytest.mark.parametrize("shape", list(_SHAPES))
def test_compressor_shapes_within_one_ulp(shape):
    """Both caches through csa_compress_all at every ratio form, ragged lengths that end inside a
    128-token tile, against the fp64 oracle; the two csa_compress calls give the same bytes."""
    wl = wl_small([1000, 333, 4], B=3, dims=_SHAPES[shape], seed=2100)
    layer = gh.new_layer(wl)
    d = wl.dims
    for b in range(wl.B):
        n = wl.n0[b]
        ref = gh.OracleSeq(wl, b, n, with_mass=True)
        n_c, n_h = n // d.m, n // d.m_hca
        checks = [(gh.u16(layer.entries[layer.csa_off[b]:layer.csa_off[b] + n_c]), ref.E64, ref.E_mass, "entries"),
                  (gh.u16(layer.entry_keys[layer.csa_off[b]:layer.csa_off[b] + n_c]), ref.KI64, ref.KI_mass, "keys")]
        if n_h:
            checks.append((gh.u16(layer.hca_entries[layer.hca_off[b]:layer.hca_off[b] + n_h]), ref.H64, ref.H_mass,
                           "hca_entries"))
        for got, want, mass, name in checks:
            far, diff = gh.ulp_compare(got, want, mass)
            assert far == 0, f"seq {b} {name}: {far} elements beyond one bf16 ulp + fp32 accumulation bound"
            assert diff <= max(2, 2e-3 * want.size), f"seq {b} {name}: {diff} of {want.size} rounded differently"
    sep = csa.HybridLayer(gh.dims_of(d), [wl.capacity(b) for b in range(wl.B)])
    sdev.fill_layer_inputs(sep, wl)
    sep.set_lengths(list(wl.n0))
    sep.compress_separately()
    torch.cuda.synchronize()
    assert csa.csa_sync_status() == csa.CSA_OK
    for name in ("entries", "entry_keys", "hca_entries"):
        assert torch.equal(getattr(layer, name).view(torch.int16), getattr(sep, name).view(torch.int16)), name


@pytest.mark.parametrize("which", [0, 1])
def test_compress_partial_ranges(which):
    """csa_compress over per-sequence entry ranges that start and end inside 128-token tiles writes
    exactly those entries, equal to the full pass, and nothing else."""
    wl = wl_small([3000, 700], B=2, dims=_SHAPES["m4_h8_d128"], seed=2200)
    d = wl.dims
    full = gh.new_layer(wl)
    part = csa.HybridLayer(gh.dims_of(d), [wl.capacity(b) for b in range(wl.B)])
    sdev.fill_layer_inputs(part, wl)
    part.set_lengths(list(wl.n0))
    m = d.m if which == 0 else d.m_hca
    ranges = [(37, 300), (0, 700 // m)] if which == 0 else [(3, 301), (1, 700 // m)]
    rt = torch.tensor(ranges, dtype=torch.int64, device="cuda")
    if which == 0:
        csa.csa_compress(gh.dims_of(d), 0, part.seqs, rt, 2, max(e - s for s, e in ranges), part.x, part.logit_c,
                         part.bias_c, part.idx_key, part.entries, part.entry_keys)
        tensors = [("entries", part.csa_off), ("entry_keys", part.csa_off)]
    else:
        csa.csa_compress(gh.dims_of(d), 1, part.seqs, rt, 2, max(e - s for s, e in ranges), part.x, part.logit_h,
                         part.bias_h, None, part.hca_entries, None)
        tensors = [("hca_entries", part.hca_off)]
    torch.cuda.synchronize()
    assert csa.csa_sync_status() == csa.CSA_OK
    for name, offs in tensors:
        P, F = getattr(part, name).view(torch.int16).cpu(), getattr(full, name).view(torch.int16).cpu()
        written = torch.zeros(P.shape[0], dtype=torch.bool)
        for b, (e0, e1) in enumerate(ranges):
            written[offs[b] + e0:offs[b] + e1] = True
        assert torch.equal(P[written], F[written]), name
        assert (P[~written] == 0).all(), f"{name}: rows outside the ranges were written"


@pytest.mark.parametrize("shape", ["m4_h8_d128", "m4_h64_d128", "m4_h256", "m2_h32"])
def test_incremental_append_equals_full_pass_shapes(shape):
    """The decode append at every ratio form leaves the caches bit-identical to one full pass."""
    d = _SHAPES[shape]
    wl = wl_small([2 * d.m_hca - 5, 37], steps=d.m_hca + 12, B=2, dims=d, seed=2300)
    layer = gh.new_layer(wl)
    q = torch.empty(wl.B, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(wl.B, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(wl.B, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(wl.B, d.H, d.d, dtype=torch.float32, device="cuda")
    ws = layer.decode_workspace()
    for s in range(wl.steps):
        for b in range(wl.B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
        layer.decode(layer.decode_args(q, qi, w, out), ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    full = gh.new_layer(wl, lens=[n + wl.steps for n in wl.n0])
    for name in ("entries", "entry_keys", "hca_entries"):
        assert torch.equal(getattr(layer, name).view(torch.int16), getattr(full, name).view(torch.int16)), name


# --------------------------------------------------------------------------------- a3/a4 (stage)

def _index_case(E_list, k, d_I=64, H_I=4, seed=3001, quantize=False, zero_w=False):
    dims = csa.make_dims(d=512, H=64, d_I=d_I, H_I=H_I, m=4, m_hca=128, k=k, W=128)
    Q = len(E_list)
    KIs = []
    for qi_, E in enumerate(E_list):
        K = synth.bf16_normal(seed, synth.KI, qi_, d_I, 0, max(E, 1))
        if quantize:  # few distinct key values -> many exactly equal scores
            K = oracle.round_bf16(np.round(synth.bf16_to_f64(K) * 2) / 2)
        KIs.append(K)
    offs = np.cumsum([0] + [max(E, 1) for E in E_list])
    keys = gh.to_dev_bf16(np.concatenate(KIs))
    seqs = torch.tensor([[0, offs[i], 0, 4 * E + 3] for i, E in enumerate(E_list)], dtype=torch.int64,
                        device="cuda")
    qt = gh.query_table([(i, 4 * E + 3) for i, E in enumerate(E_list)])
    qI = synth.bf16_normal(seed, synth.QI, 99, H_I * d_I, 0, Q).reshape(Q, H_I, d_I)
    w = synth.f32_uniform(seed, synth.W, 99, H_I, 0, Q)
    if zero_w:
        w[:] = 0
    idx = torch.full((Q, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.empty(Q, k, dtype=torch.float32, device="cuda")
    max_len = 4 * max(E_list) + 3
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, Q, max_len
    ws = torch.empty(csa.csa_workspace_size(csa.CSA_OP_INDEX_TOPK, wq), dtype=torch.uint8, device="cuda")
    csa.csa_index_topk(dims, seqs, qt, Q, max_len, gh.to_dev_bf16(qI), torch.from_numpy(w).cuda(), keys, idx, sc, ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    idx_h, sc_h = idx.cpu().numpy(), sc.cpu().numpy()
    for i, E in enumerate(E_list):
        s = oracle.index_scores(qI[i], w[i], KIs[i][:E])
        ref = oracle.topk(s, k)
        gh.sets_match(idx_h[i], ref, s, k)
        valid = idx_h[i][idx_h[i] >= 0]
        assert (np.diff(valid) > 0).all(), "indices not ascending"
        assert (idx_h[i][len(valid):] == -1).all() and len(valid) == min(E, k)
        np.testing.assert_allclose(sc_h[i][:len(valid)], s[valid], rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("E_list,k,d_I", [([5000], 1024, 64), ([300], 32, 32), ([1024], 1024, 64),
                                          ([600], 1024, 64), ([1025, 70000, 4097, 1], 1024, 64),
                                          ([262144], 1024, 64), ([40000, 33000], 2048, 64)],
                         ids=["E5000", "tiny", "E=k", "E<k", "ragged4", "E262144", "k2048"])
def test_index_topk_stage(E_list, k, d_I):
    _index_case(E_list, k, d_I)


def test_index_topk_ties_and_zero_scores():
    _index_case([20000, 3000], 1024, quantize=True)   # heavy exact ties: lower index wins
    _index_case([5000], 1024, zero_w=True)             # every score 0: indices 0..k-1


def _ordered_keys(E, pattern, d_I=64):
    """Keys whose score under q^I = (256, 1, 0, ...) on head 0 is an exact integer rank r_j < 65536:
    key_j = (r_j // 256, r_j % 256, 0, ...), every value exact in bf16 and every sum exact in fp32."""
    j = np.arange(E)
    if pattern == "increasing":
        r = j
    elif pattern == "decreasing":
        r = E - 1 - j
    elif pattern == "blocks":  # the best ranks sit in a few runs of 1,500 entries far apart
        run = j // 1500
        r = np.where(run % 17 == 3, 50000 + (run // 17) * 1500 + j % 1500, j // 7)
    else:
        raise ValueError(pattern)
    K = np.zeros((E, d_I), np.float64)
    K[:, 0] = r // 256
    K[:, 1] = r % 256
    return oracle.round_bf16(K)


@pytest.mark.parametrize("pattern", ["increasing", "decreasing", "blocks"])
def test_index_topk_concentrated_top_entries(pattern):
    """The top-k concentrated in a few scan chunks (far more than a chunk's share of them): those
    chunks' candidates do not cover their members of the threshold bin, so the select re-filters
    them from the stored scores.  The result must still be the exact top-k."""
    E, k, d_I, H_I = 60000, 1024, 64, 4
    dims = csa.make_dims(d=512, H=64, d_I=d_I, H_I=H_I, m=4, m_hca=128, k=k, W=128)
    K = _ordered_keys(E, pattern)
    qI = np.zeros((1, H_I, d_I), np.float64)
    qI[0, 0, 0], qI[0, 0, 1] = 256.0, 1.0
    qI = oracle.round_bf16(qI)
    w = np.array([[1.0, 0.0, 0.0, 0.0]], np.float32)
    seqs = torch.tensor([[0, 0, 0, 4 * E]], dtype=torch.int64, device="cuda")
    qt = gh.query_table([(0, 4 * E)])
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, 1, 4 * E
    ws = torch.empty(csa.csa_workspace_size(csa.CSA_OP_INDEX_TOPK, wq), dtype=torch.uint8, device="cuda")
    idx = torch.full((1, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.empty(1, k, dtype=torch.float32, device="cuda")
    csa.csa_index_topk(dims, seqs, qt, 1, 4 * E, gh.to_dev_bf16(qI), torch.from_numpy(w).cuda(), gh.to_dev_bf16(K),
                       idx, sc, ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    s = oracle.index_scores(qI[0], w[0], K)
    ref = oracle.topk(s, k)
    np.testing.assert_array_equal(idx.cpu().numpy()[0], ref)
    np.testing.assert_array_equal(sc.cpu().numpy()[0], s[ref].astype(np.float32))


# --------------------------------------------------------------------------------- f1: 8-bit keys

@pytest.mark.parametrize("E_list,d_I,scale", [([5000, 300], 64, 1.0), ([2000], 32, 1.0), ([700], 64, 2.0 ** -30),
                                              ([900], 64, 7.0e3)], ids=["prod", "d32", "tiny_values", "large"])
def test_quantize_keys_matches_oracle(E_list, d_I, scale):
    """csa_quantize_keys writes exactly the oracle's E4M3 bytes and scale bytes (all-zero rows and
    extreme magnitudes included)."""
    dims = csa.make_dims(d=512, H=64, d_I=d_I, H_I=4, m=4, m_hca=128, k=1024, W=128)
    Ks = [oracle.round_bf16(synth.bf16_to_f64(synth.bf16_normal(3101, synth.KI, i, d_I, 0, E)) * scale)
          for i, E in enumerate(E_list)]
    Ks[0][3] = 0
    offs = np.cumsum([0] + list(E_list))
    keys = gh.to_dev_bf16(np.concatenate(Ks))
    seqs = torch.tensor([[0, offs[i], 0, 4 * E] for i, E in enumerate(E_list)], dtype=torch.int64, device="cuda")
    ranges = torch.tensor([[0, E] for E in E_list], dtype=torch.int64, device="cuda")
    kq = torch.full((offs[-1], d_I), 0xAA, dtype=torch.uint8, device="cuda")
    ks = torch.full((offs[-1], d_I // 32), 0xAA, dtype=torch.uint8, device="cuda")
    csa.csa_quantize_keys(dims, seqs, ranges, len(E_list), max(E_list), keys, kq, ks)
    assert csa.csa_sync_status() == csa.CSA_OK
    ref_q, ref_s = oracle.quantize_keys_mx8(np.concatenate(Ks))
    np.testing.assert_array_equal(ks.cpu().numpy(), ref_s)
    np.testing.assert_array_equal(kq.cpu().numpy(), ref_q)


@pytest.mark.parametrize("E_list,k,d_I", [([5000], 1024, 64), ([300], 32, 32), ([600], 1024, 64),
                                          ([1025, 70000, 4097, 1], 1024, 64), ([262144], 1024, 64),
                                          ([40000, 33000], 2048, 64)],
                         ids=["E5000", "tiny", "E<k", "ragged4", "E262144", "k2048"])
def test_index_topk_mx8_stage(E_list, k, d_I, H_I=4, seed=3201):
    """The indexer on 8-bit keys selects the oracle's top-k of the dequantized keys' scores (both sides
    score the same bytes; ties resolved as for bf16 keys), with the scores."""
    dims = csa.make_dims(d=512, H=64, d_I=d_I, H_I=H_I, m=4, m_hca=128, k=k, W=128)
    Q = len(E_list)
    KQ, SC = [], []
    for i, E in enumerate(E_list):
        kq, sc = oracle.quantize_keys_mx8(synth.bf16_normal(seed, synth.KI, i, d_I, 0, max(E, 1)))
        KQ.append(kq)
        SC.append(sc)
    offs = np.cumsum([0] + [max(E, 1) for E in E_list])
    keys_q = torch.from_numpy(np.concatenate(KQ)).cuda()
    key_scales = torch.from_numpy(np.concatenate(SC)).cuda()
    seqs = torch.tensor([[0, offs[i], 0, 4 * E + 3] for i, E in enumerate(E_list)], dtype=torch.int64, device="cuda")
    qt = gh.query_table([(i, 4 * E + 3) for i, E in enumerate(E_list)])
    qI = synth.bf16_normal(seed, synth.QI, 99, H_I * d_I, 0, Q).reshape(Q, H_I, d_I)
    w = synth.f32_uniform(seed, synth.W, 99, H_I, 0, Q)
    idx = torch.full((Q, k), -7, dtype=torch.int32, device="cuda")
    sc_out = torch.empty(Q, k, dtype=torch.float32, device="cuda")
    max_len = 4 * max(E_list) + 3
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, Q, max_len
    ws = torch.empty(csa.csa_workspace_size(csa.CSA_OP_INDEX_TOPK, wq), dtype=torch.uint8, device="cuda")
    csa.csa_index_topk_mx8(dims, seqs, qt, Q, max_len, gh.to_dev_bf16(qI), torch.from_numpy(w).cuda(), keys_q,
                           key_scales, idx, sc_out, ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    idx_h, sc_h = idx.cpu().numpy(), sc_out.cpu().numpy()
    for i, E in enumerate(E_list):
        s = oracle.index_scores_mx8(qI[i], w[i], KQ[i][:E], SC[i][:E])
        ref = oracle.topk(s, k)
        gh.sets_match(idx_h[i], ref, s, k)
        valid = idx_h[i][idx_h[i] >= 0]
        assert (np.diff(valid) > 0).all() and len(valid) == min(E, k)
        np.testing.assert_allclose(sc_h[i][:len(valid)], s[valid], rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("wl,steps", [(workloads.tiny(), 3), (wl_small([3000, 9001], B=2), 5)], ids=["tiny", "prod"])
def test_decode_with_8bit_keys(wl, steps):
    """Decode with the indexer on 8-bit keys: the append writes the 8-bit copy of every key it completes
    (equal to quantizing the stored bf16 key), the selection is the oracle's top-k of the 8-bit keys'
    scores, and the output is the oracle's attention over the GPU's caches with that selection."""
    wl = dataclasses.replace(wl, steps=max(wl.steps, steps))  # room for every appended token
    d = wl.dims
    layer = csa.HybridLayer(gh.dims_of(d), [wl.capacity(b) for b in range(wl.B)], key_format="mx8")
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths(list(wl.n0))
    layer.compress()
    B = wl.B
    q = torch.empty(B, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(B, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(B, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(B, d.H, d.d, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, d.k, dtype=torch.int32, device="cuda")
    ws = layer.decode_workspace()
    sh = gh.oshape(d)
    for s in range(steps):
        for b in range(B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
        layer.decode(layer.decode_args(q, qi, w, out, idx_out=idx), ws)
        assert csa.csa_sync_status() == csa.CSA_OK
        keys = gh.u16(layer.entry_keys)
        kq, ks = layer.keys_q.cpu().numpy(), layer.key_scales.cpu().numpy()
        ent, hca, x = gh.u16(layer.entries), gh.u16(layer.hca_entries), gh.u16(layer.x)
        for b in range(B):
            L = wl.n0[b] + s + 1
            c0, n_c = layer.csa_off[b], L // d.m
            rq, rs = oracle.quantize_keys_mx8(keys[c0:c0 + n_c])
            np.testing.assert_array_equal(kq[c0:c0 + n_c], rq)
            np.testing.assert_array_equal(ks[c0:c0 + n_c], rs)
            qh, qih, wh = workloads.queries(wl, b, s, s + 1)
            sc = oracle.index_scores_mx8(qih[0], wh[0], rq, rs)
            gh.sets_match(idx[b].cpu().numpy(), oracle.topk(sc, d.k), sc, d.k)
            t0, h0 = layer.tok_off[b], layer.hca_off[b]
            O_c, l_c = oracle.csa_attn(qh[0], ent[c0:c0 + max(n_c, 1)], idx[b].cpu().numpy(), d.m,
                                       x[t0:t0 + L], L, d.W, sh.scale)
            O_h, l_h = oracle.hca_attn(qh[0], hca[h0:h0 + max(L // d.m_hca, 1)], d.m_hca, x[t0:t0 + L], L, 0, sh.scale)
            O, _ = oracle.lse_merge(O_c, l_c, O_h, l_h)
            gh.check_close(out[b].cpu().numpy(), O, f"8-bit keys: step {s} seq {b}")


# --------------------------------------------------------------------------------- f4: FP4 entries

def _mx4_codes_match(got, want):
    """Packed E2M1 code bytes equal, except that a zero element (magnitude bits 0) may carry either
    sign (both are the value 0)."""
    def canon(b):
        lo, hi = b & 15, b >> 4
        lo = np.where((lo & 7) == 0, 0, lo)
        hi = np.where((hi & 7) == 0, 0, hi)
        return lo | (hi << 4)
    return np.array_equal(canon(got), canon(want))


def _check_mx4(eq, es, E_rows, what):
    """The FP4 copies (codes eq, scales es) of bf16 rows E_rows are the oracle's quantization."""
    rq, rs = oracle.quantize_entries_mx4(E_rows)
    np.testing.assert_array_equal(es, rs, err_msg=f"{what}: scale bytes")
    assert _mx4_codes_match(eq, rq), f"{what}: codes"
    np.testing.assert_array_equal(oracle.dequantize_entries_mx4(eq, es), oracle.dequantize_entries_mx4(rq, rs))


@pytest.mark.parametrize("E_list,d,scale", [([700, 33], 512, 1.0), ([257], 128, 2.0 ** -60), ([100, 5], 512, 7.0e4)])
@pytest.mark.parametrize("which", [0, 1])
def test_quantize_entries_matches_oracle(E_list, d, scale, which):
    """csa_quantize_entries writes the oracle's scale bytes and E2M1 codes for stored CSA / HCA entries
    (an all-zero row and extreme magnitudes included)."""
    dims = csa.make_dims(d=d, H=8, d_I=32, H_I=4, m=4, m_hca=16, k=32, W=16)
    ratio = 4 if which == 0 else 16
    Es = [oracle.round_bf16(synth.bf16_to_f64(synth.bf16_normal(3301, synth.X, i, d, 0, E)) * scale)
          for i, E in enumerate(E_list)]
    Es[0][3] = 0
    offs = np.cumsum([0] + list(E_list))
    ent = gh.to_dev_bf16(np.concatenate(Es))
    rows = [[0, offs[i], 0, ratio * E] if which == 0 else [0, 0, offs[i], ratio * E] for i, E in enumerate(E_list)]
    seqs = torch.tensor(rows, dtype=torch.int64, device="cuda")
    ranges = torch.tensor([[0, E] for E in E_list], dtype=torch.int64, device="cuda")
    eq = torch.full((offs[-1], d // 2), 0xAA, dtype=torch.uint8, device="cuda")
    es = torch.full((offs[-1], d // 32), 0xAA, dtype=torch.uint8, device="cuda")
    csa.csa_quantize_entries(dims, seqs, ranges, len(E_list), max(E_list), which, ent, eq, es)
    assert csa.csa_sync_status() == csa.CSA_OK
    _check_mx4(eq.cpu().numpy(), es.cpu().numpy(), np.concatenate(Es), f"which={which}")


@pytest.mark.parametrize("wl,lens", [(workloads.tiny(), [1023, 17, 5]),
                                     (wl_small(5000, B=1), [5000, 4096, 130, 1]),
                                     (wl_small([3000, 1300], B=2), [3000, 1299])],
                         ids=["tiny", "prod", "prod_ragged"])
def test_fp4_attention_stage(wl, lens):
    """Sparse and HCA attention reading FP4 entry caches (the oracle's quantization of its own entries,
    the same bytes on both sides) against the oracle's attention over the dequantized entries."""
    layer, refs = _stage_layer(wl)
    d = wl.dims
    sh = gh.oshape(d)
    n_rows_c, n_rows_h = layer.entries.shape[0], layer.hca_entries.shape[0]
    eq = torch.zeros(n_rows_c, d.d // 2, dtype=torch.uint8, device="cuda")
    es = torch.zeros(n_rows_c, d.d // 32, dtype=torch.uint8, device="cuda")
    hq = torch.zeros(n_rows_h, d.d // 2, dtype=torch.uint8, device="cuda")
    hs = torch.zeros(n_rows_h, d.d // 32, dtype=torch.uint8, device="cuda")
    deq_c, deq_h = [], []
    for b in range(wl.B):
        n_c, n_h = len(refs[b].E), wl.n0[b] // d.m_hca
        q_, s_ = oracle.quantize_entries_mx4(refs[b].E)
        eq[layer.csa_off[b]:layer.csa_off[b] + n_c] = torch.from_numpy(q_).cuda()
        es[layer.csa_off[b]:layer.csa_off[b] + n_c] = torch.from_numpy(s_).cuda()
        deq_c.append(oracle.mx4_entries_as_bf16(refs[b].E))
        if n_h:
            q_, s_ = oracle.quantize_entries_mx4(refs[b].H[:n_h])
            hq[layer.hca_off[b]:layer.hca_off[b] + n_h] = torch.from_numpy(q_).cuda()
            hs[layer.hca_off[b]:layer.hca_off[b] + n_h] = torch.from_numpy(s_).cuda()
            deq_h.append(oracle.mx4_entries_as_bf16(refs[b].H[:n_h]))
        else:
            deq_h.append(refs[b].H[:1])
    pairs = [(i % wl.B, L) for i, L in enumerate(lens)]
    pairs = [(b, min(L, wl.n0[b])) for b, L in pairs]
    Q = len(pairs)
    qs = np.stack([workloads.queries(wl, b, i, i + 1)[0][0] for i, (b, _) in enumerate(pairs)])
    idxs = []
    for i, (b, L) in enumerate(pairs):
        _, qi_, w_ = workloads.queries(wl, b, i, i + 1)
        idxs.append(oracle.topk(oracle.index_scores(qi_[0], w_[0], refs[b].KI[:L // d.m]), d.k))
    qt = gh.query_table(pairs)
    q_d = gh.to_dev_bf16(qs)
    idx_d = torch.from_numpy(np.stack(idxs)).cuda()
    out = torch.empty(Q, d.H, d.d, dtype=torch.float32, device="cuda")
    lse = torch.empty(Q, d.H, dtype=torch.float32, device="cuda")
    dims = gh.dims_of(d)
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, Q, max(wl.n0)
    ws = torch.empty(max(csa.csa_workspace_size(csa.CSA_OP_SPARSE_ATTN, wq),
                         csa.csa_workspace_size(csa.CSA_OP_HCA_ATTN, wq)) + 256, dtype=torch.uint8, device="cuda")
    csa.csa_sparse_attn_fp4(dims, layer.seqs, qt, Q, q_d, eq, es, idx_d, layer.x, sh.scale, out, lse, ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    for i, (b, L) in enumerate(pairs):
        O, l = oracle.csa_attn(qs[i], deq_c[b], idxs[i], d.m, refs[b].x, L, d.W, sh.scale)
        gh.check_close(out[i].cpu().numpy(), O, f"fp4 csa q{i} L={L}")
        gh.check_close(lse[i].cpu().numpy(), l, f"fp4 csa lse q{i}")
    for W in (0, d.W):
        out.fill_(float("nan"))
        csa.hca_dense_attn_fp4(dims, layer.seqs, qt, Q, max(wl.n0), q_d, hq, hs, layer.x, W, sh.scale, out, lse, ws)
        assert csa.csa_sync_status() == csa.CSA_OK
        for i, (b, L) in enumerate(pairs):
            O, l = oracle.hca_attn(qs[i], deq_h[b], d.m_hca, refs[b].x, L, W, sh.scale)
            if np.isneginf(l).all():
                assert np.isneginf(lse[i].cpu().numpy()).all() and (out[i] == 0).all()
                continue
            gh.check_close(out[i].cpu().numpy(), O, f"fp4 hca q{i} L={L} W={W}")
            gh.check_close(lse[i].cpu().numpy(), l, f"fp4 hca lse q{i}")


@pytest.mark.parametrize("wl,steps", [(workloads.tiny(), 3), (wl_small([3000, 9001], B=2), 5)], ids=["tiny", "prod"])
def test_decode_with_fp4_entries(wl, steps):
    """Decode reading FP4 entry caches: the FP4 copies (from the full pass, and from the append for the
    entries it completes) are the oracle's quantization of the stored bf16 entries, the selection is
    the oracle's top-k, and the output is the oracle's attention over the dequantized entries."""
    wl = dataclasses.replace(wl, steps=max(wl.steps, steps))
    d = wl.dims
    layer = csa.HybridLayer(gh.dims_of(d), [wl.capacity(b) for b in range(wl.B)], kv_format="fp4")
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths(list(wl.n0))
    layer.compress()
    B = wl.B
    q = torch.empty(B, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(B, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(B, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(B, d.H, d.d, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, d.k, dtype=torch.int32, device="cuda")
    ws = layer.decode_workspace()
    sh = gh.oshape(d)
    for s in range(steps):
        for b in range(B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
        layer.decode(layer.decode_args(q, qi, w, out, idx_out=idx), ws)
        assert csa.csa_sync_status() == csa.CSA_OK
        ent, hca, x, keys = gh.u16(layer.entries), gh.u16(layer.hca_entries), gh.u16(layer.x), gh.u16(layer.entry_keys)
        eq, es = layer.entries_q.cpu().numpy(), layer.entry_scales.cpu().numpy()
        hq, hs = layer.hca_q.cpu().numpy(), layer.hca_scales.cpu().numpy()
        for b in range(B):
            L = wl.n0[b] + s + 1
            c0, n_c, h0, n_h, t0 = layer.csa_off[b], L // d.m, layer.hca_off[b], L // d.m_hca, layer.tok_off[b]
            _check_mx4(eq[c0:c0 + n_c], es[c0:c0 + n_c], ent[c0:c0 + n_c], f"CSA step {s} seq {b}")
            if n_h:
                _check_mx4(hq[h0:h0 + n_h], hs[h0:h0 + n_h], hca[h0:h0 + n_h], f"HCA step {s} seq {b}")
            qh, qih, wh = workloads.queries(wl, b, s, s + 1)
            sc = oracle.index_scores(qih[0], wh[0], keys[c0:c0 + n_c])
            gh.sets_match(idx[b].cpu().numpy(), oracle.topk(sc, d.k), sc, d.k)
            dc = oracle.mx4_entries_as_bf16(ent[c0:c0 + max(n_c, 1)])
            dh = oracle.mx4_entries_as_bf16(hca[h0:h0 + n_h]) if n_h else hca[h0:h0 + 1]
            O_c, l_c = oracle.csa_attn(qh[0], dc, idx[b].cpu().numpy(), d.m, x[t0:t0 + L], L, d.W, sh.scale)
            O_h, l_h = oracle.hca_attn(qh[0], dh, d.m_hca, x[t0:t0 + L], L, 0, sh.scale)
            O, _ = oracle.lse_merge(O_c, l_c, O_h, l_h)
            gh.check_close(out[b].cpu().numpy(), O, f"fp4 decode step {s} seq {b}")


# --------------------------------------------------------------------------------- f2: index reuse

def _oracle_on_gpu_caches(layer, b, L, qh, idx_b, d):
    """The oracle's merged output for one query of `layer` at length L over the layer's own (GPU)
    caches with a given selection."""
    sh = gh.oshape(d)
    ent, hca, x = gh.u16(layer.entries), gh.u16(layer.hca_entries), gh.u16(layer.x)
    c0, t0, h0 = layer.csa_off[b], layer.tok_off[b], layer.hca_off[b]
    O_c, l_c = oracle.csa_attn(qh, ent[c0:c0 + max(L // d.m, 1)], idx_b, d.m, x[t0:t0 + L], L, d.W, sh.scale)
    O_h, l_h = oracle.hca_attn(qh, hca[h0:h0 + max(L // d.m_hca, 1)], d.m_hca, x[t0:t0 + L], L, 0, sh.scale)
    return oracle.lse_merge(O_c, l_c, O_h, l_h)[0]


@pytest.mark.parametrize("wl", [workloads.tiny(), wl_small([3000, 9001], B=2)], ids=["tiny", "prod"])
def test_decode_reuses_the_source_layers_selection(wl):
    """Cross-layer index reuse: layer 2 (its own caches, other inputs) attends the entries layer 1's
    indexer selected in the same step; its output is the oracle's attention over layer 2's caches
    with layer 1's selection."""
    wl = dataclasses.replace(wl, steps=max(wl.steps, 2))  # room for both appended tokens
    d = wl.dims
    wl2 = workloads.Workload(wl.name + "_layer2", wl.seed + 77, d, wl.n0, wl.steps)
    l1, l2 = gh.new_layer(wl), gh.new_layer(wl2)
    B = wl.B
    mk = lambda *shape, dt=torch.bfloat16: torch.empty(*shape, dtype=dt, device="cuda")
    q, qi, w = mk(B, d.H, d.d), mk(B, d.H_I, d.d_I), mk(B, d.H_I, dt=torch.float32)
    q2 = mk(B, d.H, d.d)
    out1, out2 = mk(B, d.H, d.d, dt=torch.float32), mk(B, d.H, d.d, dt=torch.float32)
    idx = mk(B, d.k, dt=torch.int32)
    ws1, ws2 = l1.decode_workspace(), l2.decode_workspace()
    for s in range(2):
        for b in range(B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
            sdev.fill_queries(wl2, b, s, s + 1, q2[b:b + 1], qi[b:b + 1].clone(), w[b:b + 1].clone())
        l1.decode(l1.decode_args(q, qi, w, out1, idx_out=idx), ws1)
        l2.decode(l2.decode_args(q2, None, None, out2, idx_in=idx), ws2)
        assert csa.csa_sync_status() == csa.CSA_OK
        for b in range(B):
            L = wl.n0[b] + s + 1
            qh = workloads.queries(wl2, b, s, s + 1)[0][0]
            O = _oracle_on_gpu_caches(l2, b, L, qh, idx[b].cpu().numpy(), d)
            gh.check_close(out2[b].cpu().numpy(), O, f"reuse step {s} seq {b}")


def test_prefill_reuses_the_source_layers_selection():
    d = workloads.TINY_DIMS
    N = 1024
    wl1 = workloads.Workload("prefill_l1", 4101, d, (N,), 0, mode="prefill")
    wl2 = workloads.Workload("prefill_l2", 4102, d, (N,), 0, mode="prefill")
    layers, qs = [], []
    for wl in (wl1, wl2):
        layer = csa.HybridLayer(gh.dims_of(d), [N])
        sdev.fill_layer_inputs(layer, wl)
        layer.set_lengths([N])
        q = torch.empty(N, d.H, d.d, dtype=torch.bfloat16, device="cuda")
        qi = torch.empty(N, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
        w = torch.empty(N, d.H_I, dtype=torch.float32, device="cuda")
        sdev.fill_queries(wl, 0, 0, N, q, qi, w)
        layers.append(layer)
        qs.append((q, qi, w))
    idx = torch.empty(N, d.k, dtype=torch.int32, device="cuda")
    out1 = torch.empty(N, d.H, d.d, dtype=torch.float32, device="cuda")
    out2 = torch.empty_like(out1)
    l1, l2 = layers
    l1.prefill(l1.prefill_args(*qs[0], out1, 0, N, compress=True, idx_out=idx), l1.prefill_workspace(N))
    l2.prefill(l2.prefill_args(qs[1][0], None, None, out2, 0, N, compress=True, idx_in=idx), l2.prefill_workspace(N))
    assert csa.csa_sync_status() == csa.CSA_OK
    qh = workloads.queries(wl2, 0, 0, N)[0]
    idx_h, o2 = idx.cpu().numpy(), out2.cpu().numpy()
    for i in list(range(0, N, 61)) + [N - 1]:
        O = _oracle_on_gpu_caches(l2, 0, i + 1, qh[i], idx_h[i], d)
        gh.check_close(o2[i], O, f"prefill reuse row {i}")


# --------------------------------------------------------------------------------- f3: norms, sinks

def _norm_tensors(wl, seed=5101):
    d = wl.dims
    g = lambda t, rows: torch.from_numpy(1.0 + 0.25 * synth.f32_normal(seed, t, 0, d.d, 0, rows)[0]).cuda()
    q_norm, en_c, en_h = g(synth.Q, 1), g(synth.A, 1), g(synth.B, 1)
    sink = torch.from_numpy(2.0 * synth.f32_normal(seed, synth.W, 0, d.H, 0, 1)[0]).cuda()
    return q_norm, en_c, en_h, sink


def _normed_layer(wl, lens=None, eps=1e-5):
    layer = csa.HybridLayer(gh.dims_of(wl.dims), [wl.capacity(b) for b in range(wl.B)])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths(list(wl.n0) if lens is None else lens)
    t = _norm_tensors(wl)
    layer.set_norms(*t, eps=eps)
    layer.compress()
    torch.cuda.synchronize()
    return layer, t


@pytest.mark.parametrize("wl", [workloads.tiny(), wl_small([2000, 333], B=2)], ids=["tiny", "prod"])
def test_normalized_entries_within_one_ulp(wl):
    """RMS-normalized CSA and HCA entries against the oracle's normalization of its fp64 entries:
    one bf16 ulp plus the fp32 accumulation bound carried through the normalization."""
    layer, (q_norm, en_c, en_h, sink) = _normed_layer(wl)
    d = wl.dims
    eps = 1e-5
    for b in range(wl.B):
        n = wl.n0[b]
        ref = gh.OracleSeq(wl, b, n, with_mass=True)
        for name, off, E64, mass, gain, n_e in (("entries", layer.csa_off, ref.E64, ref.E_mass, en_c, n // d.m),
                                                ("hca_entries", layer.hca_off, getattr(ref, "H64", None),
                                                 getattr(ref, "H_mass", None), en_h, n // d.m_hca)):
            if n_e == 0:
                continue
            gn = gain.cpu().numpy().astype(np.float64)
            want = oracle.rms_norm(E64, gn.astype(np.float32), eps)
            inv = 1.0 / np.sqrt((E64 ** 2).mean(axis=1, keepdims=True) + eps)
            got = gh.u16(getattr(layer, name)[off[b]:off[b] + n_e])
            g64 = synth.bf16_to_f64(got)
            ulp = np.maximum(np.abs(synth.bf16_to_f64(oracle.round_bf16(want))) * 2.0 ** -7, 2.0 ** -133)
            bound = ulp + mass * 2.0 ** -18 * inv * np.abs(gn) + np.abs(want) * 2.0 ** -20
            assert (np.abs(g64 - want) <= bound).all(), f"seq {b} {name}: {(np.abs(g64 - want) > bound).sum()} beyond bound"


@pytest.mark.parametrize("wl", [workloads.tiny(), wl_small([1000, 515], B=2, steps=130)], ids=["tiny", "prod"])
def test_normalized_append_equals_full_pass(wl):
    """With entry normalization the decode append still leaves the caches bit-identical to a full pass."""
    d = wl.dims
    layer, t = _normed_layer(wl)
    q = torch.empty(wl.B, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(wl.B, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(wl.B, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(wl.B, d.H, d.d, dtype=torch.float32, device="cuda")
    ws = layer.decode_workspace()
    for s in range(wl.steps):
        for b in range(wl.B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
        layer.decode(layer.decode_args(q, qi, w, out), ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    full, _ = _normed_layer(wl, lens=[n + wl.steps for n in wl.n0])
    for name in ("entries", "entry_keys", "hca_entries"):
        assert torch.equal(getattr(layer, name).view(torch.int16), getattr(full, name).view(torch.int16)), name


def _oracle_normed(layer, b, L, qh, idx_b, d, q_gain, sink, eps):
    sh = gh.oshape(d)
    ent, hca, x = gh.u16(layer.entries), gh.u16(layer.hca_entries), gh.u16(layer.x)
    c0, t0, h0 = layer.csa_off[b], layer.tok_off[b], layer.hca_off[b]
    qn = oracle.round_bf16(oracle.rms_norm(synth.bf16_to_f64(qh), q_gain, eps))
    O_c, l_c = oracle.csa_attn(qn, ent[c0:c0 + max(L // d.m, 1)], idx_b, d.m, x[t0:t0 + L], L, d.W, sh.scale)
    O_h, l_h = oracle.hca_attn(qn, hca[h0:h0 + max(L // d.m_hca, 1)], d.m_hca, x[t0:t0 + L], L, 0, sh.scale)
    O, lse = oracle.lse_merge(O_c, l_c, O_h, l_h)
    return oracle.sink_merge(O, lse, sink)


@pytest.mark.parametrize("wl,steps", [(workloads.tiny(), 2), (wl_small([3000, 9001], B=2), 2)], ids=["tiny", "prod"])
def test_decode_with_norms_and_sinks(wl, steps):
    """Query normalization and sink logits in the decode step (merge kernel), over the GPU's own
    normalized caches and selection."""
    wl = dataclasses.replace(wl, steps=max(wl.steps, steps))  # room for every appended token
    d = wl.dims
    layer, (q_norm, en_c, en_h, sink) = _normed_layer(wl)
    B = wl.B
    q = torch.empty(B, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(B, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(B, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(B, d.H, d.d, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, d.H, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, d.k, dtype=torch.int32, device="cuda")
    ws = layer.decode_workspace()
    qg, sk = q_norm.cpu().numpy(), sink.cpu().numpy().astype(np.float64)
    for s in range(steps):
        for b in range(B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
        layer.decode(layer.decode_args(q, qi, w, out, lse=lse, idx_out=idx), ws)
        assert csa.csa_sync_status() == csa.CSA_OK
        for b in range(B):
            L = wl.n0[b] + s + 1
            qh = workloads.queries(wl, b, s, s + 1)[0][0]
            O, l = _oracle_normed(layer, b, L, qh, idx[b].cpu().numpy(), d, qg, sk, 1e-5)
            gh.check_close(out[b].cpu().numpy(), O, f"norms+sinks step {s} seq {b}")
            gh.check_close(lse[b].cpu().numpy(), l, f"norms+sinks lse step {s} seq {b}")


def test_prefill_with_norms_and_sinks():
    """The same in the prefill, where one item holds a query's whole softmax (sink in the epilogue)."""
    d = workloads.TINY_DIMS
    N = 1024
    wl = workloads.Workload("prefill_norms", 4201, d, (N,), 0, mode="prefill")
    layer = csa.HybridLayer(gh.dims_of(d), [N])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths([N])
    q_norm, en_c, en_h, sink = _norm_tensors(wl)
    layer.set_norms(q_norm, en_c, en_h, sink, eps=1e-5)
    q = torch.empty(N, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(N, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(N, d.H_I, dtype=torch.float32, device="cuda")
    sdev.fill_queries(wl, 0, 0, N, q, qi, w)
    out = torch.empty(N, d.H, d.d, dtype=torch.float32, device="cuda")
    lse = torch.empty(N, d.H, dtype=torch.float32, device="cuda")
    idx = torch.empty(N, d.k, dtype=torch.int32, device="cuda")
    layer.prefill(layer.prefill_args(q, qi, w, out, 0, N, compress=True, lse=lse, idx_out=idx),
                  layer.prefill_workspace(N))
    assert csa.csa_sync_status() == csa.CSA_OK
    qh = workloads.queries(wl, 0, 0, N)[0]
    qg, sk = q_norm.cpu().numpy(), sink.cpu().numpy().astype(np.float64)
    o, lh, ih = out.cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
    for i in [0, 1, 3, 4, 15, 16, 100, 511, N - 1]:
        O, l = _oracle_normed(layer, 0, i + 1, qh[i], ih[i], d, qg, sk, 1e-5)
        gh.check_close(o[i], O, f"prefill norms row {i}")
        gh.check_close(lh[i], l, f"prefill norms lse row {i}")


# --------------------------------------------------------------------------------- a5/a6 (stage)

def _stage_layer(wl):
    """A layer whose caches hold the ORACLE's bf16 entries (identical input bytes on both sides)."""
    layer = csa.HybridLayer(gh.dims_of(wl.dims), [wl.capacity(b) for b in range(wl.B)])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths(list(wl.n0))
    refs = []
    for b in range(wl.B):
        r = gh.OracleSeq(wl, b, wl.n0[b])
        n_c, n_h = len(r.E), wl.n0[b] // wl.dims.m_hca
        layer.entries[layer.csa_off[b]:layer.csa_off[b] + n_c] = gh.to_dev_bf16(r.E)
        layer.entry_keys[layer.csa_off[b]:layer.csa_off[b] + n_c] = gh.to_dev_bf16(r.KI)
        if n_h:
            layer.hca_entries[layer.hca_off[b]:layer.hca_off[b] + n_h] = gh.to_dev_bf16(r.H[:n_h])
        refs.append(r)
    return layer, refs


@pytest.mark.parametrize("wl,lens", [(workloads.tiny(), [1023, 17, 5]),
                                     (wl_small(5000, B=1), [5000, 4096, 130, 1]),
                                     (wl_small([3000, 1300], B=2), [3000, 1299])],
                         ids=["tiny", "prod", "prod_ragged"])
def test_sparse_and_hca_attention_stage(wl, lens):
    layer, refs = _stage_layer(wl)
    d = wl.dims
    sh = gh.oshape(d)
    pairs = [(i % wl.B, L) for i, L in enumerate(lens)]
    pairs = [(b, min(L, wl.n0[b])) for b, L in pairs]
    Q = len(pairs)
    qs = np.stack([workloads.queries(wl, b, i, i + 1)[0][0] for i, (b, _) in enumerate(pairs)])
    idxs = []
    for i, (b, L) in enumerate(pairs):
        _, qi_, w_ = workloads.queries(wl, b, i, i + 1)
        s = oracle.index_scores(qi_[0], w_[0], refs[b].KI[:L // d.m])
        idxs.append(oracle.topk(s, d.k))
    qt = gh.query_table(pairs)
    q_d = gh.to_dev_bf16(qs)
    idx_d = torch.from_numpy(np.stack(idxs)).cuda()
    out = torch.empty(Q, d.H, d.d, dtype=torch.float32, device="cuda")
    lse = torch.empty(Q, d.H, dtype=torch.float32, device="cuda")
    dims = gh.dims_of(d)
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, Q, max(wl.n0)
    ws = torch.empty(max(csa.csa_workspace_size(csa.CSA_OP_SPARSE_ATTN, wq),
                         csa.csa_workspace_size(csa.CSA_OP_HCA_ATTN, wq)) + 256, dtype=torch.uint8, device="cuda")
    csa.csa_sparse_attn(dims, layer.seqs, qt, Q, q_d, layer.entries, idx_d, layer.x, sh.scale, out, lse, ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    for i, (b, L) in enumerate(pairs):
        O, l = oracle.csa_attn(qs[i], refs[b].E, idxs[i], d.m, refs[b].x, L, d.W, sh.scale)
        gh.check_close(out[i].cpu().numpy(), O, f"csa q{i} L={L}")
        gh.check_close(lse[i].cpu().numpy(), l, f"csa lse q{i}")
    for W in (0, d.W):
        out.fill_(float("nan"))
        csa.hca_dense_attn(dims, layer.seqs, qt, Q, max(wl.n0), q_d, layer.hca_entries, layer.x, W, sh.scale, out,
                           lse, ws)
        assert csa.csa_sync_status() == csa.CSA_OK
        for i, (b, L) in enumerate(pairs):
            O, l = oracle.hca_attn(qs[i], refs[b].H, d.m_hca, refs[b].x, L, W, sh.scale)
            if np.isneginf(l).all():  # no key at all: zero output, lse = -inf
                assert np.isneginf(lse[i].cpu().numpy()).all() and (out[i] == 0).all()
                continue
            gh.check_close(out[i].cpu().numpy(), O, f"hca q{i} L={L} W={W}")
            gh.check_close(lse[i].cpu().numpy(), l, f"hca lse q{i}")


@pytest.mark.parametrize("fp4", [False, True], ids=["bf16", "fp4"])
def test_sparse_attention_persistent_ctas(fp4):
    """More queries than SMs in one direct launch: persistent CTAs take every G-th query, the loader
    warps store each later query's Q and read its slot indices ahead.  Rows that CTAs run first,
    second and third are checked against the oracle (bf16 entries, or the FP4 cache against the
    oracle's dequantized entries); one query with no visible token (length 0) is reported, gets zeros
    and lse = -inf, and leaves the others intact."""
    wl = wl_small(5000, B=1)
    layer, refs = _stage_layer(wl)
    d = wl.dims
    sh = gh.oshape(d)
    Q = 301
    lens = [1 + (i * 2711) % 5000 for i in range(Q)]
    lens[5], lens[160], lens[299] = 5000, 1, 4
    lens[200] = 0  # invalid: reported, zeros
    pairs = [(0, L) for L in lens]
    qs = np.stack([workloads.queries(wl, 0, i % 64, i % 64 + 1)[0][0] for i in range(Q)])
    idxs = []
    for i, L in enumerate(lens):
        _, qi_, w_ = workloads.queries(wl, 0, i % 64, i % 64 + 1)
        s = oracle.index_scores(qi_[0], w_[0], refs[0].KI[:L // d.m])
        idxs.append(oracle.topk(s, d.k))
    ent = refs[0].E
    qt = gh.query_table(pairs)
    q_d = gh.to_dev_bf16(qs)
    idx_d = torch.from_numpy(np.stack(idxs)).cuda()
    out = torch.full((Q, d.H, d.d), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.empty(Q, d.H, dtype=torch.float32, device="cuda")
    dims = gh.dims_of(d)
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, Q, max(wl.n0)
    ws = torch.empty(csa.csa_workspace_size(csa.CSA_OP_SPARSE_ATTN, wq) + 256, dtype=torch.uint8, device="cuda")
    if fp4:
        n_c = len(refs[0].E)
        eq = torch.zeros(layer.entries.shape[0], d.d // 2, dtype=torch.uint8, device="cuda")
        es = torch.zeros(layer.entries.shape[0], d.d // 32, dtype=torch.uint8, device="cuda")
        q_, s_ = oracle.quantize_entries_mx4(refs[0].E)
        eq[layer.csa_off[0]:layer.csa_off[0] + n_c] = torch.from_numpy(q_).cuda()
        es[layer.csa_off[0]:layer.csa_off[0] + n_c] = torch.from_numpy(s_).cuda()
        ent = oracle.mx4_entries_as_bf16(refs[0].E)
        csa.csa_sparse_attn_fp4(dims, layer.seqs, qt, Q, q_d, eq, es, idx_d, layer.x, sh.scale, out, lse, ws)
    else:
        csa.csa_sparse_attn(dims, layer.seqs, qt, Q, q_d, layer.entries, idx_d, layer.x, sh.scale, out, lse, ws)
    assert csa.csa_sync_status() == csa.CSA_ERR_INDEX
    assert csa.csa_sync_status() == csa.CSA_OK  # cleared
    assert (out[200] == 0).all() and torch.isneginf(lse[200]).all()
    keep = torch.ones(Q, dtype=torch.bool)
    keep[200] = False
    assert torch.isfinite(out[keep.cuda()]).all()
    for i in (0, 5, 7, 147, 148, 150, 160, 199, 201, 295, 296, 299, 300):
        L = lens[i]
        O, l = oracle.csa_attn(qs[i], ent, idxs[i], d.m, refs[0].x, L, d.W, sh.scale)
        gh.check_close(out[i].cpu().numpy(), O, f"csa q{i} L={L}")
        gh.check_close(lse[i].cpu().numpy(), l, f"csa lse q{i}")


def test_bad_index_is_reported_not_read():
    wl = workloads.tiny()
    layer, refs = _stage_layer(wl)
    d = wl.dims
    dims = gh.dims_of(d)
    qt = gh.query_table([(0, 64)])  # 16 causal entries
    q = gh.to_dev_bf16(workloads.queries(wl, 0, 0, 1)[0])
    idx = torch.full((1, d.k), -1, dtype=torch.int32, device="cuda")
    idx[0, 0], idx[0, 1] = 3, 200  # 200 is not causal at L = 64
    out = torch.empty(1, d.H, d.d, dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
    csa.csa_sparse_attn(dims, layer.seqs, qt, 1, q, layer.entries, idx, layer.x, 0.1, out, None, ws)
    assert csa.csa_sync_status() == csa.CSA_ERR_INDEX
    assert csa.csa_sync_status() == csa.CSA_OK  # cleared
    idx_ok = idx.clone()
    idx_ok[0, 1] = -1
    out2 = torch.empty_like(out)
    csa.csa_sparse_attn(dims, layer.seqs, qt, 1, q, layer.entries, idx_ok, layer.x, 0.1, out2, None, ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    assert torch.equal(out, out2)  # the bad slot was skipped, nothing else changed


def test_wait_that_runs_out_is_reported_and_the_device_recovers():
    """A bounded wait that runs out (fault injection: one attention loader warp never arrives on the
    first key tile) is reported as CSA_ERR_TIMEOUT after the short limit, the kernel winds down, and
    the next call on the same context returns CSA_OK with the right output."""
    wl = workloads.tiny()
    layer, refs = _stage_layer(wl)
    d = wl.dims
    dims = gh.dims_of(d)
    sh = gh.oshape(d)
    L = 1000
    qt = gh.query_table([(0, L)])
    qh, qih, wh = workloads.queries(wl, 0, 0, 1)
    idx_h = oracle.topk(oracle.index_scores(qih[0], wh[0], refs[0].KI[:L // d.m]), d.k)
    q = gh.to_dev_bf16(qh)
    idx = torch.from_numpy(idx_h[None].copy()).cuda()
    out = torch.empty(1, d.H, d.d, dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
    try:
        csa.csa_debug_inject(1, 1_000_000)  # 1 ms limit
        csa.csa_sparse_attn(dims, layer.seqs, qt, 1, q, layer.entries, idx, layer.x, sh.scale, out, None, ws)
        assert csa.csa_sync_status() == csa.CSA_ERR_TIMEOUT
    finally:
        csa.csa_debug_inject(0, 0)
    assert csa.csa_sync_status() == csa.CSA_OK  # reading the status cleared it
    csa.csa_sparse_attn(dims, layer.seqs, qt, 1, q, layer.entries, idx, layer.x, sh.scale, out, None, ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    O, _ = oracle.csa_attn(qh[0], refs[0].E, idx_h, d.m, refs[0].x, L, d.W, sh.scale)
    gh.check_close(out[0].cpu().numpy(), O, "after the timeout")


# --------------------------------------------------------------------------------- end to end

def _new_rows(wl, layer, s):
    """The appended token's raw rows of step s for every sequence as new_rows [B, 3d + d_I], after
    zeroing those rows in the layer's caches (so only the call's own copy can put them back)."""
    d = wl.dims
    rows = []
    for b in range(wl.B):
        t = wl.n0[b] + s
        parts = [workloads.raw_tokens(wl, b, t, t + 1, name)[0] for name in ("x", "a", "b", "kI")]
        rows.append(np.concatenate(parts))
        r = layer.tok_off[b] + t
        for cache in (layer.x, layer.logit_c, layer.logit_h, layer.idx_key):
            cache[r].zero_()
    return torch.from_numpy(np.stack(rows).view(np.int16)).cuda().view(torch.bfloat16)


def _decode_e2e(wl, steps, check_every=1, via_new_rows=False):
    layer = gh.new_layer(wl)
    d = wl.dims
    B = wl.B
    q = torch.empty(B, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(B, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(B, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(B, d.H, d.d, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, d.H, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, d.k, dtype=torch.int32, device="cuda")
    ws = layer.decode_workspace()
    refs = [gh.OracleSeq(wl, b, wl.n0[b] + steps) for b in range(B)]
    n_diff = 0
    for s in range(steps):
        for b in range(B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
        nr = _new_rows(wl, layer, s) if via_new_rows else None
        layer.decode(layer.decode_args(q, qi, w, out, lse=lse, idx_out=idx, new_rows=nr), ws)
        assert csa.csa_sync_status() == csa.CSA_OK
        if s % check_every and s != steps - 1:
            continue
        for b in range(B):
            L = wl.n0[b] + s + 1
            qh, qih, wh = workloads.queries(wl, b, s, s + 1)
            r = refs[b].query(L, qh[0], qih[0], wh[0])
            slack = gh.score_slack(qih[0], wh[0], refs[b].KI[:L // d.m])
            n_diff += gh.sets_explained(idx[b].cpu().numpy(), r["idx"], r["scores"], slack)
            gh.check_close(out[b].cpu().numpy(), r["O"], f"decode step {s} seq {b} L={L}")
            gh.check_close(lse[b].cpu().numpy(), r["lse"], f"decode lse step {s} seq {b}")
    return n_diff


def test_ready_word_wait_runs_out_and_the_device_recovers():
    """The front attention items of a decode step wait for their query's ready word from the top-k
    select with a bounded poll: with fault injection 2 the select publishes no word, the wait runs
    out after the short limit and is reported as CSA_ERR_TIMEOUT, and the next step on the same
    context matches the oracle."""
    wl = wl_small(6000)
    layer = gh.new_layer(wl)
    d = wl.dims
    q = torch.empty(1, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(1, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(1, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(1, d.H, d.d, dtype=torch.float32, device="cuda")
    lse = torch.empty(1, d.H, dtype=torch.float32, device="cuda")
    ws = layer.decode_workspace()
    ref = gh.OracleSeq(wl, 0, wl.n0[0] + 2)
    try:
        csa.csa_debug_inject(2, 1_000_000)  # 1 ms limit
        sdev.fill_queries(wl, 0, 0, 1, q, qi, w)
        layer.decode(layer.decode_args(q, qi, w, out, lse=lse), ws)
        assert csa.csa_sync_status() == csa.CSA_ERR_TIMEOUT
    finally:
        csa.csa_debug_inject(0, 0)
    assert csa.csa_sync_status() == csa.CSA_OK  # reading the status cleared it
    sdev.fill_queries(wl, 0, 1, 2, q, qi, w)
    layer.decode(layer.decode_args(q, qi, w, out, lse=lse), ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    L = wl.n0[0] + 2
    qh, qih, wh = workloads.queries(wl, 0, 1, 2)
    r = ref.query(L, qh[0], qih[0], wh[0])
    gh.check_close(out[0].cpu().numpy(), r["O"], "decode step after the timeout")


@pytest.mark.parametrize("wl,steps", [(workloads.tiny(), 1), (wl_small(6000), 3),
                                      (wl_small([700, 3000, 9001], B=3), 2)],
                         ids=["tiny", "prod6000", "ragged3"])
def test_decode_end_to_end(wl, steps):
    _decode_e2e(wl, steps)


@pytest.mark.parametrize("wl,steps", [(workloads.tiny(), 1), (wl_small([700, 3000, 9001], B=3), 3)],
                         ids=["tiny", "ragged3"])
def test_decode_appended_rows_from_new_rows(wl, steps):
    """The appended token's rows handed over as new_rows (the caches hold zeros there) give the same
    results as the oracle: the append kernel copies them in before it compresses (the tiny step and
    the third ragged step of sequence 2, at L = 1024 and 9004, each complete a CSA entry)."""
    _decode_e2e(wl, steps, via_new_rows=True)


@pytest.mark.parametrize("cluster", [4, 8])
def test_decode_cluster_merge(cluster):
    """The optional merge of decode partials across a thread-block cluster (CSA_DECODE_CLUSTER, read
    once per process, so the decode end-to-end cases rerun in a child process with it set)."""
    import os
    import pathlib
    import subprocess
    import sys
    here = pathlib.Path(__file__).resolve()
    env = dict(os.environ, CSA_DECODE_CLUSTER=str(cluster))
    cases = [f"{here}::test_decode_end_to_end", f"{here}::test_decode_with_norms_and_sinks"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *cases],
                       cwd=here.parents[1], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]


def test_decode_with_the_selection_in_the_scan_grid():
    """The optional exact top-k inside the scan grid (CSA_SCAN_SELECT=1, read once per process, so the
    decode end-to-end cases rerun in a child process with it set): the chunks meet on per-query
    counters, the last one selects, and the results equal the oracle's as in the two-kernel path."""
    import os
    import pathlib
    import subprocess
    import sys
    here = pathlib.Path(__file__).resolve()
    env = dict(os.environ, CSA_SCAN_SELECT="1")
    cases = [f"{here}::test_decode_end_to_end", f"{here}::test_decode_with_norms_and_sinks",
             f"{here}::test_decode_with_8bit_keys", f"{here}::test_ready_word_wait_runs_out_and_the_device_recovers"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *cases],
                       cwd=here.parents[1], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]


@pytest.mark.parametrize("N,rows,dims", [
    (1024, list(range(0, 1024, 7)) + [1023], workloads.TINY_DIMS),
    (3000, [0, 1, 2, 3, 4, 5, 127, 128, 129, 1023, 1024, 2047, 2048, 2999], SMALL_PROD)],
    ids=["tiny1024", "prod3000"])
def test_prefill_end_to_end(N, rows, dims):
    wl = workloads.Workload(f"prefill{N}", 4004, dims, (N,), 0, mode="prefill")
    layer = csa.HybridLayer(gh.dims_of(dims), [N])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths([N])
    d = dims
    q = torch.empty(N, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(N, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(N, d.H_I, dtype=torch.float32, device="cuda")
    sdev.fill_queries(wl, 0, 0, N, q, qi, w)
    out = torch.empty(N, d.H, d.d, dtype=torch.float32, device="cuda")
    idx = torch.empty(N, d.k, dtype=torch.int32, device="cuda")
    ws = layer.prefill_workspace(N)
    layer.prefill(layer.prefill_args(q, qi, w, out, 0, N, compress=True, idx_out=idx), ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    ref = gh.OracleSeq(wl, 0, N)
    qh, qih, wh = workloads.queries(wl, 0, 0, N)
    out_h, idx_h = out.cpu().numpy(), idx.cpu().numpy()
    for i in rows:
        L = i + 1
        r = ref.query(L, qh[i], qih[i], wh[i])
        slack = gh.score_slack(qih[i], wh[i], ref.KI[:L // d.m])
        gh.sets_explained(idx_h[i], r["idx"], r["scores"], slack)
        gh.check_close(out_h[i], r["O"], f"prefill row {i}")


# --------------------------------------------------------------------------------- full sizes

def _decode_sampled(wl, steps, check, oracle_seqs, max_len=None):
    """Run `steps` decode steps of the whole workload in the launch configuration of bench.py (one
    hybrid_attn_decode per step over all B sequences, max_len = capacity) and compare the sampled
    (step, sequence) queries with the oracle."""
    layer = csa.HybridLayer(gh.dims_of(wl.dims), [n + steps for n in wl.n0])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths(list(wl.n0))
    layer.compress()
    d = wl.dims
    B = wl.B
    q = torch.empty(B, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(B, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(B, d.H_I, dtype=torch.float32, device="cuda")
    out = torch.empty(B, d.H, d.d, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, d.k, dtype=torch.int32, device="cuda")
    ml = max_len or max(layer.capacity)
    ws = layer.decode_workspace(ml)
    saved = {}
    for s in range(steps):
        for b in range(B):
            sdev.fill_queries(wl, b, s, s + 1, q[b:b + 1], qi[b:b + 1], w[b:b + 1])
        layer.decode(layer.decode_args(q, qi, w, out, idx_out=idx, max_len=ml), ws)
        if s in check:
            saved[s] = (out.cpu().numpy(), idx.cpu().numpy())
    assert csa.csa_sync_status() == csa.CSA_OK
    del layer
    torch.cuda.empty_cache()
    for b in oracle_seqs:
        T = wl.n0[b] + steps
        ref = gh.OracleSeqLazy(wl, b, T) if T > 200000 else gh.OracleSeq(wl, b, T)
        for s in check:
            L = wl.n0[b] + s + 1
            qh, qih, wh = workloads.queries(wl, b, s, s + 1)
            r = ref.query(L, qh[0], qih[0], wh[0])
            o, ix = saved[s]
            slack = gh.score_slack(qih[0], wh[0], ref.KI[:L // d.m])
            nd = gh.sets_explained(ix[b], r["idx"], r["scores"], slack)
            mx, rl2 = gh.check_close(o[b], r["O"], f"step {s} seq {b} L={L}")
            print(f"seq {b} step {s} L={L}: {nd} selection differences (explained), max abs {mx:.2e}, "
                  f"rel L2 {rl2:.2e}")


@pytest.mark.slow
def test_ctx1m_decode_sampled():
    """B=4, N=2^20 (262,144 CSA + 8,192 HCA entries per sequence): two decode steps of the whole
    batch; the oracle checks sequences 0 and 3 at both steps."""
    _decode_sampled(workloads.ctx1m_decode(), 2, {0, 1}, [0, 3])


@pytest.mark.slow
def test_long_decode_sampled():
    """B=1, N0=65,536, all 256 decode steps (crossing two HCA blocks); steps 0, 127, 255 checked."""
    _decode_sampled(workloads.long_decode(), 256, {0, 127, 255}, [0])


@pytest.mark.slow
def test_ragged_decode_sampled():
    """B=32 ragged lengths in [32768, 131072]; 3 decode steps, sequences with the shortest and the
    longest length checked."""
    wl = workloads.ragged_decode()
    lo, hi = int(np.argmin(wl.n0)), int(np.argmax(wl.n0))
    _decode_sampled(wl, 3, {0, 2}, [lo, hi])


@pytest.mark.slow
def test_prefill_full_size_sampled():
    """N = 131,072 causal queries in one hybrid_attn_prefill call; sampled rows checked."""
    wl = workloads.prefill()
    N = wl.n0[0]
    d = wl.dims
    layer = csa.HybridLayer(gh.dims_of(d), [N])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths([N])
    q = torch.empty(N, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.empty(N, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(N, d.H_I, dtype=torch.float32, device="cuda")
    sdev.fill_queries(wl, 0, 0, N, q, qi, w)
    out = torch.empty(N, d.H, d.d, dtype=torch.float32, device="cuda")
    idx = torch.empty(N, d.k, dtype=torch.int32, device="cuda")
    ws = layer.prefill_workspace(N)
    layer.prefill(layer.prefill_args(q, qi, w, out, 0, N, compress=True, idx_out=idx), ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    rows = [0, 3, 4, 127, 128, 4095, 4096, 65535, 100000, N - 1]
    out_h = out[rows].cpu().numpy()
    idx_h = idx[rows].cpu().numpy()
    del q, out
    ref = gh.OracleSeq(wl, 0, N)
    for r_i, i in enumerate(rows):
        L = i + 1
        qh, qih, wh = (t[0] for t in workloads.queries(wl, 0, i, i + 1))
        r = ref.query(L, qh, qih, wh)
        slack = gh.score_slack(qih, wh, ref.KI[:L // d.m])
        gh.sets_explained(idx_h[r_i], r["idx"], r["scores"], slack)
        gh.check_close(out_h[r_i], r["O"], f"prefill row {i}")


@pytest.mark.slow
def test_prefill_select_when_the_sample_overestimates():
    """The prefill select estimates its threshold bin from a strided sample of each row (every 8th
    score at 32,768 entries).  Here only 300 entries score high and all of them sit at sampled
    positions, so the sample's estimate keeps fewer than k entries; the select must notice and keep
    the whole row, and still return the exact top-k.  Indexer keys are written directly into the
    cache (prefill with compress = 0) so that query q^I = e_0 on head 0 (weight 1, other heads 0)
    scores entry j as relu(K_j[0])."""
    N = 131072
    d = SMALL_PROD
    wl = workloads.Workload("prefill_sample_check", 4010, d, (N,), 0, mode="prefill")
    layer = csa.HybridLayer(gh.dims_of(d), [N])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths([N])
    layer.compress()
    E = N // d.m
    rng = np.random.default_rng(7)
    col0 = rng.permutation(E).astype(np.float64) / E * 0.5 + 0.25  # distinct values in [0.25, 0.75)
    high = np.arange(0, 8 * 300, 8)                                  # 300 sampled positions
    col0[high] = 10.0 + np.arange(300) / 300.0
    keys = np.zeros((E, d.d_I), dtype=np.float32)
    keys[:, 0] = col0
    keys_bf16 = torch.from_numpy(keys).to(torch.bfloat16)
    layer.entry_keys.copy_(keys_bf16.cuda())
    q0 = N - 4
    nq = 4
    q = torch.zeros(nq, d.H, d.d, dtype=torch.bfloat16, device="cuda")
    qi = torch.zeros(nq, d.H_I, d.d_I, dtype=torch.bfloat16, device="cuda")
    qi[:, 0, 0] = 1.0
    w = torch.zeros(nq, d.H_I, dtype=torch.float32, device="cuda")
    w[:, 0] = 1.0
    out = torch.empty(nq, d.H, d.d, dtype=torch.float32, device="cuda")
    idx = torch.empty(nq, d.k, dtype=torch.int32, device="cuda")
    ws = layer.prefill_workspace(N)
    # the call's query rows are positions q0 .. q0 + 3 (row r of q / qi / w is position q0 + r)
    layer.prefill(layer.prefill_args(q, qi, w, out, q0, N, compress=False, idx_out=idx), ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    kb = keys_bf16.view(torch.int16).numpy().view(np.uint16)
    qih = np.zeros((d.H_I, d.d_I), dtype=np.uint16)
    qih[0, 0] = 0x3F80  # bf16 1.0
    wh = np.array([1.0, 0.0, 0.0, 0.0], dtype=np.float32)
    got = idx.cpu().numpy()
    for r in range(nq):
        L = q0 + r + 1
        s = oracle.index_scores(qih, wh, kb[:L // d.m])
        want = oracle.topk(s, d.k)
        assert set(got[r].tolist()) == set(want.tolist()), f"row {r}"
        assert set(high.tolist()) <= set(got[r].tolist())
