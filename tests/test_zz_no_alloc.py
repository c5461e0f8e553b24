"""csa_index_topk_noalloc: the indexer top-k for callers that cannot pass device scratch memory
(for example code under a framework that owns every device buffer, or a serving loop that must not
allocate once running).  It must select exactly what csa_index_topk selects with a caller-provided
workspace, on two calls in a row (the built-in scratch keeps the previous call's contents), and
refuse sizes beyond its built-in limit with a clear error.

Kept in its own file, collected last, so that a failure here comes after every other test ran."""
import numpy as np
import pytest
import torch

import compressed_sparse_kv_overlapped_b200 as csa
import synth

pytestmark = pytest.mark.gpu


def _case(E_list, seed, k=1024, d_I=64, H_I=4):
    dims = csa.make_dims(d=512, H=64, d_I=d_I, H_I=H_I, m=4, m_hca=128, k=k, W=128)
    Q = len(E_list)
    keys = []
    for i, E in enumerate(E_list):
        keys.append(synth.bf16_normal(seed, synth.KI, i, d_I, 0, E, scale=0.5))
    offs = np.cumsum([0] + list(E_list))
    kd = torch.from_numpy(np.concatenate(keys).view(np.int16)).cuda().view(torch.bfloat16)
    seqs = torch.tensor([[0, offs[i], 0, 4 * E] for i, E in enumerate(E_list)], dtype=torch.int64, device="cuda")
    qt = torch.tensor([[i, 4 * E] for i, E in enumerate(E_list)], dtype=torch.int64, device="cuda")
    qi = torch.from_numpy(synth.bf16_normal(seed, synth.QI, 7, H_I * d_I, 0, Q).view(np.int16)).cuda()
    w = torch.from_numpy(synth.f32_uniform(seed, synth.W, 7, H_I, 0, Q)).cuda()
    return dims, Q, 4 * max(E_list), seqs, qt, qi, w, kd


def test_noalloc_matches_workspace_version_twice():
    dims, Q, max_len, seqs, qt, qi, w, keys = _case([200000, 5000, 1000, 70001], seed=515)
    ref_idx = torch.empty(Q, dims.k, dtype=torch.int32, device="cuda")
    ref_sc = torch.empty(Q, dims.k, dtype=torch.float32, device="cuda")
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, Q, max_len
    ws = torch.empty(csa.csa_workspace_size(csa.CSA_OP_INDEX_TOPK, wq), dtype=torch.uint8, device="cuda")
    csa.csa_index_topk(dims, seqs, qt, Q, max_len, qi, w, keys, ref_idx, ref_sc, ws)
    assert csa.csa_sync_status() == csa.CSA_OK
    for call in range(2):
        idx = torch.full((Q, dims.k), -9, dtype=torch.int32, device="cuda")
        sc = torch.full((Q, dims.k), -9.0, dtype=torch.float32, device="cuda")
        csa.csa_index_topk_noalloc(dims, seqs, qt, Q, max_len, qi, w, keys, idx, sc)
        assert csa.csa_sync_status() == csa.CSA_OK, f"call {call}"
        assert torch.equal(idx, ref_idx), f"call {call}: selected indices differ"
        # same kernels and keys: scores agree to the tests' score tolerance (exactly, in practice)
        np.testing.assert_allclose(sc.cpu().numpy(), ref_sc.cpu().numpy(), rtol=1e-5, atol=1e-5, equal_nan=True)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    dims, Q, max_len, seqs, qt, qi, w, keys = _case([4096, 4096], seed=9)
    idx = torch.empty(Q, dims.k, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError, match="exceed the built-in scratch"):
        csa.csa_index_topk_noalloc(dims, seqs, qt, Q, 4 * (1 << 20), qi, w, keys, idx, None)
    q17 = torch.zeros(17, 2, dtype=torch.int64, device="cuda")
    with pytest.raises(RuntimeError, match="exceed the built-in scratch"):
        csa.csa_index_topk_noalloc(dims, seqs, q17, 17, 4096, qi, w, keys, idx, None)
