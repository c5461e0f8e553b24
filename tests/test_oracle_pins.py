"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics (CPU only).

Each test pins one part of the oracle to something other than itself: a closed form, a special
case that reduces to a library routine (torch's fp64 softmax attention, numpy's sort), brute-force
enumeration, an invariant of the definition, or the counts the pages print.  A plausible slip in the
oracle (a dropped term, a wrong window offset or sign, a transposed operand, a wrong tie-break)
breaks at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SEED = 77


def bf(seed, tensor, seq, rows, cols, scale=1.0):
    return synth.bf16_normal(seed, tensor, seq, cols, 0, rows, scale=scale)


def f64(u16):
    return synth.bf16_to_f64(u16)


ONE_BF16 = np.uint16(0x3F80)


# ---------------------------------------------------------------- compressor (a1 / a2)

@pytest.mark.parametrize("m,win", [(4, 8), (16, 16), (128, 128), (4, 4)])
def test_equal_logits_give_window_mean(m, win):
    """Equal logits and an offset-independent bias make the softmax uniform: entry = window mean."""
    d, L = 16, 8 * m + 3
    x = bf(SEED, synth.X, 0, L, d)
    logit = np.full((L, d), np.uint16(0x4040), dtype=np.uint16)  # 3.0 everywhere
    colbias = synth.f32_normal(SEED, synth.BIAS_C, 0, d, 0, 1)
    bias = np.repeat(colbias, win, axis=0)  # same bias at every offset of a channel
    js = np.arange(L // m)
    E, _ = oracle.compress(x, logit, bias, None, L, m, win, js)
    xf = f64(x)
    for j in js:
        t0, t1 = max(0, m * j - (win - m)), m * j + m
        np.testing.assert_allclose(E[j], xf[t0:t1].mean(axis=0), rtol=1e-14, atol=1e-15)


def test_clipped_first_window_is_four_token_mean():
    """Entry 0 of the overlapping CSA window keeps only its 4 existing tokens [0, 4)."""
    d, L = 8, 16
    x = bf(SEED, synth.X, 1, L, d)
    logit = np.zeros((L, d), dtype=np.uint16)
    bias = np.zeros((8, d), dtype=np.float32)
    E, _ = oracle.compress(x, logit, bias, None, L, 4, 8, [0, 1])
    np.testing.assert_allclose(E[0], f64(x)[0:4].mean(0), rtol=1e-15)
    np.testing.assert_allclose(E[1], f64(x)[0:8].mean(0), rtol=1e-15)


@pytest.mark.parametrize("m,win", [(4, 8), (128, 128)])
def test_weights_sum_to_one_per_channel(m, win):
    d, L = 32, 3 * m + 1
    logit = bf(SEED, synth.A, 0, L, d)
    bias = synth.f32_normal(SEED, synth.BIAS_C, 0, d, 0, win, scale=0.5)
    js = np.arange(L // m)
    Wt = oracle.compress_weights(logit, bias, L, m, win, js)
    eps = win * np.finfo(np.float64).eps  # n-term summation bound
    np.testing.assert_allclose(Wt.sum(axis=1), 1.0, rtol=0, atol=eps)
    assert (Wt >= 0).all()
    # all-ones latent: the weighted sum reproduces the weight total, 1
    ones = np.full((L, d), ONE_BF16, dtype=np.uint16)
    E, KI = oracle.compress(ones, logit, bias, ones[:, :8], L, m, win, js)
    np.testing.assert_allclose(E, 1.0, rtol=0, atol=2 * eps)
    np.testing.assert_allclose(KI, 1.0, rtol=0, atol=2 * eps)


def test_two_token_window_is_logistic():
    """m=1 with an overlapping window of 2: weights are the logistic function of the logit gap."""
    d, L = 4, 6
    x = bf(SEED, synth.X, 2, L, d)
    logit = bf(SEED, synth.A, 2, L, d)
    bias = synth.f32_normal(SEED, synth.BIAS_C, 2, d, 0, 2, scale=0.5)
    E, _ = oracle.compress(x, logit, bias, None, L, 1, 2, np.arange(L))
    xf, lf, bb = f64(x), f64(logit), bias.astype(np.float64)
    for j in range(1, L):
        za = lf[j - 1] + bb[0]
        zb = lf[j] + bb[1]
        wb = np.array([1.0 / (1.0 + math.exp(float(a - b))) for a, b in zip(za, zb)])
        np.testing.assert_allclose(E[j], wb * xf[j] + (1 - wb) * xf[j - 1], rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(E[0], xf[0])  # clipped: only token 0 exists


def test_identity_at_m1():
    d, L = 16, 20
    x = bf(SEED, synth.X, 3, L, d)
    logit = bf(SEED, synth.A, 3, L, d)
    kI = bf(SEED, synth.KI, 3, L, 8)
    bias = synth.f32_normal(SEED, synth.BIAS_C, 3, d, 0, 1)
    E, KI = oracle.compress(x, logit, bias, kI, L, 1, 1, np.arange(L))
    np.testing.assert_array_equal(E, f64(x))
    np.testing.assert_array_equal(KI, f64(kI))


@pytest.mark.parametrize("offset", range(8))
def test_bias_offset_counts_from_unclipped_start(offset):
    """A dominant bias at one window offset selects token start_j + offset (start_j = 4j - 4)."""
    d, L = 8, 24
    x = bf(SEED, synth.X, 4, L, d)
    logit = np.zeros((L, d), dtype=np.uint16)
    bias = np.zeros((8, d), dtype=np.float32)
    bias[offset, :] = 200.0
    E, _ = oracle.compress(x, logit, bias, None, L, 4, 8, np.arange(L // 4))
    xf = f64(x)
    for j in range(L // 4):
        t = 4 * j - 4 + offset
        if t >= 0:
            np.testing.assert_allclose(E[j], xf[t], rtol=1e-15, atol=1e-60)
        else:  # the dominant token does not exist: the rest are equal-weighted
            np.testing.assert_allclose(E[j], xf[0:4].mean(0), rtol=1e-15)


@pytest.mark.parametrize("m,win", [(4, 8), (16, 16)])
def test_locality(m, win):
    """Changing token t changes only the entries whose window holds t."""
    d, L = 8, 12 * m
    x = bf(SEED, synth.X, 5, L, d)
    logit = bf(SEED, synth.A, 5, L, d)
    bias = synth.f32_normal(SEED, synth.BIAS_C, 5, d, 0, win, scale=0.5)
    js = np.arange(L // m)
    E0, _ = oracle.compress(x, logit, bias, None, L, m, win, js)
    t = 5 * m + 1
    x2, l2 = x.copy(), logit.copy()
    x2[t] ^= np.uint16(0x8000)  # flip signs of token t's latent
    l2[t] = np.uint16(0x4100)   # and change its logits
    E1, _ = oracle.compress(x2, l2, bias, None, L, m, win, js)
    changed = set(np.nonzero(np.any(E0 != E1, axis=1))[0].tolist())
    expect = {t // m, t // m + 1} if win == 2 * m else {t // m}
    assert changed == expect


@pytest.mark.parametrize("m,win", [(4, 8), (16, 16)])
def test_entry_at_completion_equals_full_pass(m, win):
    """An entry compressed the moment it completes, with only the tokens seen so far in existence
    (the decode append), equals the same entry of a pass over the whole sequence (the prefill)."""
    d, d_I, N = 8, 4, 9 * m
    x = bf(SEED, synth.X, 13, N, d)
    logit = bf(SEED, synth.A, 13, N, d)
    kI = bf(SEED, synth.KI, 13, N, d_I) if win == 2 * m else None
    bias = synth.f32_normal(SEED, synth.BIAS_C, 13, d, 0, win, scale=0.5)
    Ef, Kf = oracle.compress(x, logit, bias, kI, N, m, win, np.arange(N // m))
    for j in range(N // m):
        L = m * (j + 1)
        Ej, Kj = oracle.compress(x[:L].copy(), logit[:L].copy(), bias, None if kI is None else kI[:L].copy(), L, m,
                                 win, [j])
        np.testing.assert_array_equal(Ej[0], Ef[j])
        if kI is not None:
            np.testing.assert_array_equal(Kj[0], Kf[j])


@pytest.mark.parametrize("m,win,d_I,c,o", [(4, 8, 16, 0, 5), (4, 8, 16, 1, 2), (4, 8, 16, 9, 7),
                                            (4, 8, 16, 15, 4), (2, 4, 8, 7, 3), (4, 8, 8, 3, 6)])
def test_indexer_key_uses_its_own_channel_weights(m, win, d_I, c, o):
    """Indexer-key channel c is weighted by channel c's own softmax (channels 0..d_I-1 of the
    compressor).  Only channel c gets a dominant bias, at window offset o, so only channel c's weights
    pick one token (start_j + o) and every other channel's weights are uniform.  Then KI[j, c] must be
    that token's indexer key and every other key channel the window mean: a key channel weighted with
    another channel's weights (a shifted, reversed or tail-aligned channel index) gives a mean where a
    picked token belongs, or the reverse."""
    d, L = 24, 10 * m
    x = bf(SEED, synth.X, 15, L, d)
    kI = bf(SEED, synth.KI, 15, L, d_I)
    logit = np.zeros((L, d), dtype=np.uint16)
    bias = np.zeros((win, d), dtype=np.float32)
    bias[o, c] = 300.0
    E, KI = oracle.compress(x, logit, bias, kI, L, m, win, np.arange(L // m))
    xf, kf = f64(x), f64(kI)
    for j in range(1, L // m):  # j >= 1: the whole window exists
        start = m * j - (win - m)
        t = start + o
        mean_x, mean_k = xf[start:start + win].mean(0), kf[start:start + win].mean(0)
        for cc in range(d):
            want = xf[t, cc] if cc == c else mean_x[cc]
            np.testing.assert_allclose(E[j, cc], want, rtol=1e-14, atol=1e-15)
        for cc in range(d_I):
            want = kf[t, cc] if cc == c else mean_k[cc]
            np.testing.assert_allclose(KI[j, cc], want, rtol=1e-14, atol=1e-15, err_msg=f"entry {j} key channel {cc}")


def test_entry_existence_rule():
    x = np.zeros((10, 4), dtype=np.uint16)
    b = np.zeros((8, 4), dtype=np.float32)
    oracle.compress(x, x, b, None, 8, 4, 8, [1])
    with pytest.raises(ValueError):
        oracle.compress(x, x, b, None, 7, 4, 8, [1])  # entry 1 needs tokens up to 7


# ---------------------------------------------------------------- indexer (a3) and top-k (a4)

def test_index_score_one_hot():
    d_I, n = 16, 50
    KI = bf(SEED, synth.KI, 6, n, d_I)
    for h, c in [(0, 3), (2, 15), (3, 0)]:
        qI = np.zeros((4, d_I), dtype=np.uint16)
        qI[h, c] = ONE_BF16
        w = np.zeros(4, dtype=np.float32)
        w[h] = 0.75
        s = oracle.index_scores(qI, w, KI)
        np.testing.assert_array_equal(s, 0.75 * np.maximum(f64(KI)[:, c], 0.0))


def test_index_score_relu_split_matches_matmul():
    """relu(x) - relu(-x) = x: one head's score at q minus at -q is the plain dot product."""
    d_I, n = 64, 300
    KI = bf(SEED, synth.KI, 7, n, d_I)
    q = bf(SEED, synth.QI, 7, 1, d_I)
    qn = q ^ np.uint16(0x8000)
    qI = np.zeros((4, d_I), dtype=np.uint16)
    qI[1] = q[0]
    qIn = np.zeros((4, d_I), dtype=np.uint16)
    qIn[1] = qn[0]
    w = np.array([0, 1, 0, 0], dtype=np.float32)
    diff = oracle.index_scores(qI, w, KI) - oracle.index_scores(qIn, w, KI)
    ref = torch.from_numpy(f64(KI)) @ torch.from_numpy(f64(q)[0])
    np.testing.assert_allclose(diff, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_index_score_heads_add():
    d_I, n = 32, 100
    KI = bf(SEED, synth.KI, 8, n, d_I)
    qI = bf(SEED, synth.QI, 8, 4, d_I)
    w = synth.f32_uniform(SEED, synth.W, 8, 4, 0, 1)[0]
    total = oracle.index_scores(qI, w, KI)
    parts = 0
    for h in range(4):
        wh = np.zeros(4, np.float32)
        wh[h] = w[h]
        parts = parts + oracle.index_scores(qI, wh, KI)
    np.testing.assert_allclose(total, parts, rtol=1e-14)


def test_index_score_follows_entry_permutation():
    """Each entry's score depends on that entry's key alone: permuting the keys permutes the scores."""
    d_I, n = 32, 77
    KI = bf(SEED, synth.KI, 14, n, d_I)
    qI = bf(SEED, synth.QI, 14, 4, d_I)
    w = synth.f32_uniform(SEED, synth.W, 14, 4, 0, 1)[0]
    perm = np.random.default_rng(3).permutation(n)
    np.testing.assert_array_equal(oracle.index_scores(qI, w, KI[perm].copy()), oracle.index_scores(qI, w, KI)[perm])


def brute_topk(s, k):
    n = len(s)
    keep = min(n, k)
    for S in itertools.combinations(range(n), keep):
        Sset = set(S)
        ok = all((s[i] > s[j]) or (s[i] == s[j] and i < j) for i in S for j in range(n) if j not in Sset)
        if ok:
            return list(S) + [-1] * (k - keep)
    raise AssertionError("no valid selection")


@pytest.mark.parametrize("trial", range(30))
def test_topk_brute_force(trial):
    rng = np.random.default_rng(trial)
    n = int(rng.integers(0, 10))
    k = int(rng.integers(1, 6))
    s = rng.integers(0, 4, size=n).astype(np.float64)  # many ties on purpose
    assert oracle.topk(s, k).tolist() == brute_topk(s.tolist(), k)


def test_topk_matches_library_sort():
    rng = np.random.default_rng(5)
    s = np.round(rng.standard_normal(20000), 2)  # ties
    k = 1024
    order = np.lexsort((np.arange(len(s)), -s))  # score desc, index asc
    np.testing.assert_array_equal(oracle.topk(s, k), np.sort(order[:k]))
    short = s[:100]
    out = oracle.topk(short, k)
    assert (out[:100] == np.arange(100)).all() and (out[100:] == -1).all()


# ---------------------------------------------------------------- attention (a5 / a6 / a7)

def sdpa64(qf, kf, scale, causal_rows=None):
    """torch fp64 softmax attention; qf [H,d] for one query, kf [n,d] keys=values."""
    q = torch.from_numpy(qf)[None, :, None, :]          # [1,H,1,d]
    k = torch.from_numpy(kf)[None, None, :, :].expand(1, qf.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, k, scale=scale)
    lse = torch.logsumexp(scale * (torch.from_numpy(qf) @ torch.from_numpy(kf).T), dim=-1)
    return o[0, :, 0, :].numpy(), lse.numpy()


def test_csa_dense_special_case_matches_library():
    """m=1, k >= L, W=0: the CSA partial is dense softmax attention over all L tokens."""
    H, d, L = 4, 32, 57
    x = bf(SEED, synth.X, 9, L, d)
    q = bf(SEED, synth.Q, 9, H, d)
    idx = np.arange(L, dtype=np.int32)
    O, lse = oracle.csa_attn(q, x, idx, 1, x, L, 0, 1 / math.sqrt(d))
    Oref, lref = sdpa64(f64(q), f64(x), 1 / math.sqrt(d))
    np.testing.assert_allclose(O, Oref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lref, rtol=1e-13)


def test_full_pipeline_m1_is_dense_causal_attention():
    """Compressor at m=1 (identity), k >= N, W=0 for CSA, and HCA at m'=1 each reduce to dense
    causal attention; checked for every query position against torch's causal fp64 softmax."""
    H, d, N, d_I = 2, 16, 24, 8
    x = bf(SEED, synth.X, 10, N, d)
    logit = bf(SEED, synth.A, 10, N, d)
    kI = bf(SEED, synth.KI, 10, N, d_I)
    bias = np.zeros((1, d), np.float32)
    E, KI = oracle.compress(x, logit, bias, kI, N, 1, 1, np.arange(N))
    Eb, KIb = oracle.round_bf16(E), oracle.round_bf16(KI)
    qs = bf(SEED, synth.Q, 10, N * H, d).reshape(N, H, d)
    qI = bf(SEED, synth.QI, 10, N * 4, d_I).reshape(N, 4, d_I)
    w = synth.f32_uniform(SEED, synth.W, 10, 4, 0, N)
    scale = 1 / math.sqrt(d)
    qt = torch.from_numpy(f64(qs)).permute(1, 0, 2)[None]          # [1,H,N,d]
    kt = torch.from_numpy(f64(x))[None, None].expand(1, H, N, d)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, is_causal=True, scale=scale)[0]
    for i in range(N):
        L = i + 1
        s = oracle.index_scores(qI[i], w[i], KIb[:L])
        idx = oracle.topk(s, N + 5)
        O_c, _ = oracle.csa_attn(qs[i], Eb, idx, 1, x, L, 0, scale)
        O_h, _ = oracle.hca_attn(qs[i], Eb, 1, x, L, 0, scale)
        np.testing.assert_allclose(O_c, ref[:, i, :].numpy(), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(O_h, ref[:, i, :].numpy(), rtol=1e-12, atol=1e-13)


def test_single_key_returns_it():
    H, d = 3, 16
    x = bf(SEED, synth.X, 11, 8, d)
    q = bf(SEED, synth.Q, 11, H, d)
    O, lse = oracle.csa_attn(q, x, np.array([-1, -1], np.int32), 4, x, 1, 1, 0.25)  # window = token 0
    np.testing.assert_array_equal(O, np.repeat(f64(x)[0:1], H, axis=0))
    np.testing.assert_allclose(lse, 0.25 * f64(q) @ f64(x)[0], rtol=1e-14)


def test_key_permutation_invariance():
    H, d, n = 4, 32, 40
    E = bf(SEED, synth.X, 12, n, d)
    q = bf(SEED, synth.Q, 12, H, d)
    idx = np.arange(0, n, 2, dtype=np.int32)
    perm = np.random.default_rng(1).permutation(idx).astype(np.int32)
    O1, l1 = oracle.csa_attn(q, E, idx, 1, E, n, 5, 0.2)
    O2, l2 = oracle.csa_attn(q, E, perm, 1, E, n, 5, 0.2)
    np.testing.assert_allclose(O1, O2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-14)


def test_lse_merge_of_a_partition_equals_one_softmax():
    H, d, n = 4, 32, 64
    E = bf(SEED, synth.X, 13, n, d)
    q = bf(SEED, synth.Q, 13, H, d, scale=3.0)
    rng = np.random.default_rng(3)
    mask = rng.random(n) < 0.4
    A = np.nonzero(mask)[0].astype(np.int32)
    Bp = np.nonzero(~mask)[0].astype(np.int32)
    Oa, la = oracle.csa_attn(q, E, A, 1, E, n, 0, 0.2)
    Ob, lb = oracle.csa_attn(q, E, Bp, 1, E, n, 0, 0.2)
    Oall, lall = oracle.csa_attn(q, E, np.arange(n, dtype=np.int32), 1, E, n, 0, 0.2)
    O, l = oracle.lse_merge(Oa, la, Ob, lb)
    np.testing.assert_allclose(O, Oall, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l, lall, rtol=1e-13)
    Oe, le = oracle.csa_attn(q, E, np.array([-1], np.int32), 1, E, n, 0, 0.2)   # empty partial
    assert np.isneginf(le).all() and (Oe == 0).all()
    O2, l2 = oracle.lse_merge(Oall, lall, Oe, le)
    np.testing.assert_array_equal(O2, Oall)


def test_noncausal_index_rejected():
    E = np.zeros((8, 4), np.uint16)
    q = np.zeros((1, 4), np.uint16)
    with pytest.raises(ValueError):
        oracle.csa_attn(q, E, np.array([2], np.int32), 4, E, 8, 0, 1.0)  # L=8 -> entries 0,1 only


@pytest.mark.parametrize("L", [1, 3, 9, 15, 16, 17, 40, 63, 64, 200, 777])
def test_hybrid_query_composition_at_zero_query(L):
    """The composed query at q = 0 and q^I = 0: every logit and every indexer score is 0, so the
    top-k keeps entries 0..min(k, L/m)-1 (ties to the lower index) and the merged softmax is
    uniform over exactly those entries, the raw window counted once and every visible HCA entry:
    lse = log(min(k, floor(L/m)) + min(W, L) + floor(L/m')) and O is the plain mean of those keys.
    A window counted twice, an HCA partial taken with the window, or a wrong visibility rule
    changes the count."""
    sh = oracle.Shape(d=16, H=2, d_I=8, H_I=4, m=4, m_hca=16, k=5, W=8)
    raw = bf(SEED, synth.X, 16, L, sh.d)
    n_c, n_h = L // sh.m, L // sh.m_hca
    entries = bf(SEED, synth.A, 16, max(n_c, 1), sh.d)
    KI = bf(SEED, synth.KI, 16, max(n_c, 1), sh.d_I)
    hca = bf(SEED, synth.B, 16, max(n_h, 1), sh.d)
    q = np.zeros((sh.H, sh.d), np.uint16)
    qI = np.zeros((sh.H_I, sh.d_I), np.uint16)
    w = np.full(sh.H_I, 0.5, np.float32)
    r = oracle.hybrid_query(sh, L, q, qI, w, raw, entries, KI, hca)
    n_sel, n_win = min(sh.k, n_c), min(sh.W, L)
    count = n_sel + n_win + n_h
    np.testing.assert_allclose(r["lse"], math.log(count), rtol=1e-14)
    assert r["idx"][:n_sel].tolist() == list(range(n_sel))
    assert (r["idx"][n_sel:] == -1).all()
    keys = np.concatenate([f64(entries)[:n_sel], f64(raw)[L - n_win:L], f64(hca)[:n_h]])
    np.testing.assert_allclose(r["O"], np.repeat(keys.mean(0)[None], sh.H, axis=0), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- the pages' printed counts

def test_page_counts_one_million_tokens():
    """1M tokens: 250,000 CSA entries, ~7,800 HCA entries, ~1,100 attended positions (~900x).

    The attended-position count is read off the oracle itself: with q = 0 every logit is 0, so the
    softmax is uniform and lse = log(number of keys)."""
    g = json.load(open(os.path.join(GOLDEN, "page_counts.json")))
    N, m, mh, k, W = g["tokens"], g["m"], g["m_hca"], g["k"], g["W"]
    d = 4
    tol = g["approx_rel_tol"]
    assert N // m == g["csa_entries"]
    assert abs(N // mh - g["hca_entries_approx"]) <= tol * g["hca_entries_approx"]
    raw = np.zeros((N, d), np.uint16)
    entries = np.zeros((N // m, d), np.uint16)
    s = np.random.default_rng(0).random(N // m)
    idx = oracle.topk(s, k)
    q = np.zeros((1, d), np.uint16)
    _, lse = oracle.csa_attn(q, entries, idx, m, raw, N, W, 0.5)
    n_keys = round(math.exp(lse[0]))
    assert n_keys == k + W
    assert abs(n_keys - g["positions_approx"]) <= tol * g["positions_approx"]
    assert abs(N / n_keys - g["reduction_approx"]) <= tol * g["reduction_approx"]
    hca = np.zeros((N // mh, d), np.uint16)
    _, lse_h = oracle.hca_attn(q, hca, mh, raw, N, 0, 0.5)
    assert round(math.exp(lse_h[0])) == N // mh


def test_two_pow_20_counts():
    assert (1 << 20) // 4 == 262144 and (1 << 20) // 128 == 8192


# ---------------------------------------------------------------- bf16 rounding of stored caches

def test_oracle_bf16_rounding_matches_library_on_float32_values():
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-30, 30, 200000),
                        [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0, 3.0e38]])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.round_bf16(v32.astype(np.float64)), ref)


def test_oracle_bf16_rounding_matches_generator_on_doubles():
    """Two independent direct double->bf16 roundings (the oracle's and the input generator's)."""
    rng = np.random.default_rng(12)
    v = rng.standard_normal(20000) * 10.0 ** rng.integers(-20, 20, 20000)
    lib = synth.host_lib()
    gen = np.array([lib.synth_bf16_host(float(a)) for a in v], dtype=np.uint16)
    np.testing.assert_array_equal(oracle.round_bf16(v), gen)


# ---------------------------------------------------------------- 8-bit block-scaled indexer keys

def test_e4m3_rounding_matches_library():
    """The oracle's nearest-even rounding onto the FP8 E4M3 grid equals torch's float32 -> float8_e4m3fn
    conversion on float32 values in [-448, 448], subnormals and exact ties included."""
    rng = np.random.default_rng(21)
    v = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000) * 2.0 ** rng.integers(-12, 8, 20000),
                        np.arange(-64, 65) * 2.0 ** -10,  # ties on the subnormal grid (steps of 2^-9)
                        [1.0625, 1.1875, -3.125, 448.0, -448.0, 0.0, 2.0 ** -6, 2.0 ** -9]]).astype(np.float32)
    v = v[np.abs(v) <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_round(v.astype(np.float64)), ref)


def test_e4m3_values_match_library():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)  # every code but NaN
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.e4m3_value(codes), ref)


@pytest.mark.parametrize("scale", [1.0, 2.0 ** -20, 3.0e4])
def test_mx8_block_scale_is_the_smallest_power_of_two(scale):
    """Each block's scale 2^e is the smallest power of two with amax <= 448 * 2^e, so the largest
    magnitude lands in (224, 448]; every element is x / 2^e rounded on the E4M3 grid, so the
    dequantized key is within half an E4M3 step (relative 2^-4 for normal values) of x."""
    n, d_I = 300, 64
    K = oracle.round_bf16(synth.bf16_to_f64(bf(SEED, synth.KI, 17, n, d_I)) * scale)
    K[5] = 0  # an all-zero entry: scale byte 0, zero elements
    Kq, sc = oracle.quantize_keys_mx8(K)
    Kf = synth.bf16_to_f64(K)
    for j in range(n):
        for b in range(d_I // 32):
            x = Kf[j, 32 * b:32 * b + 32]
            e = int(sc[j, b]) - 127
            amax = np.abs(x).max()
            if amax == 0:
                assert e == -127 and (Kq[j, 32 * b:32 * b + 32] & 0x7F == 0).all()
                continue
            assert 224 < amax / 2.0 ** e <= 448
            np.testing.assert_array_equal(Kq[j, 32 * b:32 * b + 32], oracle.e4m3_round(x / 2.0 ** e))
            deq = oracle.e4m3_value(Kq[j, 32 * b:32 * b + 32]) * 2.0 ** e
            bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** (e - 10))
            assert (np.abs(deq - x) <= bound).all()


def test_mx8_scores_are_the_plain_scores_of_the_dequantized_keys():
    """The 8-bit scorer equals the bf16 scorer applied to the dequantized keys (which bf16 holds
    exactly: 4 significant bits times a power of two)."""
    n, d_I = 500, 64
    K = bf(SEED, synth.KI, 18, n, d_I)
    qI = bf(SEED, synth.QI, 18, 4, d_I)
    w = synth.f32_uniform(SEED, synth.W, 18, 4, 0, 1)[0]
    Kq, sc = oracle.quantize_keys_mx8(K)
    deq = oracle.e4m3_value(Kq) * np.repeat(2.0 ** (sc.astype(np.float64) - 127), 32, axis=1)
    Kd = oracle.round_bf16(deq)
    np.testing.assert_array_equal(synth.bf16_to_f64(Kd), deq)
    np.testing.assert_array_equal(oracle.index_scores_mx8(qI, w, Kq, sc), oracle.index_scores(qI, w, Kd))


# ---------------------------------------------------------------- FP4 entries (R15)

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # the magnitudes of codes 0..7 (sign bit 3)


def test_e2m1_grid_midpoints_and_saturation():
    """Every E2M1 value maps to its own code, a midpoint to the neighbour whose mantissa bit (code
    bit 0) is 0, anything just past a midpoint to the upper neighbour, magnitudes above 6 to 6, and
    a negative value keeps its sign bit even when it rounds to zero."""
    vals, want = [], []
    for c, g in enumerate(E2M1):
        vals += [g, -g]
        want += [c, (8 | c) if g > 0 else 8]
    for i in range(7):
        lo, hi = E2M1[i], E2M1[i + 1]
        mid = (lo + hi) / 2
        vals += [mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf)]
        want += [i if i % 2 == 0 else i + 1, i + 1, i]
    vals += [6.5, 7.0, 1e30, -100.0, -0.1, -0.25]
    want += [7, 7, 7, 15, 8, 8]
    np.testing.assert_array_equal(oracle.e2m1_code(np.array(vals)), np.array(want, dtype=np.uint8))


@pytest.mark.parametrize("scale", [1.0, 2.0 ** -30, 5.0e3])
def test_mx4_block_scale_and_nearest_value(scale):
    """Each 32-channel block's scale 2^e is the smallest power of two with amax <= 6 * 2^e (so
    3 < amax / 2^e <= 6), and every element dequantizes to a nearest point of the grid scaled by
    2^e (brute force over the 8 magnitudes and both signs)."""
    n, d = 60, 128
    E = oracle.round_bf16(synth.bf16_to_f64(bf(SEED, synth.X, 31, n, d)) * scale)
    E[7] = 0  # an all-zero entry: scale byte 0, zero codes
    Eq, sc = oracle.quantize_entries_mx4(E)
    deq = oracle.dequantize_entries_mx4(Eq, sc)
    Ef = synth.bf16_to_f64(E)
    grid = np.array(E2M1 + [-g for g in E2M1])
    for j in range(n):
        for b in range(d // 32):
            x = Ef[j, 32 * b:32 * b + 32]
            e = int(sc[j, b]) - 127
            amax = np.abs(x).max()
            if amax == 0:
                assert e == -127 and not deq[j, 32 * b:32 * b + 32].any()
                continue
            assert 3 < amax / 2.0 ** e <= 6
            dist = np.abs(grid[None, :] * 2.0 ** e - x[:, None]).min(axis=1)
            np.testing.assert_array_equal(np.abs(deq[j, 32 * b:32 * b + 32] - x), dist)


def test_mx4_round_trip_and_nibble_order():
    """Rows whose blocks hold only grid values times 2^e, with 6 * 2^e present, come back exactly;
    the even channel sits in the low nibble of each byte."""
    rng = np.random.default_rng(5)
    n, d = 8, 64
    rows = np.empty((n, d))
    for j in range(n):
        for b in range(d // 32):
            e = int(rng.integers(-20, 20))
            blk = rng.choice(E2M1, size=32) * rng.choice([-1.0, 1.0], size=32)
            blk[int(rng.integers(0, 32))] = 6.0
            rows[j, 32 * b:32 * b + 32] = blk * 2.0 ** e
    E = oracle.round_bf16(rows)
    assert np.array_equal(synth.bf16_to_f64(E), rows)
    Eq, sc = oracle.quantize_entries_mx4(E)
    np.testing.assert_array_equal(oracle.dequantize_entries_mx4(Eq, sc), rows)
    row = np.zeros((1, 32))
    row[0, 0], row[0, 1], row[0, 2], row[0, 3] = 0.5, 6.0, -1.5, 0.0
    Eq, sc = oracle.quantize_entries_mx4(oracle.round_bf16(row))
    assert sc[0, 0] == 127 and Eq[0, 0] == (1 | (7 << 4)) and Eq[0, 1] == (8 | 3)


# ---------------------------------------------------------------- sinks and normalization

def test_rms_norm_matches_library_and_closed_forms():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((50, 64)) * rng.uniform(0.01, 100, (50, 1))
    g = synth.f32_normal(SEED, synth.BIAS_C, 31, 64, 0, 1)[0]
    eps = 1e-6
    out = oracle.rms_norm(x, g, eps)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(g.astype(np.float64)), eps)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-13, atol=1e-15)
    ones = np.ones(64, np.float32)
    y = oracle.rms_norm(x, ones, 0.0)
    np.testing.assert_allclose((y ** 2).mean(axis=1), 1.0, rtol=1e-13)           # unit RMS
    np.testing.assert_allclose(oracle.rms_norm(7.5 * x, ones, 0.0), y, rtol=1e-13)  # scale invariant
    c = np.full((1, 64), 3.0)
    np.testing.assert_allclose(oracle.rms_norm(c, g, 0.5), 3.0 / math.sqrt(9.5) * g[None].astype(np.float64),
                               rtol=1e-14)


@pytest.mark.parametrize("L", [9, 40, 200])
def test_sink_at_zero_query_and_vanishing_sink(L):
    """The sink is one more softmax term with a zero value: at q = 0 every key has logit 0, so with n
    keys lse = log(n + e^z) and O = (n / (n + e^z)) * mean of the keys; a sink of -inf changes nothing."""
    sh = oracle.Shape(d=16, H=2, d_I=8, H_I=4, m=4, m_hca=16, k=5, W=8)
    raw = bf(SEED, synth.X, 19, L, sh.d)
    entries = bf(SEED, synth.A, 19, max(L // sh.m, 1), sh.d)
    KI = bf(SEED, synth.KI, 19, max(L // sh.m, 1), sh.d_I)
    hca = bf(SEED, synth.B, 19, max(L // sh.m_hca, 1), sh.d)
    q = np.zeros((sh.H, sh.d), np.uint16)
    qI = np.zeros((sh.H_I, sh.d_I), np.uint16)
    w = np.full(sh.H_I, 0.5, np.float32)
    z = np.array([0.7, -2.0])
    base = oracle.hybrid_query(sh, L, q, qI, w, raw, entries, KI, hca)
    r = oracle.hybrid_query(sh, L, q, qI, w, raw, entries, KI, hca, sink=z)
    n = min(sh.k, L // sh.m) + min(sh.W, L) + L // sh.m_hca
    np.testing.assert_allclose(r["lse"], np.log(n + np.exp(z)), rtol=1e-14)
    np.testing.assert_allclose(r["O"], base["O"] * (n / (n + np.exp(z)))[:, None], rtol=1e-13, atol=1e-15)
    q2 = bf(SEED, synth.Q, 19, sh.H, sh.d)
    a = oracle.hybrid_query(sh, L, q2, qI, w, raw, entries, KI, hca)
    b = oracle.hybrid_query(sh, L, q2, qI, w, raw, entries, KI, hca, sink=np.full(sh.H, -np.inf))
    np.testing.assert_array_equal(a["O"], b["O"])
    np.testing.assert_array_equal(a["lse"], b["lse"])
