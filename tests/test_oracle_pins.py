"""Pins for the float64 oracle: checks against what the pages and mathematics fix, never
against the oracle itself.  CPU only.

Sources: xllm-io paper review of DashAttention, section 3 (background alpha-entmax formula,
Eq. 4, Eq. 6, Eq. 9, Eq. 11-12, Proposition 4.1) and section 6.5 (DA+FA: full softmax is a
special case); gist.science technical summary, "Methodology".
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.optimize import brentq

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- entmax
def sparsemax_sorted(s):
    """Textbook sort-based sparsemax (Martins & Astudillo, 2016)."""
    z = np.sort(s)[::-1]
    cs = np.cumsum(z)
    k = np.arange(1, len(s) + 1)
    ok = 1 + k * z > cs
    kmax = k[ok][-1]
    tau = (cs[kmax - 1] - 1) / kmax
    return np.maximum(s - tau, 0)


def entmax_bruteforce(s, alpha):
    """Enumerate the support sizes k of the sorted scores; for each, find the root of
    sum_{j<=k} (x_j - t)^{1/(alpha-1)} = 1 with brentq and keep the k whose root is consistent
    (x_(k) > t >= x_(k+1))."""
    x = (alpha - 1) * np.asarray(s, dtype=np.float64)
    xs = np.sort(x)[::-1]
    p = 1 / (alpha - 1)
    for k in range(1, len(x) + 1):
        f = lambda t: np.sum((xs[:k] - t) ** p) - 1
        hi = xs[k - 1]
        lo = xs[0] - 1
        if f(lo) < -1e-12 or f(hi) > 0:
            continue
        t = lo if f(lo) <= 0 else brentq(f, lo, hi, xtol=1e-15, rtol=1e-15, maxiter=500)
        nxt = xs[k] if k < len(x) else -np.inf
        if t >= nxt - 1e-13 and t < xs[k - 1]:
            return np.maximum(x - t, 0) ** p
    raise AssertionError("no consistent support")


def _golden_cases():
    out = []
    with open(os.path.join(GOLDEN, "entmax_closed_forms.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            a, s, p, _ = [f.strip() for f in line.split("|")]
            ev = lambda e: float(eval(e, {"__builtins__": {}}, {"sqrt": math.sqrt}))
            out.append((float(a), [ev(v) for v in s.split(",")], [ev(v) for v in p.split(",")]))
    return out


@pytest.mark.parametrize("alpha,s,expect", _golden_cases())
def test_entmax_golden_closed_forms(alpha, s, expect):
    p = oracle.entmax(s, alpha)
    np.testing.assert_allclose(p, expect, rtol=0, atol=1e-13)
    for pi, ei in zip(p, expect):
        if ei == 0:
            assert pi == 0.0  # exact zeros where (alpha-1)s <= tau


@pytest.mark.parametrize("n", [1, 2, 5, 31, 64, 257, 1000])
def test_alpha2_is_sparsemax(n):
    rng = np.random.default_rng(n)
    for scale in (0.1, 1.0, 10.0):
        s = rng.standard_normal(n) * scale
        np.testing.assert_allclose(oracle.entmax(s, 2.0), sparsemax_sorted(s), atol=1e-13)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 1.75, 2.0])
@pytest.mark.parametrize("n", [1, 3, 7, 12])
def test_entmax_bruteforce_tau(alpha, n):
    rng = np.random.default_rng(100 + n)
    for _ in range(20):
        s = rng.standard_normal(n) * rng.choice([0.3, 1.0, 4.0])
        np.testing.assert_allclose(oracle.entmax(s, alpha), entmax_bruteforce(s, alpha), atol=1e-11)


@pytest.mark.parametrize("alpha", [1.1, 1.25, 1.5, 1.9, 2.0])
def test_entmax_simplex_and_exact_zeros(alpha):
    rng = np.random.default_rng(7)
    for n in (4, 50, 511, 2047):
        s = rng.standard_normal(n) * 3
        p = oracle.entmax(s, alpha)
        assert abs(p.sum() - 1) < 1e-12
        tau = oracle.entmax_threshold((alpha - 1) * s, alpha)
        off = (alpha - 1) * s <= tau
        assert np.all(p[off] == 0.0)
        assert np.all(p[~off] > 0.0)
        # translation invariance
        np.testing.assert_allclose(oracle.entmax(s + 3.7, alpha), p, atol=1e-10)


def test_entmax_tends_to_softmax():
    rng = np.random.default_rng(3)
    s = rng.standard_normal(40)
    sm = np.exp(s - s.max())
    sm /= sm.sum()
    errs = [np.abs(oracle.entmax(s, 1 + e) - sm).max() for e in (1e-1, 1e-2, 1e-3)]
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 2e-3


def test_entmax_temperature_limits():
    rng = np.random.default_rng(4)
    s = rng.standard_normal(30)
    np.testing.assert_allclose(oracle.entmax(s * 1e-9, 1.5), np.full(30, 1 / 30), atol=1e-6)
    p = oracle.entmax(s * 1e3, 1.5)
    assert p[np.argmax(s)] == 1.0 and np.count_nonzero(p) == 1


# ----------------------------------------------------------------------------- Stage 0 (Eq. 4)
def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


def test_stage0_zero_query_is_mean_pooling():
    K = _rand((2, 256, 3, 32), 1)
    kbar = oracle.stage0(K, np.zeros((3, 32), np.float32), 64)
    ref = K.astype(np.float64).reshape(2, 4, 64, 3, 32).mean(axis=2).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(kbar, ref, atol=1e-12)


def test_stage0_chunk_one_is_identity():
    K = _rand((1, 40, 2, 16), 2)
    kbar = oracle.stage0(K, _rand((2, 16), 3), 1)
    np.testing.assert_allclose(kbar, K.transpose(0, 2, 1, 3), atol=0)


def test_stage0_weights_closed_form():
    """Chunk of 4 keys: e0 three times and e1 once; qbar = 4 log2 e0 with d = 16 makes the
    logits <qbar,k>/sqrt(d) equal log 2 and 0, so the weights are 2:2:2:1 and
    kbar = (6 e0 + e1)/7.  A missing or extra 1/sqrt(d) changes the answer."""
    d = 16
    K = np.zeros((1, 4, 1, d), np.float32)
    K[0, :3, 0, 0] = 1
    K[0, 3, 0, 1] = 1
    qbar = np.zeros((1, d), np.float32)
    qbar[0, 0] = 4 * math.log(2)
    kbar = oracle.stage0(K, qbar, 4)[0, 0, 0]
    expect = np.zeros(d)
    expect[0], expect[1] = 6 / 7, 1 / 7
    np.testing.assert_allclose(kbar, expect, atol=1e-6)


def test_chunk_summary_matches_stage0_and_partial():
    K = _rand((1, 128, 2, 32), 5)
    qb = _rand((2, 32), 6, 0.3)
    kbar = oracle.stage0(K, qb, 32)
    np.testing.assert_allclose(oracle.chunk_summary(K, qb, 0, 1, 64, 96), kbar[0, 1, 2], atol=1e-14)
    one = oracle.chunk_summary(K, qb, 0, 0, 70, 71)
    np.testing.assert_allclose(one, K[0, 70, 0], atol=1e-7)


# ----------------------------------------------------------------------------- Stage 1 (Eq. 6)
def test_route_alpha2_union_matches_sparsemax_per_head():
    """alpha = 2: each head's routing is the textbook sparsemax of gamma*zbar; the group weights
    are their mean and the routed set is the union of the head supports (Eq. 6 + GQA text)."""
    b, n, hq, hkv, d, B, gamma = 1, 384, 4, 2, 32, 32, 6.0
    Q, K, V = _rand((b, n, hq, d), 10), _rand((b, n, hkv, d), 11), _rand((b, n, hkv, d), 12)
    qb = _rand((hkv, d), 13, 0.2)
    pos = np.array([31, 32, 33, 100, 200, 383])
    O, kbar, rt = oracle.prefill(Q, K, V, qb, chunk=B, alpha=2.0, gamma=gamma, positions=pos,
                                 want_route=True)
    g = hq // hkv
    for t, i in enumerate(pos):
        nvis = i // B
        for r in range(hkv):
            if nvis == 0:
                assert rt["counts"][0, r, t] == 0
                continue
            zbar = Q[0, i, r * g:(r + 1) * g].astype(np.float64) @ kbar[0, r, :nvis].T / math.sqrt(d)
            heads = np.stack([sparsemax_sorted(gamma * z) for z in zbar])
            w = heads.mean(0)
            np.testing.assert_allclose(rt["w"][0, r, t, :nvis], w, atol=1e-12)
            union = (heads > 0).any(0)
            assert np.array_equal(rt["w"][0, r, t, :nvis] > 0, union)
            assert rt["counts"][0, r, t] == union.sum()
            assert np.array_equal(rt["margin"][0, r, t, :nvis] > 0, union)
            lw = np.log(w[union])
            np.testing.assert_allclose(rt["bias"][0, r, t, :nvis][union], lw - lw.mean(), atol=1e-10)


def test_route_gamma_zero_is_uniform_and_unbiased():
    Q, K, V = _rand((1, 200, 2, 16), 20), _rand((1, 200, 1, 16), 21), _rand((1, 200, 1, 16), 22)
    O, kbar, rt = oracle.prefill(Q, K, V, _rand((1, 16), 23), chunk=16, alpha=1.5, gamma=0.0,
                                 want_route=True)
    for i in (16, 17, 100, 199):
        nvis = i // 16
        assert rt["counts"][0, 0, i] == nvis
        np.testing.assert_allclose(rt["w"][0, 0, i, :nvis], 1 / nvis, atol=1e-13)
        np.testing.assert_allclose(rt["bias"][0, 0, i, :nvis], 0, atol=1e-12)


# ----------------------------------------------------------------------------- Stage 2
def _sdpa(Q, K, V, mask):
    """torch reference: softmax(QK^T/sqrt(d) + mask) V per head, float64, GQA by head//g."""
    b, n, hq, d = Q.shape
    g = hq // K.shape[2]
    q = torch.from_numpy(Q.astype(np.float64)).permute(0, 2, 1, 3)
    k = torch.from_numpy(K.astype(np.float64)).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    v = torch.from_numpy(V.astype(np.float64)).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("n,hq,hkv,d,B", [(200, 2, 1, 16, 16), (257, 4, 2, 32, 32),
                                          (96, 8, 2, 8, 1), (130, 4, 4, 16, 64)])
@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_gamma_zero_full_routing_is_dense_causal_attention(n, hq, hkv, d, B, alpha):
    """gamma = 0 makes every visible chunk's weight equal, so all are routed with zero bias and
    Stage 2 must reduce to dense causal softmax attention (the DA+FA special case of section
    6.5), for any sigma."""
    Q, K, V = _rand((2, n, hq, d), 30), _rand((2, n, hkv, d), 31), _rand((2, n, hkv, d), 32)
    mask = torch.ones(n, n, dtype=torch.bool).tril()
    ref = _sdpa(Q, K, V, mask)
    for inv_sigma in (1.0, 0.3):
        O, _ = oracle.prefill(Q, K, V, _rand((hkv, d), 33), chunk=B, alpha=alpha, gamma=0.0,
                              inv_sigma=inv_sigma)
        np.testing.assert_allclose(O, ref, atol=1e-12)


def _route_mask(rt, n, B, r, b=0):
    m = torch.zeros(n, n, dtype=torch.bool)
    for i in range(n):
        m[i, (i // B) * B:i + 1] = True
        for c in np.nonzero(rt["w"][b, r, i] > 0)[0]:
            m[i, c * B:(c + 1) * B] = True
    return m


def test_infinite_sigma_is_softmax_restricted_to_routed_and_diagonal():
    """sigma -> infinity (inv_sigma = 0) removes the prior: Stage 2 is a plain softmax over the
    routed tokens and the diagonal branch (Eq. 11 discussion)."""
    n, hq, hkv, d, B = 192, 4, 2, 16, 16
    Q, K, V = _rand((1, n, hq, d), 40), _rand((1, n, hkv, d), 41), _rand((1, n, hkv, d), 42)
    O, _, rt = oracle.prefill(Q, K, V, _rand((hkv, d), 43), chunk=B, alpha=1.5, gamma=8.0,
                              inv_sigma=0.0, want_route=True)
    frac = rt["counts"][0, :, B:].sum() / sum(i // B for i in range(B, n)) / hkv
    assert 0.05 < frac < 0.95  # routing is genuinely sparse here
    g = hq // hkv
    for r in range(hkv):
        ref = _sdpa(Q[:, :, r * g:(r + 1) * g], K[:, :, r:r + 1], V[:, :, r:r + 1],
                    _route_mask(rt, n, B, r))
        np.testing.assert_allclose(O[:, :, r * g:(r + 1) * g], ref, atol=1e-12)


@pytest.mark.parametrize("inv_sigma", [1.0, 0.5, 2.0, 0.0])
@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_bias_form_equals_prior_form(alpha, inv_sigma):
    """Proposition 4.1 (additive bias d_ij) against Eq. 9 with the Eq. 11-12 prior
    (w', lambda), computed independently inside the oracle."""
    n, hq, hkv, d, B = 160, 4, 2, 16, 16
    Q, K, V = _rand((1, n, hq, d), 50), _rand((1, n, hkv, d), 51), _rand((1, n, hkv, d), 52)
    kw = dict(chunk=B, alpha=alpha, gamma=6.0, inv_sigma=inv_sigma)
    O1, _ = oracle.prefill(Q, K, V, _rand((hkv, d), 53), **kw)
    O2, _ = oracle.prefill(Q, K, V, _rand((hkv, d), 53), prior_form=True, **kw)
    np.testing.assert_allclose(O1, O2, atol=1e-12)


def test_first_chunk_rows_are_local_causal_softmax():
    n, hq, hkv, d, B = 64, 2, 1, 8, 32
    Q, K, V = _rand((1, n, hq, d), 60), _rand((1, n, hkv, d), 61), _rand((1, n, hkv, d), 62)
    O, _ = oracle.prefill(Q, K, V, _rand((hkv, d), 63), chunk=B, alpha=1.5, gamma=5.0)
    mask = torch.ones(B, B, dtype=torch.bool).tril()
    ref = _sdpa(Q[:, :B], K[:, :B], V[:, :B], mask)
    np.testing.assert_allclose(O[:, :B], ref, atol=1e-12)


# ----------------------------------------------------------------------------- decode
def test_decode_row_equals_prefill_row():
    b, n, hq, hkv, d, B = 2, 300, 4, 2, 16, 32
    Q, K, V = _rand((b, n, hq, d), 70), _rand((b, n, hkv, d), 71), _rand((b, n, hkv, d), 72)
    qb = _rand((hkv, d), 73, 0.3)
    kw = dict(chunk=B, alpha=1.5, gamma=6.0)
    O, _ = oracle.prefill(Q, K, V, qb, **kw)
    for L in (1, 32, 33, 64, 65, 257, 300):
        seqlens = np.array([L, max(1, L - 7)])
        q = np.stack([Q[0, L - 1], Q[1, seqlens[1] - 1]])
        o = oracle.decode(q, K, V, qb, seqlens, **kw)
        np.testing.assert_allclose(o[0], O[0, L - 1], atol=1e-12)
        np.testing.assert_allclose(o[1], O[1, seqlens[1] - 1], atol=1e-12)
