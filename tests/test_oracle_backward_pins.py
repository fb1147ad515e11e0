"""Pins for the float64 oracle's backward pass (oracle.backward), CPU only.

The paper review page of DashAttention (section 3, the text after Eq. 9, and the Stage 2 kernel
row) states that the output is differentiable in q, k, v and the prior, with the gradient
reaching the Stage 1 entmax scores and the Stage 0 summaries.  The backward oracle writes that
chain out by hand; these tests pin it to things it does not compute itself:
  - central finite differences of the FORWARD oracle (a different code path: it never forms a
    derivative) at sampled coordinates of Q, K, V and qbar, for alpha = 1.5 (quadratic tau),
    alpha = 2 (sparsemax) and alpha = 1.3 (Newton tau), with a ragged tail chunk;
  - sum_j dV_j = sum over the group's query rows of dO (each softmax row sums to one);
  - sigma -> infinity (inv_sigma = 0) or gamma = 0: no gradient reaches qbar, and dQ, dK, dV
    equal torch float64 autograd of a plain masked softmax attention over the routed and
    diagonal tokens (a textbook routine, the mask taken from the forward oracle's routes).
"""
import numpy as np
import pytest
import torch

import oracle
from adaptive_sparse_hierarchical_b200 import inputs

H = 2.0 ** -13   # perturbation: x +- H is exact in float32 for the bf16-valued inputs


def _case(seed, b, n, hq, hkv, d, B, qbar_scale=20.0):
    x = inputs.planted(seed, b, n, hq, hkv, d, B, dtype="bf16", chunk_frac=0.25)
    qbar = inputs.round_bf16(x["qbar"] * qbar_scale)   # larger qbar: Stage 0 softmax far from uniform
    rng = np.random.default_rng(seed + 100)
    dO = inputs.round_bf16(rng.standard_normal((b, n, hq, d)))
    return {"Q": x["Q"].astype(np.float32), "K": x["K"].astype(np.float32), "V": x["V"].astype(np.float32),
            "qbar": qbar.astype(np.float32), "dO": dO.astype(np.float32)}


def _loss(t, kw):
    O, _, rt = oracle.prefill(t["Q"], t["K"], t["V"], t["qbar"], want_route=True, nthreads=1, **kw)
    return float(np.sum(O * t["dO"].astype(np.float64))), rt["w"] > 0


def _fd(t, name, idx, h, kw):
    x0 = t[name][idx]
    vals, masks = [], []
    for s in (+1, -1):
        tt = dict(t)
        tt[name] = t[name].copy()
        tt[name][idx] = np.float32(x0 + s * h)
        f, m = _loss(tt, kw)
        vals.append(f)
        masks.append(m)
    same = np.array_equal(masks[0], masks[1])
    return (vals[0] - vals[1]) / (2 * h), same


CONFIGS = [
    # (alpha, gamma, inv_sigma, b, n, hq, hkv, d, B)
    (1.5, 6.0, 1.0, 1, 150, 4, 2, 16, 32),
    (2.0, 4.0, 0.5, 2, 100, 2, 1, 16, 16),
    (1.3, 5.0, 1.0, 1, 140, 4, 1, 16, 32),
]


@pytest.mark.parametrize("cfg", CONFIGS, ids=["alpha1.5", "alpha2", "alpha1.3"])
def test_backward_matches_finite_differences(cfg):
    alpha, gamma, inv_sigma, b, n, hq, hkv, d, B = cfg
    kw = dict(chunk=B, alpha=alpha, gamma=gamma, inv_sigma=inv_sigma)
    t = _case(7, b, n, hq, hkv, d, B)
    dQ, dK, dV, dqbar = oracle.backward(t["Q"], t["K"], t["V"], t["qbar"], t["dO"], nthreads=1, **kw)
    grads = {"Q": dQ, "K": dK, "V": dV, "qbar": dqbar}
    rng = np.random.default_rng(11)
    for name, g in grads.items():
        shape = t[name].shape
        gmax = np.abs(g).max()
        assert gmax > 0, name
        checked = 0
        for k in range(10):
            if name == "Q" and k < 6:   # rows past the first chunk: the Stage 1 chain is live there
                pos = int(rng.integers(B, n))
                idx = (int(rng.integers(shape[0])), pos, int(rng.integers(hq)), int(rng.integers(d)))
            elif name == "K" and k < 6:  # keys of complete chunks: the Stage 0 chain is live there
                pos = int(rng.integers(0, (n // B) * B))
                idx = (int(rng.integers(shape[0])), pos, int(rng.integers(hkv)), int(rng.integers(d)))
            else:
                idx = tuple(int(rng.integers(s)) for s in shape)
            f1, same1 = _fd(t, name, idx, H, kw)
            f2, same2 = _fd(t, name, idx, H / 2, kw)
            # a support change inside +-H (a kink of the piecewise-smooth map) shows up as a
            # changed routed set or as two step sizes that disagree: such coordinates are skipped
            if not (same1 and same2) or abs(f1 - f2) > 1e-6 + 1e-5 * gmax:
                continue
            checked += 1
            assert abs(g[idx] - f2) <= 2e-6 + 2e-5 * gmax, (name, idx, g[idx], f2, gmax)
        assert checked >= 7, (name, checked)


def test_stage1_and_stage0_terms_are_live():
    """The finite-difference cases above exercise the routing chain: switching it off
    (inv_sigma = 0 removes the bias) changes dQ and dK and zeroes dqbar."""
    alpha, gamma, inv_sigma, b, n, hq, hkv, d, B = CONFIGS[0]
    t = _case(7, b, n, hq, hkv, d, B)
    on = oracle.backward(t["Q"], t["K"], t["V"], t["qbar"], t["dO"], chunk=B, alpha=alpha, gamma=gamma,
                         inv_sigma=1.0)
    off = oracle.backward(t["Q"], t["K"], t["V"], t["qbar"], t["dO"], chunk=B, alpha=alpha, gamma=gamma,
                          inv_sigma=0.0)
    assert np.abs(on[3]).max() > 1e-3 and np.all(off[3] == 0.0)
    assert np.abs(on[0] - off[0]).max() > 1e-3 and np.abs(on[1] - off[1]).max() > 1e-3


@pytest.mark.parametrize("cfg", CONFIGS[:2], ids=["alpha1.5", "alpha2"])
def test_dv_rows_sum_to_group_dO(cfg):
    alpha, gamma, inv_sigma, b, n, hq, hkv, d, B = cfg
    t = _case(3, b, n, hq, hkv, d, B)
    _, _, dV, _ = oracle.backward(t["Q"], t["K"], t["V"], t["qbar"], t["dO"], chunk=B, alpha=alpha, gamma=gamma,
                                  inv_sigma=inv_sigma)
    g = hq // hkv
    want = t["dO"].astype(np.float64).reshape(b, n, hkv, g, d).sum(axis=(1, 3))
    np.testing.assert_allclose(dV.sum(axis=1), want, rtol=1e-12, atol=1e-10)


def _masked_attention_grads(t, mask_fn, B):
    """torch float64 autograd of softmax(Q K^T / sqrt(d) + log mask) V per (b, head)."""
    Q, K, V, dO = (torch.tensor(t[k], dtype=torch.float64, requires_grad=k != "dO") for k in ("Q", "K", "V", "dO"))
    b, n, hq, d = Q.shape
    hkv = K.shape[2]
    g = hq // hkv
    outs = []
    for bb in range(b):
        for h in range(hq):
            r = h // g
            s = Q[bb, :, h] @ K[bb, :, r].T / np.sqrt(d)
            s = s.masked_fill(~mask_fn(bb, r), float("-inf"))
            outs.append((torch.softmax(s, dim=-1) @ V[bb, :, r] * dO[bb, :, h]).sum())
    torch.stack(outs).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


@pytest.mark.parametrize("alpha,gamma,inv_sigma", [(1.5, 6.0, 0.0), (2.0, 0.0, 1.0)])
def test_no_prior_reduces_to_masked_softmax_autograd(alpha, gamma, inv_sigma):
    b, n, hq, hkv, d, B = 1, 130, 4, 2, 16, 32
    t = _case(5, b, n, hq, hkv, d, B)
    kw = dict(chunk=B, alpha=alpha, gamma=gamma, inv_sigma=inv_sigma)
    _, _, rt = oracle.prefill(t["Q"], t["K"], t["V"], t["qbar"], want_route=True, **kw)
    routed = rt["w"] > 0   # [b, hkv, n, T]

    def mask_fn(bb, r):
        i = np.arange(n)[:, None]
        j = np.arange(n)[None, :]
        diag = (j // B == i // B) & (j <= i)
        cj = np.minimum(j // B, routed.shape[3] - 1)
        rout = routed[bb, r][i, cj] & (j // B < i // B)
        return torch.from_numpy(diag | rout)

    dQ, dK, dV, dqbar = oracle.backward(t["Q"], t["K"], t["V"], t["qbar"], t["dO"], **kw)
    rQ, rK, rV = _masked_attention_grads(t, mask_fn, B)
    assert np.all(dqbar == 0.0)
    for a, ref in ((dQ, rQ), (dK, rK), (dV, rV)):
        np.testing.assert_allclose(a, ref, rtol=1e-10, atol=1e-12)


def test_chunk_one_degenerate_case():
    """B = 1: every token is its own chunk, k̄_c = k_c (Stage 0 of one key), so qbar has no effect
    (dqbar = 0 exactly) and the routing runs over the previous tokens themselves.  Finite
    differences of the forward oracle pin dQ, dK and dV there."""
    alpha, gamma, inv_sigma, b, n, hq, hkv, d, B = 1.5, 3.0, 1.0, 1, 24, 2, 1, 8, 1
    kw = dict(chunk=B, alpha=alpha, gamma=gamma, inv_sigma=inv_sigma)
    t = _case(9, b, n, hq, hkv, d, B)
    dQ, dK, dV, dqbar = oracle.backward(t["Q"], t["K"], t["V"], t["qbar"], t["dO"], nthreads=1, **kw)
    assert np.all(dqbar == 0.0)
    rng = np.random.default_rng(13)
    for name, g in (("Q", dQ), ("K", dK), ("V", dV)):
        gmax = np.abs(g).max()
        checked = 0
        for _ in range(10):
            idx = tuple(int(rng.integers(s)) for s in t[name].shape)
            f1, same1 = _fd(t, name, idx, H, kw)
            f2, same2 = _fd(t, name, idx, H / 2, kw)
            if not (same1 and same2) or abs(f1 - f2) > 1e-6 + 1e-5 * gmax:
                continue
            checked += 1
            assert abs(g[idx] - f2) <= 2e-6 + 2e-5 * gmax, (name, idx, g[idx], f2, gmax)
        assert checked >= 7, (name, checked)


@pytest.mark.parametrize("seed", range(6))
def test_dv_identity_on_random_shapes(seed):
    """sum_j dV_j = sum of the group's dO rows on random shapes, chunk sizes, alpha and sigma."""
    rng = np.random.default_rng(200 + seed)
    hkv = int(rng.choice([1, 2]))
    g = int(rng.choice([1, 2, 4]))
    B = int(rng.choice([1, 4, 16, 32]))
    n = int(rng.integers(B + 1, 5 * B + 40))
    d = int(rng.choice([8, 16]))
    alpha = float(rng.choice([1.25, 1.5, 2.0]))
    inv_sigma = float(rng.choice([0.0, 0.5, 1.0]))
    t = _case(300 + seed, 1, n, hkv * g, hkv, d, B)
    _, _, dV, dqbar = oracle.backward(t["Q"], t["K"], t["V"], t["qbar"], t["dO"], chunk=B, alpha=alpha, gamma=4.0,
                                      inv_sigma=inv_sigma)
    want = t["dO"].astype(np.float64).reshape(1, n, hkv, g, d).sum(axis=(1, 3))
    np.testing.assert_allclose(dV.sum(axis=1), want, rtol=1e-12, atol=1e-10)
    assert np.all(np.isfinite(dqbar)) and (inv_sigma > 0 or np.all(dqbar == 0.0))
