"""GPU parity of the backward pass (dash_backward through the C ABI) against the float64 oracle's
backward (oracle.backward, itself pinned by finite differences of the forward oracle).

The forward runs on the GPU first (its route lists and summaries feed the backward, as in
training); the test requires that those routes equal the oracle's (no near-threshold chunk), so
that both sides differentiate the same piecewise-smooth branch.

Tolerance.  Both sides read the same bf16 / fp32 input values; the GPU computes in fp32.  Away
from the support boundary the gradients carry ~1e-6 relative rounding.  The bias term
d log w / dx scales as 1/(margin) for a chunk whose margin x - tau is small (the forward's
ill-conditioning, seen in the backward), so a chunk at margin 1e-4 turns 1e-6 of logit rounding
into ~1e-2 relative error in its own entries.  Hence, per tensor: every element within
2e-2 |ref| + 2e-3 max|ref|, and the relative Frobenius error below 5e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import adaptive_sparse_hierarchical_b200 as D
from adaptive_sparse_hierarchical_b200 import inputs, workloads as W

from parity import check_routes, gpu_sets

pytestmark = pytest.mark.gpu


def _dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", torch.bfloat16 if dtype == "bf16" else torch.float32)


def _compare(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    scale = np.abs(ref).max()
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    bad = err > 2e-2 * np.abs(ref) + 2e-3 * scale
    stats = {"max_abs": float(err.max()), "max_ref": float(scale), "fro_rel": float(fro), "bad": int(bad.sum())}
    assert bad.sum() == 0 and fro <= 5e-3, (name, stats, np.argwhere(bad)[:5])
    return stats


CASES = [
    # (dtype, b, n, hq, hkv, d, B, alpha, gamma, inv_sigma)
    ("bf16", 2, 700, 8, 2, 128, 64, 1.5, 6.0, 1.0),
    ("bf16", 1, 520, 16, 2, 64, 32, 1.5, 6.0, 0.5),
    ("f32", 1, 400, 4, 2, 128, 64, 2.0, 4.0, 1.0),
    ("bf16", 1, 300, 4, 1, 64, 16, 1.3, 5.0, 1.0),
    ("bf16", 1, 600, 4, 2, 128, 128, 1.5, 6.0, 1.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_oracle(case):
    dtype, b, n, hq, hkv, d, B, alpha, gamma, inv_sigma = case
    x = inputs.planted(41, b, n, hq, hkv, d, B, dtype=dtype, chunk_frac=0.1)
    x["qbar"] = inputs.round_bf16(x["qbar"] * 10.0)   # Stage 0 weights away from uniform
    rng = np.random.default_rng(42)
    dO = rng.standard_normal((b, n, hq, d))
    dO = inputs.round_bf16(dO) if dtype == "bf16" else dO.astype(np.float32)
    kw = dict(chunk=B, alpha=alpha, gamma=gamma, inv_sigma=inv_sigma)

    Q, K, V = (_dev(x[k], dtype) for k in ("Q", "K", "V"))
    qbar = torch.from_numpy(np.ascontiguousarray(x["qbar"], dtype=np.float32)).cuda()
    pf = D.Prefill(Q, K, V, qbar, want_route=True, **kw)
    pf()
    dQ, dK, dV, dqb = pf.backward(_dev(dO, dtype))
    torch.cuda.synchronize()

    positions = np.arange(n)
    _, _, rt = oracle.prefill(x["Q"], x["K"], x["V"], x["qbar"], want_route=True, **kw)
    gs = gpu_sets(pf.counts.cpu().numpy(), pf.chunk_idx.cpu().numpy(), positions, B)
    mism, _ = check_routes(gs, rt, B, positions, n // B)
    assert not mism, f"routes differ from the oracle's on {len(mism)} rows (near-threshold chunks)"

    rQ, rK, rV, rqb = oracle.backward(x["Q"], x["K"], x["V"], x["qbar"], dO, **kw)
    st = {k: _compare(k, g.cpu().numpy(), r) for k, g, r in
          (("dQ", dQ, rQ), ("dK", dK, rK), ("dV", dV, rV), ("dqbar", dqb, rqb))}
    print(case, st)


def test_backward_is_deterministic_and_reuses_buffers():
    x = inputs.planted(43, 1, 640, 8, 2, 128, 64, dtype="bf16", chunk_frac=0.1)
    Q, K, V = (_dev(x[k], "bf16") for k in ("Q", "K", "V"))
    pf = D.Prefill(Q, K, V, torch.from_numpy(x["qbar"]).cuda(), chunk=64, alpha=1.5, gamma=6.0, want_route=True)
    pf()
    dO = torch.randn(Q.shape, device="cuda").to(torch.bfloat16)
    first = [t.clone() for t in pf.backward(dO)]
    second = pf.backward(dO)
    torch.cuda.synchronize()
    for a, c in zip(first, second):
        assert torch.equal(a, c)


def test_backward_full_size_prefill_32k_properties():
    """The 32K prefill workload (b=1, n=32768, 16/2 heads, d=128, B=64, ~25% routed): the
    backward runs at full size, every gradient is finite, and sum_j dV_j equals the sum of the
    group's dO rows (each row's attention weights sum to one), per KV head and element."""
    wl = W.get("prefill_32k")
    x = wl.make()
    Q, K, V = (_dev(x[k], "bf16") for k in ("Q", "K", "V"))
    pf = D.Prefill(Q, K, V, torch.from_numpy(x["qbar"]).cuda(), chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma,
                   want_route=True)
    pf()
    g = torch.Generator(device="cuda").manual_seed(7)
    dO = torch.randn(Q.shape, device="cuda", generator=g).to(torch.bfloat16)
    dQ, dK, dV, dqb = pf.backward(dO)
    torch.cuda.synchronize()
    for t in (dQ, dK, dV, dqb):
        assert torch.isfinite(t).all()
    hkv = K.shape[2]
    want = dO.double().reshape(1, wl.n, hkv, -1, Q.shape[3]).sum(dim=(1, 3))
    got = dV.double().sum(dim=1)
    rel = ((got - want).abs().max() / want.abs().max()).item()
    assert rel < 1e-4, rel
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(3):
        pf.backward(dO)
    ev[1].record()
    torch.cuda.synchronize()
    print("prefill_32k backward ms", ev[0].elapsed_time(ev[1]) / 3)
