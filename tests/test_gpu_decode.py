"""GPU parity of incremental decoding (dash_summary_build / dash_summary_append / dash_decode
through the C ABI) against the float64 oracle: summary cache, incomplete-chunk state, routes and
outputs, step after step."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import adaptive_sparse_hierarchical_b200 as D
from adaptive_sparse_hierarchical_b200 import inputs, workloads as W

from parity import check_outputs, check_routes

pytestmark = pytest.mark.gpu


def _tdt(dtype):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def _state(x, lengths, capacity, *, chunk, alpha, gamma, dtype, inv_sigma=1.0):
    b, _, hkv, d = x["K"].shape
    hq = x["Q"].shape[2]
    st = D.DecodeState(b, capacity, hq, hkv, d, chunk=chunk, alpha=alpha, gamma=gamma, inv_sigma=inv_sigma,
                       dtype=_tdt(dtype), qbar=torch.from_numpy(x["qbar"]).cuda())
    L0 = int(max(lengths))
    st.fill(torch.from_numpy(x["K"][:, :L0]).to("cuda", _tdt(dtype)),
            torch.from_numpy(x["V"][:, :L0]).to("cuda", _tdt(dtype)), lengths)
    counts = torch.zeros((b, hkv), dtype=torch.int32, device="cuda")
    idx = torch.zeros((b, hkv, max(capacity // chunk, 1)), dtype=torch.int32, device="cuda")
    bias = torch.zeros((b, hkv, max(capacity // chunk, 1)), dtype=torch.float32, device="cuda")
    words = (capacity // chunk + 31) // 32
    bm = torch.full((b, hkv, max(words, 1)), -1, dtype=torch.int32, device="cuda")   # all bits set: must be rewritten
    st.route = D.route_out(counts, idx, bias, bm)
    st.rt = (counts, idx, bias)
    st.bm = bm
    return st


def _check_bitmask(st):
    """The bitmask output holds exactly the chunks of the route list (32 chunks per word)."""
    counts, idx, _ = (t.cpu().numpy() for t in st.rt)
    bm = st.bm.cpu().numpy().view(np.uint32)
    b, hkv, words = bm.shape
    for bb in range(b):
        for r in range(hkv):
            want = np.zeros(words * 32, dtype=bool)
            want[idx[bb, r, :counts[bb, r]]] = True
            got = ((bm[bb, r][:, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool).reshape(-1)
            assert np.array_equal(got, want), (bb, r)


def _check_summaries(st, x, chunk):
    K = x["K"]
    lens = st.seqlens.cpu().numpy()
    kb = st.kbar.cpu().numpy()
    state = st.state.cpu().numpy()
    b, _, hkv, d = K.shape
    for bb in range(b):
        L = int(lens[bb])
        ref = oracle.stage0(K[bb:bb + 1, :L], x["qbar"], chunk)[0]
        np.testing.assert_allclose(kb[bb, :, :L // chunk], ref, atol=2e-5, rtol=1e-5)
        if L % chunk:
            for r in range(hkv):
                part = oracle.chunk_summary(K, x["qbar"], bb, r, (L // chunk) * chunk, L)
                np.testing.assert_allclose(state[bb, r, :d] / state[bb, r, d + 1], part, atol=2e-5, rtol=1e-5)


def _check_step(st, x, q, lengths, *, chunk, alpha, gamma, dtype, inv_sigma=1.0):
    b, _, hkv, d = x["K"].shape
    hq = x["Q"].shape[2]
    O = st.O.float().cpu().numpy()
    oref, rt = oracle.decode(q, x["K"], x["V"], x["qbar"], lengths, chunk=chunk, alpha=alpha, gamma=gamma,
                             inv_sigma=inv_sigma, want_route=True)
    counts, idx, _ = (t.cpu().numpy() for t in st.rt)
    T = x["K"].shape[1] // chunk
    gs = {(bb, r, 0): idx[bb, r, :counts[bb, r]] for bb in range(b) for r in range(hkv)}
    pos = (np.asarray(lengths) - 1).reshape(b, 1)
    # oracle route arrays are [b, hkv, 1, T']; pad T' to the cache's chunk count
    mism, _ = check_routes(gs, rt, chunk, pos, T)
    _check_bitmask(st)
    return check_outputs(O[:, None], oref[:, None], dtype, hq // hkv, mism, rt, chunk, pos, T)


@pytest.mark.parametrize("dtype,d,B,g", [("bf16", 128, 64, 4), ("bf16", 64, 32, 16), ("f32", 128, 64, 8),
                                         ("bf16", 128, 128, 8), ("bf16", 128, 16, 2), ("bf16", 128, 1, 4),
                                         ("f32", 64, 1, 2)])
def test_decode_steps_small(dtype, d, B, g):
    hkv, cap, b = 2, 1024, 3
    x = inputs.planted(21, b, cap, g * hkv, hkv, d, B, dtype=dtype, chunk_frac=0.1)
    lengths = np.array([300, 511, B])
    st = _state(x, lengths, cap, chunk=B, alpha=1.5, gamma=6.0, dtype=dtype)
    _check_summaries(st, x, B)
    for step in range(70):
        L = lengths.copy()
        k = torch.from_numpy(x["K"][np.arange(b), L]).to("cuda", _tdt(dtype)).contiguous()
        v = torch.from_numpy(x["V"][np.arange(b), L]).to("cuda", _tdt(dtype)).contiguous()
        qn = x["Q"][np.arange(b), L]
        q = torch.from_numpy(qn).to("cuda", _tdt(dtype)).contiguous()
        st.step(q, k, v)
        torch.cuda.synchronize()
        lengths = L + 1
        assert np.array_equal(st.seqlens.cpu().numpy(), lengths)
        if step % 7 == 0 or step == 69:
            _check_step(st, x, qn, lengths, chunk=B, alpha=1.5, gamma=6.0, dtype=dtype)
    _check_summaries(st, x, B)


def test_decode_matches_prefill_rows():
    """Decode of position i equals prefill row i (same kernels' numerics up to bf16 rounding)."""
    b, n, hq, hkv, d, B = 2, 700, 8, 2, 128, 64
    x = inputs.planted(22, b, n, hq, hkv, d, B, dtype="bf16")
    tq = {k: torch.from_numpy(x[k]).to("cuda", torch.bfloat16) for k in ("Q", "K", "V")}
    pf = D.Prefill(tq["Q"], tq["K"], tq["V"], torch.from_numpy(x["qbar"]).cuda(), chunk=B, alpha=1.5, gamma=6.0)
    Opf = pf().float()
    st = _state(x, [600, 640], 1024, chunk=B, alpha=1.5, gamma=6.0, dtype="bf16")
    for _ in range(40):
        L = st.seqlens.cpu().numpy()
        k = tq["K"][torch.arange(b), torch.from_numpy(L).long()].contiguous()
        v = tq["V"][torch.arange(b), torch.from_numpy(L).long()].contiguous()
        q = tq["Q"][torch.arange(b), torch.from_numpy(L).long()].contiguous()
        o = st.step(q, k, v).float()
        ref = Opf[torch.arange(b), torch.from_numpy(L).long()]
        assert (o - ref).abs().max().item() < 2e-2


def test_decode_128k_full_size_sampled():
    """Full-size decode workload (b=8, 131072-token caches, 32/2 heads, d=128, B=64, ~25% routed):
    fill, then append+decode steps; steps 0, 15 and 31 are checked against the oracle."""
    wl = W.get("decode_128k")
    x = wl.make()   # K, V for every position; queries for positions prefix..prefix+steps-1
    prefix = wl.extra["prefix"]
    st = _state(x, [prefix] * wl.batch, wl.n, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma, dtype="bf16")
    Kt = torch.from_numpy(x["K"][:, prefix:prefix + 32]).to("cuda", torch.bfloat16)
    Vt = torch.from_numpy(x["V"][:, prefix:prefix + 32]).to("cuda", torch.bfloat16)
    Qt = torch.from_numpy(x["Q"][:, :32]).to("cuda", torch.bfloat16)
    for s in range(32):
        st.step(Qt[:, s].contiguous(), Kt[:, s].contiguous(), Vt[:, s].contiguous())
        if s in (0, 15, 31):
            torch.cuda.synchronize()
            lengths = np.full(wl.batch, prefix + s + 1)
            stt = _check_step(st, x, x["Q"][:, s], lengths, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma,
                              dtype="bf16")
            print("decode_128k step", s, stt)
    frac = st.rt[0].sum().item() / (wl.batch * 2 * ((prefix + 31) // 64))
    assert 0.15 < frac < 0.35, frac


def test_decode_96k_batch24_full_size_sampled():
    """The pages' decode shape: batch 24, 96K-token caches (32/2 heads, d=128, B=64) at 75% and
    93.75% sparsity (one set of inputs, gamma tuned per sparsity); 8 append+decode steps each,
    steps 0 and 7 checked against the oracle."""
    wl0 = W.get(W.DECODE_96K[0])
    x = wl0.make()
    prefix = wl0.extra["prefix"]
    Kt = torch.from_numpy(x["K"][:, prefix:prefix + 8]).to("cuda", torch.bfloat16)
    Vt = torch.from_numpy(x["V"][:, prefix:prefix + 8]).to("cuda", torch.bfloat16)
    Qt = torch.from_numpy(x["Q"][:, :8]).to("cuda", torch.bfloat16)
    for name in W.DECODE_96K:
        wl = W.get(name)
        st = _state(x, [prefix] * wl.batch, wl.n, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma, dtype="bf16")
        for s in range(8):
            st.step(Qt[:, s].contiguous(), Kt[:, s].contiguous(), Vt[:, s].contiguous())
            if s in (0, 7):
                torch.cuda.synchronize()
                lengths = np.full(wl.batch, prefix + s + 1)
                stt = _check_step(st, x, x["Q"][:, s], lengths, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma,
                                  dtype="bf16")
                print(name, "step", s, stt)
        frac = st.rt[0].sum().item() / (wl.batch * 2 * ((prefix + 7) // 64))
        target = wl.extra["target"]
        assert 0.6 * target < frac < 1.4 * target, (name, frac)
        del st
        torch.cuda.empty_cache()


def test_decode_long_run_is_deterministic():
    """300 append+decode steps, run twice from the same saved state: the outputs must agree bit for
    bit at every step (a race between the producer and consumer warps of a K/V ring would show up
    here), and the last step must match the oracle.  Saving / restoring the caller-owned tensors is
    also how a decode session is checkpointed."""
    b, cap, hq, hkv, d, B = 4, 4096, 16, 2, 128, 64
    x = inputs.planted(23, b, cap, hq, hkv, d, B, dtype="bf16", chunk_frac=0.1)
    lengths = np.array([3000, 2500, 1999, 3300])
    st = _state(x, lengths, cap, chunk=B, alpha=1.5, gamma=5.0, dtype="bf16")
    saved = [t.clone() for t in (st.K, st.V, st.kbar, st.state, st.seqlens)]
    dev = {k: torch.from_numpy(x[k]).to("cuda", torch.bfloat16) for k in ("Q", "K", "V")}
    runs = []
    for rep in range(2):
        for t, sv in zip((st.K, st.V, st.kbar, st.state, st.seqlens), saved):
            t.copy_(sv)
        outs = []
        for step in range(300):
            pos = torch.from_numpy(lengths + step).long().cuda()
            rows = torch.arange(b, device="cuda")
            o = st.step(dev["Q"][rows, pos].contiguous(), dev["K"][rows, pos].contiguous(),
                        dev["V"][rows, pos].contiguous())
            outs.append(o.clone())
        torch.cuda.synchronize()
        runs.append(torch.stack(outs))
    assert torch.equal(runs[0], runs[1])
    last = lengths + 300
    _check_step(st, x, x["Q"][np.arange(b), last - 1], last, chunk=B, alpha=1.5, gamma=5.0, dtype="bf16")


def test_decode_per_head_routing_kernels():
    """The per-head decode routing kernels (used when a group's logits do not fit the cluster
    kernel's shared memory, i.e. very long contexts) selected by DASH_DEC_ROUTE=heads: the small
    decode cases pass through them too."""
    env = dict(os.environ, DASH_DEC_ROUTE="heads")
    here = os.path.dirname(os.path.abspath(__file__))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-x",
                        os.path.join(here, "test_gpu_decode.py"), "-k", "test_decode_steps_small"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
