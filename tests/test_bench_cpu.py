"""CPU checks of bench.py's derived figures: the executed Stage 2 work per 128-row tile (the union
of its positions' routed and diagonal chunks), counted against a brute-force union on small
random routes, in sequence order and in a permuted position order."""
import os
import sys
import types

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from adaptive_sparse_hierarchical_b200 import _lib as L  # noqa: E402


def _tri(i, B):
    c = i // B
    return B * c * (c - 1) // 2 + (i - c * B) * c


def _routes(rng, n, B, hkv):
    cap = _tri(n, B)
    counts = np.zeros((1, hkv, n), np.int32)
    idx = np.full((1, hkv, max(cap, 1)), -7, np.int32)
    lists = {}
    for r in range(hkv):
        for i in range(n):
            nv = i // B
            k = int(rng.integers(0, nv + 1)) if nv else 0
            sel = np.sort(rng.choice(nv, size=k, replace=False)) if k else np.zeros(0, np.int64)
            counts[0, r, i] = k
            idx[0, r, _tri(i, B):_tri(i, B) + k] = sel
            lists[(r, i)] = sel
    return counts, idx, lists


@pytest.mark.parametrize("B,g,permuted", [(32, 8, False), (64, 8, True), (128, 16, True), (32, 4, False)])
def test_executed_work_is_the_tile_union(monkeypatch, B, g, permuted):
    rng = np.random.default_rng(B + g)
    n, hkv = 700, 2
    wl = types.SimpleNamespace(h_q=g * hkv, h_kv=hkv, chunk=B, n=n, d=128, dtype="bf16", batch=1)
    counts, idx, lists = _routes(rng, n, B, hkv)
    order = np.stack([rng.permutation(n) if permuted else np.arange(n) for _ in range(hkv)]).astype(np.int32)
    ws = torch.from_numpy(np.concatenate([np.zeros(64, np.uint8), order.reshape(-1).view(np.uint8)]))
    pf = types.SimpleNamespace(p=None, workspace=ws, chunk_idx=torch.from_numpy(idx))
    monkeypatch.setattr(L, "dash_prefill_order_offset", lambda p: 64 if permuted else -1)
    got = bench.stage2_executed_flops(pf, wl, counts)
    P, CPT = 128 // g, (2 if B == 32 else 1)
    units = 0
    for r in range(hkv):
        for t in range((n + P - 1) // P):
            u = set()
            for i in order[r, t * P:(t + 1) * P]:
                u |= {int(c) // CPT for c in lists[(r, int(i))]}
                u.add((int(i) // B) // CPT)
            units += len(u)
    assert got == 4.0 * 128 * 128 * B * CPT * units
