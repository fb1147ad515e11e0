"""Seeded synthetic inputs for the DashAttention forward pass.

This module only draws random numbers with the shapes and value distributions of the
workloads; it holds none of the method's arithmetic, and it is the one piece shared by the
CUDA path's tests/benchmark and the CPU oracle.

Generator: numpy PCG64, one child stream per tensor (SeedSequence(seed).spawn).  Draws are
float64, rounded once to float32 and, for bf16 workloads, once more to bf16 (round to nearest
even), so both sides read bit-identical values.  Noise scales such as "N(0, 0.1)" are standard
deviations.

Planting (the synthetic stand-in for "informative" chunks): one unit vector u_r per KV head;
a fraction of the complete chunks of each (sequence, KV head) has +strength*u_r added to every
key; a fraction of the query positions of each (sequence, KV head) has +strength*u_r added to
every query head of that group.
"""
from __future__ import annotations

import numpy as np


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round finite float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    try:   # torch's float32 -> bf16 conversion rounds to nearest even, multi-threaded
        import torch
        return torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    except ImportError:  # pragma: no cover
        u = a.view(np.uint32)
        r = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) & np.uint32(0xFFFF0000)
        return r.view(np.float32)


def _streams(seed: int, k: int):
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(k)]


def _finish(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    return round_bf16(a) if dtype == "bf16" else a


def _draw(rng, shape, dtype, scale=1.0, add=None, block=4096):
    """Standard normals of `shape` = [b, n, ...] drawn in C order, position block by position block
    (consecutive draws continue one stream, so the values equal a single draw), times `scale`,
    plus add(b, n0, n1, block) applied in float64, then rounded to float32 (and bf16)."""
    out = np.empty(shape, dtype=np.float32)
    for b in range(shape[0]):
        for n0 in range(0, shape[1], block):
            n1 = min(n0 + block, shape[1])
            x = rng.standard_normal((n1 - n0,) + tuple(shape[2:]))
            if scale != 1.0:
                x *= scale
            if add is not None:
                add(b, n0, n1, x)
            out[b, n0:n1] = round_bf16(x.astype(np.float32)) if dtype == "bf16" else x
    return out


def _unit(rng, hkv, d):
    u = rng.standard_normal((hkv, d))
    return u / np.linalg.norm(u, axis=1, keepdims=True)


def planted(seed: int, batch: int, n: int, h_q: int, h_kv: int, d: int, chunk: int, *,
            dtype: str = "bf16", chunk_frac: float = 0.05, query_frac: float = 0.30,
            strength: float = 2.0, qbar_std: float = 0.05, q_rows=None):
    """Q, K, V ~ N(0, 1) with planted chunks/queries; qbar ~ N(0, qbar_std).

    q_rows=(start, count) draws queries only for positions start..start+count-1 (incremental
    decoding: the query of decode step s is the one at position start+s); the planted fraction
    then applies to those rows."""
    rq, rk, rv, rb, ru, rp = _streams(seed, 6)
    g = h_q // h_kv
    T = n // chunk
    nrow = n if q_rows is None else int(q_rows[1])
    nc = int(round(chunk_frac * T))
    nq = int(round(query_frac * nrow))
    # the planted sets, drawn in the recipe's order: per (sequence, KV head) chunks, then rows
    kplant = np.zeros((batch, h_kv, max(T, 1)), dtype=bool)
    qplant = np.zeros((batch, h_kv, nrow), dtype=bool)
    for b in range(batch):
        for r in range(h_kv):
            if nc > 0:
                kplant[b, r, rp.choice(T, nc, replace=False)] = True
            if nq > 0:
                qplant[b, r, rp.choice(nrow, nq, replace=False)] = True
    # the draws of qbar and u come from their own streams, so their order does not matter
    qbar = rb.standard_normal((h_kv, d)) * qbar_std
    u = _unit(ru, h_kv, d)

    def add_q(b, n0, n1, x):
        for r in range(h_kv):
            rows = np.nonzero(qplant[b, r, n0:n1])[0]
            x[rows, r * g:(r + 1) * g] += strength * u[r]

    def add_k(b, n0, n1, x):
        pos = np.arange(n0, n1)
        c = pos // chunk
        for r in range(h_kv):
            sel = (c < T) & kplant[b, r, np.minimum(c, max(T, 1) - 1)]
            x[sel, r] += strength * u[r]

    Q = _draw(rq, (batch, nrow, h_q, d), dtype, add=add_q)
    K = _draw(rk, (batch, n, h_kv, d), dtype, add=add_k)
    V = _draw(rv, (batch, n, h_kv, d), dtype)
    return {"Q": Q, "K": K, "V": V, "qbar": qbar.astype(np.float32)}


def tiny(seed: int = 0, *, n: int = 512, h_q: int = 4, h_kv: int = 1, d: int = 64,
         chunk: int = 64, planted_chunks=(2, 5), strength: float = 1.5, qbar_std: float = 0.1,
         dtype: str = "f32"):
    """Tiny check case: Q, K, V ~ N(0,1); the keys of the listed chunks and every query get
    +strength*u for one fixed random unit vector u; qbar ~ N(0, qbar_std)."""
    rq, rk, rv, rb, ru = _streams(seed, 5)
    Q = rq.standard_normal((1, n, h_q, d))
    K = rk.standard_normal((1, n, h_kv, d))
    V = rv.standard_normal((1, n, h_kv, d))
    qbar = rb.standard_normal((h_kv, d)) * qbar_std
    u = ru.standard_normal(d)
    u /= np.linalg.norm(u)
    for c in planted_chunks:
        K[0, c * chunk:(c + 1) * chunk] += strength * u
    Q[0] += strength * u
    return {"Q": _finish(Q, dtype), "K": _finish(K, dtype), "V": _finish(V, dtype),
            "qbar": qbar.astype(np.float32)}


def mixture(seed: int, batch: int, n: int, h_q: int, h_kv: int, d: int, *, components: int = 64,
            segment: int = 128, spread: float = 0.5, qbar_std: float = 0.05, dtype: str = "bf16"):
    """Gaussian-mixture keys and queries: centres ~ N(0, I) per KV head; every `segment`-token
    block of keys takes one uniformly drawn component (key = centre + spread*eps); every query
    position takes its own component per KV group (query = centre + spread*eps for each head
    of the group); V ~ N(0, 1)."""
    rc, ra, rk, rq, rv, rb = _streams(seed, 6)
    g = h_q // h_kv
    cen = rc.standard_normal((h_kv, components, d))
    nseg = (n + segment - 1) // segment
    comp = np.zeros((batch, h_kv, nseg), dtype=np.int64)
    qc = np.zeros((batch, h_kv, n), dtype=np.int64)
    for b in range(batch):
        for r in range(h_kv):
            comp[b, r] = ra.integers(0, components, nseg)
            qc[b, r] = ra.integers(0, components, n)

    def add_k(b, n0, n1, x):
        seg = np.arange(n0, n1) // segment
        for r in range(h_kv):
            x[:, r] += cen[r, comp[b, r, seg]]

    def add_q(b, n0, n1, x):
        for r in range(h_kv):
            x[:, r * g:(r + 1) * g] += cen[r, qc[b, r, n0:n1]][:, None, :]

    K = _draw(rk, (batch, n, h_kv, d), dtype, scale=spread, add=add_k)
    Q = _draw(rq, (batch, n, h_q, d), dtype, scale=spread, add=add_q)
    V = _draw(rv, (batch, n, h_kv, d), dtype)
    qbar = rb.standard_normal((h_kv, d)) * qbar_std
    return {"Q": Q, "K": K, "V": V, "qbar": qbar.astype(np.float32)}
