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
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16 << 16
    out = (u & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    nan = np.isnan(a)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def _streams(seed: int, k: int):
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(k)]


def _finish(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    return round_bf16(a) if dtype == "bf16" else a


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
    Q = rq.standard_normal((batch, nrow, h_q, d))
    K = rk.standard_normal((batch, n, h_kv, d))
    V = rv.standard_normal((batch, n, h_kv, d))
    qbar = rb.standard_normal((h_kv, d)) * qbar_std
    u = _unit(ru, h_kv, d)
    nc = int(round(chunk_frac * T))
    nq = int(round(query_frac * nrow))
    for b in range(batch):
        for r in range(h_kv):
            if nc > 0:
                for c in rp.choice(T, nc, replace=False):
                    K[b, c * chunk:(c + 1) * chunk, r] += strength * u[r]
            if nq > 0:
                pos = rp.choice(nrow, nq, replace=False)
                Q[b, pos, r * g:(r + 1) * g] += strength * u[r]
    return {"Q": _finish(Q, dtype), "K": _finish(K, dtype), "V": _finish(V, dtype),
            "qbar": qbar.astype(np.float32)}


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
    K = rk.standard_normal((batch, n, h_kv, d)) * spread
    Q = rq.standard_normal((batch, n, h_q, d)) * spread
    for b in range(batch):
        for r in range(h_kv):
            comp = ra.integers(0, components, nseg)
            K[b, :, r] += np.repeat(cen[r, comp], segment, axis=0)[:n]
            qc = ra.integers(0, components, n)
            Q[b, :, r * g:(r + 1) * g] += cen[r, qc][:, None, :]
    V = rv.standard_normal((batch, n, h_kv, d))
    qbar = rb.standard_normal((h_kv, d)) * qbar_std
    return {"Q": _finish(Q, dtype), "K": _finish(K, dtype), "V": _finish(V, dtype),
            "qbar": qbar.astype(np.float32)}
