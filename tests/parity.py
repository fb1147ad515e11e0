"""Comparison helpers for the GPU-vs-oracle parity tests.

Policy (tolerances from the benchmark spec of the forward pass; readings of the pages for the
ill-conditioned cases):
  * routed chunk sets are bit-exact wherever the oracle's margin max_h((alpha-1) gamma zbar - tau)
    is larger than 1e-4 in magnitude;
  * outputs: max-abs <= 1e-4 for fp32 inputs; max-abs <= 2e-2 and mean-relative
    (mean |diff| / mean |ref|) <= 1e-2 for bf16 inputs, on every row whose routed set matches;
  * log w -> -inf as a chunk's margin -> 0+, so a row may exceed the output tolerance only if one
    of its visible chunks has |margin| < 1e-3; such rows are returned (and reported), never dropped
    silently.
"""
from __future__ import annotations

import numpy as np

MARGIN_EXACT = 1e-4
MARGIN_ILL = 1e-3
TOL = {"f32": dict(max_abs=1e-4, mean_rel=None), "bf16": dict(max_abs=2e-2, mean_rel=1e-2)}


def tri_offset(i, B):
    c = i // B
    return B * (c * (c - 1) // 2) + (i - c * B) * c


def gpu_sets(counts, idx, positions, B, decode=False):
    """Routed chunk sets per (b, r, row) from the GPU lists (host numpy arrays)."""
    bsz, hkv = counts.shape[0], counts.shape[1]
    out = {}
    for b in range(bsz):
        for r in range(hkv):
            for t, i in enumerate(positions[b] if np.ndim(positions) == 2 else positions):
                if decode:
                    cnt = counts[b, r]
                    lst = idx[b, r, :cnt]
                else:
                    cnt = counts[b, r, i]
                    off = tri_offset(int(i), B)
                    lst = idx[b, r, off:off + cnt]
                out[(b, r, t)] = lst
    return out


def check_routes(gsets, orc_route, B, positions, T):
    """Returns (mismatched rows set, number of rows).  Raises on a violation of the bit-exact rule
    or on a GPU list that is not strictly ascending."""
    w, margin = orc_route["w"], orc_route["margin"]
    mism = set()
    for (b, r, t), lst in gsets.items():
        i = int(positions[b][t] if np.ndim(positions) == 2 else positions[t])
        nv = min(i // B, T)
        assert np.all(np.diff(lst) > 0), f"list not ascending at {(b, r, i)}"
        gs = np.zeros(nv, bool)
        gs[lst] = True
        os_ = w[b, r, t, :nv] > 0
        diff = np.nonzero(gs != os_)[0]
        if diff.size:
            bad = diff[np.abs(margin[b, r, t, diff]) > MARGIN_EXACT]
            assert bad.size == 0, (f"route mismatch beyond the margin rule at b={b} r={r} i={i}: chunks {bad} "
                                   f"margins {margin[b, r, t, bad]}")
            mism.add((b, r, t))
    return mism, len(gsets)


def bias_tolerance(margins, alpha, gamma, inv_sigma):
    """Allowed |GPU bias - oracle bias| for each routed chunk of one row (margins: the oracle's
    max over the group's heads of x_c - tau, in units of x = (alpha-1) gamma zbar).

    The bias is (log w_c - mu) / sigma with w_c the group mean of [x_c - tau]_+^(1/(alpha-1)).  A
    logit error of delta (in x units) moves log w_c by at most delta / ((alpha-1) m_c) through the
    head that sets the margin m_c, and mu by the mean of that over the routed chunks.  The GPU's
    chunk logits carry an absolute error of about 1e-5 in zbar (fp32 summaries and fp32
    accumulation), i.e. delta = 2e-5 (alpha-1) max(gamma, 1) with a factor 2 of headroom."""
    m = np.maximum(np.asarray(margins, dtype=np.float64), 1e-12)
    delta = 2e-5 * (alpha - 1) * max(gamma, 1.0)
    s = delta / ((alpha - 1) * m)
    return 1e-4 + inv_sigma * (s + s.mean())


def check_outputs(O_gpu, O_ref, dtype, g, mism=(), orc_route=None, B=None, positions=None, T=None):
    """O_* [b, rows, h_q, d].  Returns dict of error statistics and the list of ill-conditioned rows
    that exceeded the tolerance (each explained by a near-threshold chunk)."""
    tol = TOL[dtype]
    O_gpu = np.asarray(O_gpu, dtype=np.float64)
    err = np.abs(O_gpu - O_ref)
    bsz, nrows, hq, _ = O_ref.shape
    keep = np.ones((bsz, nrows, hq), bool)
    for (b, r, t) in mism:
        keep[b, t, r * g:(r + 1) * g] = False
    row_err = err.max(-1)
    over = (row_err > tol["max_abs"]) & keep
    explained = []
    for b, t, h in zip(*np.nonzero(over)):
        r = h // g
        assert orc_route is not None, f"row b={b} t={t} h={h} error {row_err[b, t, h]:.3g} over tolerance"
        i = int(positions[b][t] if np.ndim(positions) == 2 else positions[t])
        nv = min(i // B, T)
        mm = np.abs(orc_route["margin"][b, r, t, :nv])
        assert nv > 0 and mm.min() < MARGIN_ILL, (f"row b={b} i={i} h={h} error {row_err[b, t, h]:.3g} over "
                                                  f"tolerance without a near-threshold chunk (min margin "
                                                  f"{mm.min() if nv else None})")
        explained.append((int(b), i, int(h), float(row_err[b, t, h]), float(mm.min())))
        keep[b, t, h] = False
    e = err[keep]
    ref = np.abs(O_ref)[keep]
    stats = {"max_abs": float(e.max()) if e.size else 0.0,
             "mean_rel": float(e.mean() / max(ref.mean(), 1e-30)) if e.size else 0.0,
             "rows": int(keep.sum()), "route_mismatch_rows": len(mism), "ill_conditioned": explained}
    assert stats["max_abs"] <= tol["max_abs"], stats
    if tol["mean_rel"] is not None:
        assert stats["mean_rel"] <= tol["mean_rel"], stats
    # ill-conditioned rows must stay a small minority
    assert len(explained) <= max(2, 0.01 * keep.size), stats
    return stats
