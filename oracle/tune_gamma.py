"""Choose the routing scale gamma of each workload so that the mean routed fraction hits its
target, using only the CPU oracle (Stage 0 + Stage 1), and write the values to
adaptive_sparse_hierarchical_b200/workloads.json.  TEST/INPUT INFRASTRUCTURE: run by hand.

Routed fraction = sum |R| / sum floor(i/B) over the sampled rows with floor(i/B) >= 1, sampled
every `stride`-th position (decode: every 8th step).  Bisection on log(gamma).

    python oracle/tune_gamma.py
"""
from __future__ import annotations

import json
import math
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from adaptive_sparse_hierarchical_b200 import workloads as W  # noqa: E402


def _fraction(Qrows, pos, K, kbar, chunk, alpha, gamma):
    counts = oracle.route_counts(Qrows, pos, K, kbar, chunk=chunk, alpha=alpha, gamma=gamma)
    vis = np.minimum(np.asarray(pos) // chunk, kbar.shape[2])
    den = vis.sum() * kbar.shape[1]
    return counts.sum() / den


def tune(Qrows, pos, K, kbar, chunk, alpha, target, lo=0.25, hi=1024.0, iters=22):
    a, b = math.log(lo), math.log(hi)
    for _ in range(iters):
        m = 0.5 * (a + b)
        f = _fraction(Qrows, pos, K, kbar, chunk, alpha, math.exp(m))
        if f > target:
            a = m   # too dense: raise gamma
        else:
            b = m
    g = math.exp(0.5 * (a + b))
    return g, _fraction(Qrows, pos, K, kbar, chunk, alpha, g)


def prefill_case(name, stride):
    wl = W.get(name)
    x = wl.make()
    kbar = oracle.stage0(x["K"], x["qbar"], wl.chunk)
    pos = np.arange(stride // 2, wl.n, stride, dtype=np.int32)
    Qrows = x["Q"][:, pos]
    target = wl.extra.get("target", 0.25)
    g, f = tune(Qrows, np.broadcast_to(pos, (wl.batch, pos.size)), x["K"], kbar, wl.chunk, wl.alpha, target)
    print(f"{name}: gamma={g:.4f} routed fraction={f:.4f} (target {target})", flush=True)
    return g


def decode_case(name):
    wl = W.get(name)
    x = wl.make()
    prefix, steps = wl.extra["prefix"], wl.extra["steps"]
    kbar = oracle.stage0(x["K"][:, :prefix + steps], x["qbar"], wl.chunk)
    sel = np.arange(0, steps, 8)
    pos = (prefix + sel).astype(np.int32)
    Qrows = x["Q"][:, sel]
    target = wl.extra.get("target", 0.25)
    g, f = tune(Qrows, np.broadcast_to(pos, (wl.batch, pos.size)), x["K"], kbar, wl.chunk, wl.alpha, target)
    print(f"{name}: gamma={g:.4f} routed fraction={f:.4f} (target {target})", flush=True)
    return g


def main():
    path = os.path.join(ROOT, "adaptive_sparse_hierarchical_b200", "workloads.json")
    out = W.tuned_gammas()
    todo = sys.argv[1:] or ["prefill_32k", "decode_128k", *W.PREFILL_64K, *W.DECODE_96K]
    for name in todo:
        out[name] = round(prefill_case(name, 64) if name.startswith("prefill") else decode_case(name), 4)
        with open(path, "w") as fh:
            json.dump(out, fh, indent=1, sort_keys=True)
            fh.write("\n")


if __name__ == "__main__":
    main()
