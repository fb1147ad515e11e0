"""Named synthetic workloads (shapes, hyper-parameters, input recipe).  No arithmetic of the
method lives here; the routing scales gamma that hit a target routed fraction are read from
workloads.json, which oracle/tune_gamma.py writes with the CPU oracle.

Routed fraction = sum over (b, KV head, row) of |R| / sum of floor(i/B) over rows with
floor(i/B) >= 1 (the pages' "sparsity" is 1 - fraction).
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass, field

from . import inputs

_JSON = os.path.join(os.path.dirname(os.path.abspath(__file__)), "workloads.json")


def tuned_gammas() -> dict:
    if not os.path.exists(_JSON):
        return {}
    with open(_JSON) as fh:
        return json.load(fh)


@dataclass
class Workload:
    name: str
    batch: int
    n: int
    h_q: int
    h_kv: int
    d: int
    chunk: int
    alpha: float
    gamma: float
    dtype: str
    recipe: str
    inv_sigma: float = 1.0
    extra: dict = field(default_factory=dict)

    def make(self):
        """Q, K, V (float32 arrays holding dtype-exact values) and qbar."""
        if self.recipe == "tiny":
            return inputs.tiny(0, n=self.n, h_q=self.h_q, h_kv=self.h_kv, d=self.d, chunk=self.chunk,
                               dtype=self.dtype)
        if self.recipe == "planted":
            return inputs.planted(self.extra.get("seed", 2), self.batch, self.n, self.h_q, self.h_kv, self.d,
                                  self.chunk, dtype=self.dtype, q_rows=self.extra.get("q_rows"))
        if self.recipe == "mixture":
            return inputs.mixture(self.extra.get("seed", 5), self.batch, self.n, self.h_q, self.h_kv, self.d,
                                  dtype=self.dtype)
        raise ValueError(self.recipe)


def get(name: str) -> Workload:
    g = tuned_gammas()
    if name == "tiny_f32":   # batch 1, n=512, 4/1 heads, d=64, B=64, alpha 1.5, gamma 1 (not sparse)
        return Workload(name, 1, 512, 4, 1, 64, 64, 1.5, 1.0, "f32", "tiny")
    if name == "tiny_f32_sparse":   # the same inputs with gamma = 32 so routing is sparse
        return Workload(name, 1, 512, 4, 1, 64, 64, 1.5, 32.0, "f32", "tiny")
    if name == "tiny_bf16_sparse":
        return Workload(name, 1, 512, 4, 1, 64, 64, 1.5, 32.0, "bf16", "tiny")
    if name == "prefill_32k":   # 1B-class layer: b=1, n=32768, 16/2 heads, d=128, B=64, ~25% routed
        return Workload(name, 1, 32768, 16, 2, 128, 64, 1.5, g.get("prefill_32k", 8.0), "bf16", "planted",
                        extra={"seed": 2})
    if name == "decode_128k":   # b=8, cache 131072 (+1000 steps), 32/2 heads, d=128, B=64, ~25% routed
        return Workload(name, 8, 132096, 32, 2, 128, 64, 1.5, g.get("decode_128k", 8.0), "bf16", "planted",
                        extra={"seed": 3, "q_rows": (131072, 1000), "prefix": 131072, "steps": 1000})
    if name.startswith("prefill_64k_"):   # 8B-class layer: b=2, n=65536, 32/2 heads, B=128
        frac = name.rsplit("_", 1)[1]     # "50", "25" or "12.5"
        return Workload(name, 2, 65536, 32, 2, 128, 128, 1.5, g.get(name, 8.0), "bf16", "planted",
                        extra={"seed": 4, "target": float(frac) / 100})
    if name.startswith("sweep_128k_"):   # b=1, n=131072, 16/2 heads; alpha x B sweep, gamma 1
        _, _, a, B = name.split("_")      # sweep_128k_<alpha>_<B>
        return Workload(name, 1, 131072, 16, 2, 128, int(B), float(a), 1.0, "bf16", "mixture",
                        extra={"seed": 5})
    if name.startswith("decode_96k_b24_"):   # the pages' decode shape: batch 24, 96K contexts
        frac = name.rsplit("_", 1)[1]        # routed fraction "25" or "6.25" (sparsity 75 / 93.75%)
        return Workload(name, 24, 98304 + 256, 32, 2, 128, 64, 1.5, g.get(name, 8.0), "bf16", "planted",
                        extra={"seed": 6, "q_rows": (98304, 256), "prefix": 98304, "steps": 256,
                               "target": float(frac) / 100})
    if name == "mixture_32k_b32":   # profiling case of the long-row routing kernel: the 128K sweep's
        # inputs at n=32768 with 32-key chunks (T = 1024 > 512), alpha 1.5, gamma 1
        return Workload(name, 1, 32768, 16, 2, 128, 32, 1.5, 1.0, "bf16", "mixture", extra={"seed": 5})
    raise KeyError(name)


PREFILL_64K = ["prefill_64k_50", "prefill_64k_25", "prefill_64k_12.5"]
SWEEP_128K = [f"sweep_128k_{a}_{B}" for a in ("1.25", "1.5", "2.0") for B in (32, 64, 128)]
DECODE_96K = ["decode_96k_b24_25", "decode_96k_b24_6.25"]
