#!/usr/bin/env python
"""Benchmark of the DashAttention forward pass on B200.

Default (N=1): the 1B-class prefill layer (b=1, n=32768, 16 query / 2 KV heads, d=128, chunk 64,
alpha 1.5, gamma tuned for 25% routed chunks), one step = Stage 0 + Stage 1 + Stage 2 over the
whole sequence, plus the decode workload (b=8, 131072-token caches, 32/2 heads, one append +
decode per step) reported under "decode", and the backward pass of the prefill workload (dQ, dK,
dV, dqbar) reported under "backward".  Under torchrun every rank runs its own replica
(no data-path collective): scaling is weak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dash|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "prefill Mtok/s and decode µs/token at 32K–128K ctx; % of HBM / bf16 TC roofline"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes per launch of a Stage 2 kernel (dram__bytes_read.sum + dram__bytes_write.sum from one
# ncu capture of the current kernel on that workload), keyed by (kernel, workload); absent until
# the current kernel has been captured.
STAGE2_TRAFFIC = {("attend_prefill_tc_kernel (tcgen05, one tile per block)", "prefill_32k"): 314.5e6}


def stage2_kernel_name():
    sel = os.environ.get("DASH_STAGE2", "")
    if sel.startswith("m"):
        return "attend_prefill_mma_kernel (mma.sync)"
    if sel.startswith("p"):
        return "attend_pair_kernel (tcgen05, two tiles per block)"
    return "attend_prefill_tc_kernel (tcgen05, one tile per block)"

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK), "fallback"


def args_():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="dash", choices=["dash", "reference"])
    ap.add_argument("--workload", default="prefill_32k")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--only-backward", action="store_true",
                    help="time the backward pass of the workload alone and print its object")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=16384)
    ap.add_argument("--sweep", action="store_true",
                    help="time the 64K sparsity sweep and the 128K alpha x chunk-size sweep (one line each)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave the sweeps out of the default line (they run at N=1 only)")
    ap.add_argument("--sweep-steps", type=int, default=3)
    ap.add_argument("--sweep-decode-steps", type=int, default=64)
    return ap.parse_args()


# ---------------------------------------------------------------------------------------- ranks
class Ranks:
    def __init__(self, want_gpu=True):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.dist = None
        if self.world > 1:
            import datetime

            import torch
            import torch.distributed as dist
            backend = "nccl" if (want_gpu and torch.cuda.is_available()) else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
            self.dist = dist
            self.backend = backend

    def barrier(self):
        if self.dist:
            self.dist.barrier()

    def max(self, x: float) -> float:
        """Max over ranks (timing only; not a data-path collective)."""
        if not self.dist:
            return x
        import torch
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist:
            self.dist.destroy_process_group()


# ---------------------------------------------------------------------------------------- clocks
class Clocks:
    """Samples nvidia-smi clocks / throttle reasons while the timed region runs."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.index), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for nm, v in zip(names, f[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------- prefill
def stage2_routed_flops(counts, n, B, g, d, hq):
    """4 d sum_{b,h,i} (|S_i^r| B + |D_i|): routed chunks' tokens plus the diagonal tokens."""
    diag = sum((i % B) + 1 for i in range(n))
    return 4.0 * d * (float(counts.sum()) * B * g + counts.shape[0] * hq * diag)


def stage2_executed_flops(pf, wl, counts):
    """FLOPs the tensor-core Stage 2 executes: a tile of 128 query rows (128/g positions, in the
    order Stage 2 tiled them) walks the union of its positions' routed chunks and diagonal chunks,
    and every walked unit of keys costs 4 d flops per (row, key) for all 128 rows.  None when
    the default Stage 2 is not the grouped tensor-core kernel for this shape."""
    import torch
    from adaptive_sparse_hierarchical_b200 import _lib as L

    g, B, n, d = wl.h_q // wl.h_kv, wl.chunk, wl.n, wl.d
    if wl.dtype != "bf16" or d != 128 or B not in (32, 64, 128) or 128 % g:
        return None
    off = L.dash_prefill_order_offset(pf.p)
    P, CPT = 128 // g, (2 if B == 32 else 1)
    nb = wl.batch * wl.h_kv
    if off >= 0:
        order = pf.workspace[off: off + nb * n * 4].view(torch.int32).cpu().numpy().reshape(nb, n)
    else:
        order = np.broadcast_to(np.arange(n, dtype=np.int64), (nb, n))
    idx = pf.chunk_idx.cpu().numpy().reshape(nb, -1)
    cnt = counts.reshape(nb, n).astype(np.int64)
    pos = np.arange(n, dtype=np.int64)
    c = pos // B
    tri = B * c * (c - 1) // 2 + (pos - c * B) * c
    units = (n // B + CPT) // CPT + 1
    total = 0
    for x in range(nb):
        inv = np.empty(n, dtype=np.int64)
        inv[order[x]] = pos
        tile = inv // P
        tot = int(cnt[x].sum())
        rep_pos = np.repeat(pos, cnt[x])
        start = np.repeat(np.cumsum(cnt[x]) - cnt[x], cnt[x])
        ent = idx[x][np.repeat(tri, cnt[x]) + (np.arange(tot) - start)].astype(np.int64)
        keys = np.concatenate([tile[rep_pos] * units + ent // CPT, tile * units + c // CPT])
        total += np.unique(keys).size
    return 4.0 * d * 128 * B * CPT * total


def prefill_launches(wl):
    """Kernels of this library one prefill step launches: Stage 0, Stage 1, Stage 2, plus the
    position grouping ahead of the tensor-core Stage 2 (g = 8 or 16) and, for rows of more than
    512 chunks, the per-shape routing kernel that recomputes overflowed position blocks."""
    g = wl.h_q // wl.h_kv
    tc = wl.dtype == "bf16" and wl.d == 128
    group = tc and wl.chunk in (32, 64, 128) and g in (8, 16) and os.environ.get("DASH_CLUSTER", "") != "0"
    long_rows = tc and wl.n // wl.chunk > 512 and g in (4, 8, 16)
    return 3 + int(group) + int(long_rows)


def run_prefill(wl, steps, warmup, ranks, pk, pk_kind, x=None, lite=False):
    import torch
    import adaptive_sparse_hierarchical_b200 as D

    dev = torch.device("cuda", ranks.local)
    x = wl.make() if x is None else x
    tq = {k: torch.from_numpy(x[k]).to(dev, torch.bfloat16) for k in ("Q", "K", "V")}
    qbar = torch.from_numpy(x["qbar"]).to(dev)
    pf = D.Prefill(tq["Q"], tq["K"], tq["V"], qbar, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma,
                   inv_sigma=wl.inv_sigma, want_route=True)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(rec=None):
        if rec:
            rec[0].record(stream)
        pf.stage(0)
        if rec:
            rec[1].record(stream)
        pf.stage(1)
        if rec:
            rec[2].record(stream)
        pf.stage(2)
        if rec:
            rec[3].record(stream)

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    counts = pf.counts.cpu().numpy()
    flops = stage2_routed_flops(counts, wl.n, wl.chunk, wl.h_q // wl.h_kv, wl.d, wl.h_q)
    recs = [[ev() for _ in range(4)] for _ in range(steps)]
    ranks.barrier()
    torch.cuda.synchronize(dev)
    with Clocks(ranks.local) as clk:
        for k in range(steps):
            flush.fill_(k & 0xff)                 # evict K/V/Q from L2 between steps (not timed)
            step(recs[k])
        torch.cuda.synchronize(dev)
    ranks.barrier()
    st = [[recs[k][j].elapsed_time(recs[k][j + 1]) for j in range(3)] for k in range(steps)]
    per_step = [sum(s) for s in st]
    ms = ranks.max(statistics.mean(per_step))
    stage_ms = [statistics.mean(s[j] for s in st) for j in range(3)]
    t2 = stage_ms[2] / 1e3
    achieved = flops / t2 / 1e12
    peak = pk["bf16_tflops"]
    tokens = wl.batch * wl.n
    out = {
        "ms_per_step": ms, "value": ranks.world * tokens / (ms / 1e3) / 1e6,
        "stages_ms": {"stage0_summary": stage_ms[0], "stage1_route": stage_ms[1], "stage2_attend": stage_ms[2]},
        "routed_fraction": float(counts.sum()) / (wl.batch * wl.h_kv * sum(i // wl.chunk for i in range(wl.n))),
        "roofline": {"kernel": stage2_kernel_name(), "bound": "tensor", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": STAGE2_TRAFFIC.get((stage2_kernel_name(), wl.name)),
                     "peak_kind": f"bf16 dense burst, of {pk_kind}",
                     "flops_per_launch": flops, "launch_ms": stage_ms[2]},
        "clocks": clk.summary(),
        "gpu_launches": prefill_launches(wl) * steps,
    }
    try:
        ex = stage2_executed_flops(pf, wl, counts)
    except Exception as e:   # a diagnostic: reported, not fatal
        ex, out["stage2_work_error"] = None, f"{type(e).__name__}: {e}"[:200]
    if ex:
        out["stage2_work"] = {"routed_tflop": flops / 1e12, "executed_tflop": ex / 1e12,
                              "executed_over_routed": ex / flops,
                              "executed_tflops": ex / t2 / 1e12, "executed_frac": ex / t2 / 1e12 / peak,
                              "note": "executed: every 128-row tile's union of its positions' routed and "
                                      "diagonal chunks, all 128 rows, in the order Stage 2 tiled them"}
    if lite:   # sweep mode: the device-timed step and the per-row support only
        c = counts.reshape(-1, wl.n)[:, wl.chunk:].astype("float64")
        vis = (np.arange(wl.n) // wl.chunk)[wl.chunk:].astype("float64")
        frac = (c / vis).reshape(-1)
        out["support_fraction_deciles"] = [round(float(v), 4) for v in np.quantile(frac, np.linspace(0.1, 0.9, 9))]
        out["support_chunks_deciles"] = [int(v) for v in np.quantile(c.reshape(-1), np.linspace(0.1, 0.9, 9))]
        # per-row support histogram: rows (position, KV head) by routed / visible chunks
        edges = [0.0, 0.005, 0.01, 0.02, 0.05, 0.1, 0.2, 0.3, 0.5, 0.75, 1.0]
        hist, _ = np.histogram(frac, bins=edges)
        out["support_histogram"] = {"bin_edges": edges, "rows": [int(h) for h in hist]}
        del pf
        return out
    # e2e: host (pinned) inputs copied in, result copied out, every step, through the public API.
    # Two device buffer sets and three streams (copy in, compute, copy out): step k+1's inputs
    # cross PCIe while step k computes and step k-1's output comes back; every copy of every step
    # is inside the timed region (first copy-in to last copy-out).
    hq = {k: tq[k].cpu().pin_memory() for k in ("Q", "K", "V")}
    ho = [torch.empty(tq["Q"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dbuf = [tq] + [{k: torch.empty_like(tq[k]) for k in ("Q", "K", "V")}]
    pfs = [pf] + [D.Prefill(dbuf[1]["Q"], dbuf[1]["K"], dbuf[1]["V"], qbar, chunk=wl.chunk, alpha=wl.alpha,
                            gamma=wl.gamma, inv_sigma=wl.inv_sigma)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [ev() for _ in range(2)]
    ev_cmp = [ev() for _ in range(2)]
    ev_out = [ev() for _ in range(2)]

    def e2e_steps(n, start=None, stop=None):
        for k in range(n):
            i = k & 1
            if k >= 2:
                s_in.wait_event(ev_cmp[i])      # step k-2 is done reading buffer set i
            with torch.cuda.stream(s_in):
                if k == 0 and start is not None:
                    start.record(s_in)
                for name in ("Q", "K", "V"):
                    dbuf[i][name].copy_(hq[name], non_blocking=True)
                ev_in[i].record(s_in)
            s_cmp.wait_event(ev_in[i])
            if k >= 2:
                s_cmp.wait_event(ev_out[i])     # step k-2's output has left the device
            pfs[i](stream=s_cmp)
            ev_cmp[i].record(s_cmp)
            s_out.wait_event(ev_cmp[i])
            with torch.cuda.stream(s_out):
                ho[i].copy_(pfs[i].O, non_blocking=True)
                ev_out[i].record(s_out)
        if stop is not None:
            s_out.wait_stream(s_in)
            s_out.wait_stream(s_cmp)
            stop.record(s_out)

    e2e_steps(4)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    e_s, e_e = ev(), ev()
    e2e_steps(steps, e_s, e_e)
    torch.cuda.synchronize(dev)
    ems = ranks.max(e_s.elapsed_time(e_e) / steps)
    nbytes = lambda t: t.numel() * t.element_size()
    out["e2e"] = {"value": ranks.world * tokens / (ems / 1e3) / 1e6, "unit": "Mtok/s", "ms_per_step": ems,
                  "h2d_bytes_per_step": sum(nbytes(hq[k]) for k in hq), "d2h_bytes_per_step": nbytes(ho[0]),
                  "pipelining": "double-buffered: copy-in of step k+1 and copy-out of step k-1 overlap step k"}
    del dbuf[1], pfs[1]
    out["dense_causal"] = dense_denominators(wl, tq, qbar, pf, steps, flush, ms, dev)
    out["stage2_list_vs_bitmask"] = stage2_variants(wl, tq, qbar, steps, flush, dev)
    out["_inputs"] = x
    return out


def run_backward(wl, steps, warmup, ranks, pk, pk_kind, x=None, cpu=False):
    """The backward pass (dash_backward) of the prefill workload: gradients of Q, K, V and qbar
    for a seeded dO, device-timed with CUDA events, L2 flushed between steps.  Algorithmic FLOPs:
    the five Stage 2 products of a softmax-attention backward (S, dP, dV, dQ, dK: 10 d per routed
    or diagonal (row, key) pair, 2.5x the forward's 4 d); the Stage 1 / Stage 0 chain is not
    counted."""
    import torch
    import adaptive_sparse_hierarchical_b200 as D

    dev = torch.device("cuda", ranks.local)
    x = wl.make() if x is None else x
    tq = {k: torch.from_numpy(x[k]).to(dev, torch.bfloat16) for k in ("Q", "K", "V")}
    qbar = torch.from_numpy(x["qbar"]).to(dev)
    pf = D.Prefill(tq["Q"], tq["K"], tq["V"], qbar, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma,
                   inv_sigma=wl.inv_sigma, want_route=True)
    pf()
    g = torch.Generator(device=dev).manual_seed(1234)
    dO = torch.randn(tq["Q"].shape, device=dev, generator=g).to(torch.bfloat16)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(max(warmup, 3)):
        pf.backward(dO)
    torch.cuda.synchronize(dev)
    counts = pf.counts.cpu().numpy()
    flops = 2.5 * stage2_routed_flops(counts, wl.n, wl.chunk, wl.h_q // wl.h_kv, wl.d, wl.h_q)
    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    ranks.barrier()
    torch.cuda.synchronize(dev)
    with Clocks(ranks.local) as clk:
        for k in range(steps):
            flush.fill_(k & 0xff)
            recs[k][0].record(stream)
            pf.backward(dO)
            recs[k][1].record(stream)
        torch.cuda.synchronize(dev)
    ranks.barrier()
    ms = ranks.max(statistics.mean(r[0].elapsed_time(r[1]) for r in recs))
    achieved = flops / (ms / 1e3) / 1e12
    T = wl.n // wl.chunk
    launches = 2 + (5 if T > 0 else 0)
    del pf
    torch.cuda.empty_cache()
    base = oracle_backward_sample(wl, x, counts) if cpu else None
    return {"workload": f"{wl.name} backward: dQ, dK, dV, dqbar of sum(dO * O), dO ~ N(0, 1) bf16",
            "cpu_baseline": base,
            "ms_per_step": ms, "tokens_per_s_M": ranks.world * wl.batch * wl.n / (ms / 1e3) / 1e6,
            "roofline": {"kernel": "bwd_rows_kernel + bwd_keys_kernel (fp32 CUDA cores)", "bound": "tensor",
                         "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_tflops"], "traffic": None,
                         "peak_kind": f"bf16 dense burst, of {pk_kind}", "flops_per_step": flops},
            "clocks": clk.summary(), "steps": steps, "gpu_launches": launches * steps}


def oracle_backward_sample(wl, x, counts, ntok=2048):
    """Time the float64 oracle's backward on a bounded sample of the workload: the first `ntok`
    positions of every sequence (all heads; routing is causal, so these rows route exactly as in
    the full sequence).  Rows near the start see fewer chunks than the average row, so the
    per-token rate overstates the oracle's full-sequence rate; the algorithmic rate on the same
    prefix (2.5x the forward's Stage 2 FLOPs of those rows) is comparable with the GPU's."""
    import oracle
    from adaptive_sparse_hierarchical_b200 import inputs

    dO = inputs.round_bf16(np.random.default_rng(5).standard_normal((wl.batch, ntok, wl.h_q, wl.d)))
    t0 = time.perf_counter()
    oracle.backward(x["Q"][:, :ntok], x["K"][:, :ntok], x["V"][:, :ntok], x["qbar"], dO, chunk=wl.chunk,
                    alpha=wl.alpha, gamma=wl.gamma, inv_sigma=wl.inv_sigma)
    secs = time.perf_counter() - t0
    flops = 2.5 * stage2_routed_flops(counts[..., :ntok], ntok, wl.chunk, wl.h_q // wl.h_kv, wl.d, wl.h_q)
    return {"value": wl.batch * ntok / secs / 1e6, "unit": "Mtok/s", "tflops": flops / secs / 1e12,
            "cores": min(oracle.num_threads(), wl.batch * wl.h_kv), "kind": "oracle",
            "sample": f"oracle.backward on the first {ntok} positions of each sequence, all heads ({secs:.1f} s); "
                      f"the oracle parallelises over (sequence, KV head) pairs"}


def stage2_variants(wl, tq, qbar, steps, flush, dev):
    """Stage 2 driven by the compact ascending chunk lists (the default) and by the bit-packed
    block mask M_i (32 chunks per word, as the paper review's Stage 2 kernel walks it) on the same
    routes, device-timed side by side (L2 flushed); the two outputs must agree bit for bit."""
    import torch
    import adaptive_sparse_hierarchical_b200 as D
    from adaptive_sparse_hierarchical_b200 import _lib as L

    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    pfm = D.Prefill(tq["Q"], tq["K"], tq["V"], qbar, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma,
                    inv_sigma=wl.inv_sigma, want_route=True, bitmask=True)
    try:
        pfm()
        torch.cuda.synchronize(dev)
        o_list = pfm.O.clone()

        def timed(stage):
            for _ in range(3):
                pfm.stage(stage)
            torch.cuda.synchronize(dev)
            tot = 0.0
            for k in range(steps):
                flush.fill_(k & 0xff)
                a, b = ev(), ev()
                a.record(stream)
                pfm.stage(stage)
                b.record(stream)
                torch.cuda.synchronize(dev)
                tot += a.elapsed_time(b)
            return tot / steps

        res = {"stage1_with_bitmask_output_ms": timed(L.DASH_STAGE1), "stage2_list_ms": timed(L.DASH_STAGE2)}
        res["stage2_bitmask_ms"] = timed(L.DASH_STAGE2_BITMASK)
        torch.cuda.synchronize(dev)
        res["bit_identical"] = bool(torch.equal(pfm.O, o_list))
        res["error_word"] = pfm.error_word()
        return res
    except Exception as e:   # reported, not fatal
        return {"error": f"{type(e).__name__}: {e}"[:300]}
    finally:
        del pfm


def dense_denominators(wl, tq, qbar, pf, steps, flush, sparse_ms, dev):
    """Same-box dense causal attention on the same Q, K, V (context for the sparse step, not part
    of `value`): (a) this library at gamma = 0, where every visible chunk is routed with bias 0 and
    the method reduces to dense causal attention; (b) torch's scaled_dot_product_attention."""
    import torch
    import adaptive_sparse_hierarchical_b200 as D

    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(fn, n):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        tot = 0.0
        for k in range(n):
            flush.fill_(k & 0xff)
            a, b = ev(), ev()
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            tot += a.elapsed_time(b)
        return tot / n

    res = {}
    pfd = D.Prefill(tq["Q"], tq["K"], tq["V"], qbar, chunk=wl.chunk, alpha=wl.alpha, gamma=0.0,
                    inv_sigma=wl.inv_sigma)
    res["own_kernels_gamma0_ms"] = timed(pfd, steps)
    res["own_stage2_gamma0_ms"] = timed(lambda: pfd.stage(2), steps)
    del pfd
    try:
        import torch.nn.functional as F
        q = tq["Q"].transpose(1, 2).contiguous()
        k = tq["K"].transpose(1, 2).contiguous()
        v = tq["V"].transpose(1, 2).contiguous()
        res["torch_sdpa_ms"] = timed(lambda: F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True),
                                     steps)
        del q, k, v
    except Exception as e:   # pragma: no cover - backend availability differs by build
        res["torch_sdpa_ms"] = None
        res["torch_sdpa_error"] = str(e)[:200]
    res["sparse_step_ms"] = sparse_ms
    res["speedup_vs_own_dense"] = res["own_kernels_gamma0_ms"] / sparse_ms
    if res.get("torch_sdpa_ms"):
        res["speedup_vs_torch_sdpa"] = res["torch_sdpa_ms"] / sparse_ms
    return res


# ---------------------------------------------------------------------------------------- decode
def run_decode(steps, warmup, ranks, pk, pk_kind, name="decode_128k", paged=True):
    import torch
    import adaptive_sparse_hierarchical_b200 as D
    from adaptive_sparse_hierarchical_b200 import workloads as W

    wl = W.get(name)
    dev = torch.device("cuda", ranks.local)
    x = wl.make()
    prefix = wl.extra["prefix"]
    nst = min(steps, wl.extra["steps"])
    st = D.DecodeState(wl.batch, wl.n, wl.h_q, wl.h_kv, wl.d, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma,
                       device=dev, qbar=torch.from_numpy(x["qbar"]).to(dev))
    counts = torch.zeros((wl.batch, wl.h_kv), dtype=torch.int32, device=dev)
    idx = torch.zeros((wl.batch, wl.h_kv, st.T), dtype=torch.int32, device=dev)
    bias = torch.zeros((wl.batch, wl.h_kv, st.T), dtype=torch.float32, device=dev)
    st.route = D.route_out(counts, idx, bias)
    K0 = torch.from_numpy(x["K"][:, :prefix]).to(dev, torch.bfloat16)
    V0 = torch.from_numpy(x["V"][:, :prefix]).to(dev, torch.bfloat16)
    kn = torch.from_numpy(np.ascontiguousarray(x["K"][:, prefix:prefix + wl.extra["steps"]].swapaxes(0, 1))).to(dev, torch.bfloat16)
    vn = torch.from_numpy(np.ascontiguousarray(x["V"][:, prefix:prefix + wl.extra["steps"]].swapaxes(0, 1))).to(dev, torch.bfloat16)
    qn = torch.from_numpy(np.ascontiguousarray(x["Q"].swapaxes(0, 1))).to(dev, torch.bfloat16)
    del x
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    snapshot = (st.K.clone(), st.V.clone())

    def reset():
        st.K.copy_(snapshot[0]); st.V.copy_(snapshot[1])
        st.seqlens.fill_(prefix)
        D.dash_summary_build(st.p, st.K, st.qbar, st.seqlens, st.kbar, st.state)

    st.K[:, :prefix].copy_(K0); st.V[:, :prefix].copy_(V0)
    snapshot = (st.K.clone(), st.V.clone())
    del K0, V0
    reset()
    for s in range(max(warmup, 3)):
        st.step(qn[s], kn[s], vn[s])
    reset()
    torch.cuda.synchronize(dev)
    # eager pass: per-kernel-group times (append / decode) and the routed counts
    evs = [(ev(), ev(), ev()) for _ in range(nst)]
    routed = []
    for s in range(nst):
        evs[s][0].record(stream)
        st.append(kn[s], vn[s])
        evs[s][1].record(stream)
        st.decode(qn[s])
        evs[s][2].record(stream)
        if s % 50 == 0:
            routed.append((s, counts.clone()))
    torch.cuda.synchronize(dev)
    eager_ms = statistics.mean(a.elapsed_time(c) for a, b, c in evs)
    dec_ms = [b.elapsed_time(c) for a, b, c in evs]
    # timed pass: each step = one copy of the step's q, k, v (packed back to back, as a model's
    # projection would write them) into the graph's staging buffer + one graph replay
    reset()
    st.graph_step(qn[0], kn[0], vn[0])   # eager first step, then capture
    qkv = [st.pack(qn[s], kn[s], vn[s]) for s in range(nst)]
    torch.cuda.synchronize(dev)
    ranks.barrier()
    gevs = [(ev(), ev()) for _ in range(nst - 1)]
    with Clocks(ranks.local) as clk:
        for s in range(1, nst):
            gevs[s - 1][0].record(stream)
            st.graph_step_packed(qkv[s])
            gevs[s - 1][1].record(stream)
        torch.cuda.synchronize(dev)
    ranks.barrier()
    step_ms = [a.elapsed_time(b) for a, b in gevs]
    ms = ranks.max(statistics.mean(step_ms))
    # routed K+V bytes per step (numerator of the HBM roofline), from sampled steps' counts
    byts = []
    for s, c in routed:
        L = prefix + s + 1
        diag = (L - 1) % wl.chunk + 1
        byts.append(2 * wl.d * 2 * (float(c.sum()) * wl.chunk + wl.batch * wl.h_kv * diag))
    bps = statistics.mean(byts)
    achieved = bps / (ms / 1e3) / 1e9   # whole graph step (append + route + attend + merge)
    res = {"workload": f"{name}: b={wl.batch}, {prefix}-token caches (+1 per step), {wl.h_q}/{wl.h_kv} heads, "
                       f"d={wl.d}, B={wl.chunk}, alpha {wl.alpha}, gamma {wl.gamma} "
                       f"(~{100 * wl.extra.get('target', 0.25):g}% routed)",
           "us_per_step": ms * 1e3, "us_per_step_eager": eager_ms * 1e3,
           "timing": "per step: one copy of the packed q, k, v into the captured graph's staging buffer + graph replay (append + decode)",
           "steps": nst, "append_us": statistics.mean(a.elapsed_time(b) for a, b, c in evs) * 1e3,
           "decode_us": statistics.mean(dec_ms) * 1e3,
           "routed_fraction": float(routed[-1][1].sum()) / (wl.batch * wl.h_kv * ((prefix + routed[-1][0]) // wl.chunk)),
           "roofline": {"kernel": "decode step (append, route, dec_attend_tma_kernel, merge)", "bound": "hbm",
                        "achieved": achieved,
                        "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": None,
                        "peak_kind": f"hbm copy, of {pk_kind}", "bytes_per_step": bps},
           "clocks": clk.summary(), "gpu_launches": 4 * (nst - 1),   # append, routing, attend, merge
           "l2": f"KV caches ({2 * wl.batch * wl.n * wl.h_kv * wl.d * 2 / 1e9:.2f} GB) larger than L2"}
    res["us_per_token"] = res["us_per_step"] / wl.batch   # per sequence-token, one GPU
    if not paged:
        return res
    try:
        res["paged"] = paged_decode(wl, st, qn, kn, vn, prefix, nst, reset, stream, bps, pk, pk_kind, ranks)
        res["gpu_launches"] += res["paged"]["gpu_launches"]
    except Exception as e:   # reported, not fatal: the contiguous numbers above stand
        res["paged"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    return res


def paged_decode(wl, st, qn, kn, vn, prefix, nst, reset, stream, bps, pk, pk_kind, ranks):
    """The same decode steps on paged K/V pools (128-token pages, pool pages in a seeded random
    order): eager append + decode per step, device-timed; the first step's output is compared
    with the contiguous caches' bit for bit."""
    import torch
    import adaptive_sparse_hierarchical_b200 as D

    dev = st.K.device
    psz = 128
    per_seq = (wl.n + psz - 1) // psz
    npages = wl.batch * per_seq
    table = torch.from_numpy(np.random.default_rng(9).permutation(npages).reshape(wl.batch, per_seq).astype(np.int32))
    pg = D.PagedDecodeState(wl.batch, wl.n, wl.h_q, wl.h_kv, wl.d, chunk=wl.chunk, alpha=wl.alpha, gamma=wl.gamma,
                            page_size=psz, num_pages=npages, page_table=table, device=dev, qbar=st.qbar)
    reset()
    pg.fill(st.K[:, :prefix], st.V[:, :prefix], [prefix] * wl.batch)
    o_ref = st.step(qn[0], kn[0], vn[0]).clone()
    o = pg.step(qn[0], kn[0], vn[0])
    torch.cuda.synchronize(dev)
    same = bool(torch.equal(o, o_ref))
    for s in range(1, 4):
        pg.step(qn[s], kn[s], vn[s])
    torch.cuda.synchronize(dev)
    # restart both from the prefix for the timed steps
    pg.seqlens.fill_(prefix)
    D.dash_summary_build_paged(pg.p, pg.pk, pg.K, pg.qbar, pg.seqlens, pg.kbar, pg.state)
    torch.cuda.synchronize(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    evs = [(ev(), ev()) for _ in range(nst)]
    ranks.barrier()
    for s in range(nst):
        evs[s][0].record(stream)
        pg.step(qn[s], kn[s], vn[s])
        evs[s][1].record(stream)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    ms = ranks.max(statistics.mean(a.elapsed_time(b) for a, b in evs))
    achieved = bps / (ms / 1e3) / 1e9
    del pg
    torch.cuda.empty_cache()
    return {"workload": f"the decode steps above on paged pools: {psz}-token pages, {npages} pages in a seeded "
                        f"random order", "us_per_step_eager": ms * 1e3, "us_per_token": ms * 1e3 / wl.batch,
            "matches_contiguous": same, "steps": nst,
            "roofline": {"kernel": "decode step, paged (append, route, dec_attend_tma_kernel, merge)", "bound": "hbm",
                         "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "traffic": None, "peak_kind": f"hbm copy, of {pk_kind}",
                         "bytes_per_step": bps},
            "gpu_launches": 4 * nst}


# ---------------------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, x, nrows):
    """Time the float64 oracle on a bounded sample of the workload: Stage 0 over the whole
    sequence (its share per token is charged) plus Stages 1-2 for `nrows` evenly spaced query
    positions with all heads.  Returns (tokens per second, seconds, threads)."""
    import oracle

    pos = np.linspace(0, wl.n - 1, nrows).astype(np.int32)
    t0 = time.perf_counter()
    kbar = oracle.stage0(x["K"], x["qbar"], wl.chunk)
    t1 = time.perf_counter()
    oracle.rows(x["Q"][:, pos], np.broadcast_to(pos, (wl.batch, nrows)), x["K"], x["V"], kbar, chunk=wl.chunk,
                alpha=wl.alpha, gamma=wl.gamma, inv_sigma=wl.inv_sigma)
    t2 = time.perf_counter()
    secs = (t1 - t0) * nrows / wl.n + (t2 - t1)
    return wl.batch * nrows / secs, t2 - t0, oracle.num_threads()


def reference_arm(args, ranks):
    """The CPU oracle as the reference arm: each step is a bounded sample of the workload."""
    from adaptive_sparse_hierarchical_b200 import workloads as W

    wl = W.get(args.workload)
    x = wl.make()
    nrows = 256
    for _ in range(args.warmup):
        oracle_sample(wl, x, 8)
    vals, secs = [], []
    for _ in range(args.steps):
        v, s, thr = oracle_sample(wl, x, nrows)
        vals.append(v)
        secs.append(s)
    tps = statistics.mean(vals)
    value = tps / 1e6
    sample = (f"{nrows} evenly spaced query positions (all {wl.h_q} heads) per step + Stage 0 share, "
              f"of {wl.name}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Mtok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(secs) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, args),
            "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(wl, args):
    return {"workload": f"{wl.name}: b={wl.batch}, n={wl.n}, h_q={wl.h_q}, h_kv={wl.h_kv}, d={wl.d}, "
                        f"chunk={wl.chunk}, alpha={wl.alpha}, gamma={wl.gamma}, sigma=1",
            "batch": wl.batch, "seq_len": wl.n, "h_q": wl.h_q, "h_kv": wl.h_kv, "d_h": wl.d, "chunk": wl.chunk,
            "alpha": wl.alpha, "gamma": wl.gamma, "parallelism": f"replicas x{args.gpus}",
            "l2": "flushed between steps (256 MB write, outside the per-step events)"}


def run_sweep(args, ranks, pk, pk_kind, steps=None, decode_steps=None, emit=True):
    """The 8B-class 64K prefill at 50 / 25 / 12.5% routed and the 128K alpha x chunk-size sweep on
    Gaussian-mixture inputs: per workload the device-timed step, Mtok/s, Stage 2 roofline and the
    per-row support (routed chunks / visible chunks) deciles.  Inputs shared by several workloads
    are drawn once."""
    import gc
    from adaptive_sparse_hierarchical_b200 import workloads as W

    steps = args.steps if steps is None else steps
    decode_steps = args.decode_steps if decode_steps is None else decode_steps
    lines = []
    cache = {}
    for name in W.PREFILL_64K + W.SWEEP_128K:
        wl = W.get(name)
        key = (wl.recipe, wl.extra.get("seed"), wl.batch, wl.n, wl.h_q, wl.h_kv, wl.d)
        if key not in cache:
            cache.clear()
            gc.collect()
            cache[key] = wl.make()
        r = run_prefill(wl, steps, args.warmup, ranks, pk, pk_kind, x=cache[key], lite=True)
        line = {"sweep": name, "metric": "prefill Mtok/s", "value": r["value"], "unit": "Mtok/s",
                "ms_per_step": r["ms_per_step"], "stages_ms": r["stages_ms"], "routed_fraction": r["routed_fraction"],
                "stage2_work": r.get("stage2_work"),
                "stage2_roofline_frac": r["roofline"]["frac"], "stage2_routed_tflops": r["roofline"]["achieved"],
                "support_fraction_deciles": r["support_fraction_deciles"],
                "support_chunks_deciles": r["support_chunks_deciles"],
                "support_histogram": r["support_histogram"], "roofline": r["roofline"],
                "gpu_launches": r["gpu_launches"], "clocks": r["clocks"],
                "config": {"batch": wl.batch, "seq_len": wl.n, "h_q": wl.h_q, "h_kv": wl.h_kv, "d_h": wl.d,
                           "chunk": wl.chunk, "alpha": wl.alpha, "gamma": wl.gamma}}
        lines.append(line)
        if emit and ranks.rank == 0:
            print(json.dumps(line), flush=True)
    cache.clear()
    gc.collect()
    # decode at the pages' own shape: batch 24, 96K contexts, 75% and 93.75% sparsity
    for name in W.DECODE_96K:
        r = run_decode(decode_steps, args.warmup, ranks, pk, pk_kind, name=name, paged=False)
        line = {"sweep": name, "metric": "decode us/token", "value": r["us_per_token"], "unit": "us/token",
                "higher_is_better": False, "us_per_step": r["us_per_step"], "routed_fraction": r["routed_fraction"],
                "roofline": r["roofline"], "clocks": r["clocks"], "steps": r["steps"], "workload": r["workload"],
                "gpu_launches": r["gpu_launches"]}
        lines.append(line)
        if emit and ranks.rank == 0:
            print(json.dumps(line), flush=True)
        gc.collect()
    return lines


def main():
    args = args_()
    if args.impl == "reference":
        ranks = Ranks(want_gpu=False) if int(os.environ.get("WORLD_SIZE", "1")) > 1 else Ranks(want_gpu=False)
        if ranks.rank == 0:
            reference_arm(args, ranks)
        ranks.close()
        return
    import torch
    from adaptive_sparse_hierarchical_b200 import workloads as W
    from adaptive_sparse_hierarchical_b200.build import build

    build()
    ranks = Ranks()
    torch.cuda.set_device(ranks.local)
    pk, pk_kind = peaks()
    if args.sweep:
        run_sweep(args, ranks, pk, pk_kind)
        ranks.close()
        return
    wl = W.get(args.workload)
    if args.only_backward:
        bw = run_backward(wl, args.steps, args.warmup, ranks, pk, pk_kind,
                          cpu=ranks.rank == 0 and ranks.world == 1 and not args.no_cpu_baseline)
        if ranks.rank == 0:
            print(json.dumps({"backward": bw}), flush=True)
        ranks.close()
        return
    pre = run_prefill(wl, args.steps, args.warmup, ranks, pk, pk_kind)
    x = pre.pop("_inputs")
    line = {"metric": METRIC, "value": pre["value"], "unit": "Mtok/s", "n_gpus": ranks.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": pre["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Gaussian inputs with planted chunk directions)",
            "config": config_of(wl, args), "roofline": pre["roofline"], "e2e": pre["e2e"],
            "gpu_launches": pre["gpu_launches"], "clocks": pre["clocks"], "stages_ms": pre["stages_ms"],
            "routed_fraction": pre["routed_fraction"], "dense_causal": pre["dense_causal"],
            "stage2_list_vs_bitmask": pre["stage2_list_vs_bitmask"], "stage2_work": pre.get("stage2_work")}
    if not args.no_decode:
        line["decode"] = run_decode(args.decode_steps, args.warmup, ranks, pk, pk_kind)
        line["gpu_launches"] += line["decode"]["gpu_launches"]
    if not args.no_backward:
        try:
            line["backward"] = run_backward(wl, max(2, min(args.steps, 5)), args.warmup, ranks, pk, pk_kind, x=x,
                                            cpu=ranks.rank == 0 and ranks.world == 1 and not args.no_cpu_baseline)
            line["gpu_launches"] += line["backward"]["gpu_launches"]
        except Exception as e:   # reported in the line; the forward numbers above stand
            line["backward"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if ranks.world == 1 and not args.no_sweep:
        # the 8B-class 64K prefill at 50 / 25 / 12.5% routed, the 128K alpha x chunk-size sweep with
        # its per-row support histogram, and the batch-24 decode at 96K (75% and 93.75% sparsity),
        # a few device-timed steps each (the inputs are generated outside the timed regions)
        try:
            line["sweeps"] = run_sweep(args, ranks, pk, pk_kind, steps=args.sweep_steps,
                                       decode_steps=args.sweep_decode_steps, emit=False)
            line["gpu_launches"] += sum(ln.get("gpu_launches", 0) for ln in line["sweeps"])
        except Exception as e:   # reported in the line; the numbers above stand
            line["sweeps"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if ranks.rank == 0 and ranks.world == 1 and not args.no_cpu_baseline:
        v, secs, thr = oracle_sample(wl, x, args.cpu_rows)
        line["cpu_baseline"] = {"value": v / 1e6, "unit": "Mtok/s", "cores": thr, "kind": "oracle",
                                "sample": f"{args.cpu_rows} evenly spaced query positions x {wl.h_q} heads + "
                                          f"Stage 0 share ({secs:.1f} s)"}
    if ranks.rank == 0:
        print(json.dumps(line), flush=True)
    ranks.close()


if __name__ == "__main__":
    main()
