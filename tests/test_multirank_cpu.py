"""The N > 1 launch path of bench.py on the CPU: world_size 2, gloo, 127.0.0.1.

The path shards by replica (each rank runs its own copy of the workload; no data-path
collective), so what multi-rank code exists is the timing plumbing: a barrier around the timed
region, the max over ranks of the device time, and rank 0 alone printing the JSON line.  These
tests run that plumbing with real gloo process groups; nothing touches a GPU.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_RANKS_SCRIPT = r"""
import os, sys
sys.path.insert(0, {root!r})
import bench
r = bench.Ranks(want_gpu=False)
assert r.world == 2 and r.dist is not None and r.backend == "gloo"
r.barrier()
got = r.max(10.0 + 5.0 * r.rank)          # rank-dependent timings: the max must come back on every rank
assert got == 15.0, got
got = r.max(-1.0 - r.rank)
assert got == -1.0, got
r.barrier()
r.close()
print("rank", r.rank, "ok")
"""


def _torchrun(args, timeout):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}"] + args
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def test_ranks_barrier_and_max_over_two_gloo_ranks(tmp_path):
    script = tmp_path / "ranks_probe.py"
    script.write_text(_RANKS_SCRIPT.format(root=ROOT))
    r = _torchrun([str(script)], timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert r.stdout.count("ok") == 2


def test_reference_arm_under_torchrun_prints_one_line_from_rank0():
    """`bench.py --impl reference` launched like the scaling run (two ranks): rank 0 times the
    oracle on a bounded sample and prints one JSON line; rank 1 exits 0 without work."""
    r = _torchrun(["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"], timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
