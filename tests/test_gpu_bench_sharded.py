"""bench.py's multi-GPU path (one context sharded over ranks) on one GPU.

Under torchrun, bench.py gives each rank H / N KV heads of every layer, scores
and compacts them locally and selects globally through the sharded selection
(histograms all-reduced per radix round, tie counts all-gathered).  Here two
ranks share cuda:0 and exchange through gloo (--dist-backend gloo), which runs
the same code as the NCCL run on several GPUs except for the collective
backend.  No kernel waits on another rank.  A small case: 2 layers of the 128K
LLaMA3.1-8B shape.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_two_ranks_sharded_on_one_gpu():
    from attention_score_reduction_b200 import build
    build.build()
    port = str(32500 + os.getpid() % 1000)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", port, "bench.py", "--gpus", "2",
           "--dist-backend", "gloo", "--layers", "2", "--steps", "1", "--warmup", "1",
           "--no-e2e", "--no-cpu", "--no-decode", "--no-variants"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]       # rank 0 prints the one line
    out = json.loads(lines[0])
    assert out["n_gpus"] == 2 and out["scaling"] == "strong"
    assert "sharded over 2 GPUs" in out["parallelism"]
    assert out["config"]["H"] == 8 and out["value"] > 0
    assert out["gpu_launches"] > 0
