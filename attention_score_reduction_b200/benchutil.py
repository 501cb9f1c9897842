"""Host-side helpers for timing runs: rank layout, cross-rank reduction of
device times, clock sampling and roofline arithmetic.  No kernel code."""
from __future__ import annotations

import csv
import io
import os
import statistics
import subprocess
import tempfile

import torch


def dist_env():
    """(rank, world, local_rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_salt(rank: int) -> int:
    """Seed salt of the independent context each rank compresses (weak scaling)."""
    return 1000 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value over all ranks (one all-reduce); identity for one rank."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling every 200 ms while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="kvzip_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = list(csv.reader(io.StringIO(open(self.path).read())))
        os.unlink(self.path)
        return summarize_clock_rows(rows)


def summarize_clock_rows(rows) -> dict:
    """Median SM clock, max clock and the throttle reasons seen Active."""
    sm, mx, reasons, n = [], None, set(), 0
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        r = [c.strip() for c in r]
        if len(r) < 9:
            continue
        try:
            sm.append(float(r[1]))
            mx = float(r[2])
        except ValueError:
            continue
        n += 1
        for name, val in zip(names, r[5:9]):
            if val.lower().startswith("active"):
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
            "reasons": sorted(reasons), "samples": n}


def load_peaks(path: str) -> dict:
    """Measured HBM GB/s and bf16 TF/s (generated file), else the machine's fallback."""
    import json
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def clock_peak_tflops(sms: int, sm_mhz: float) -> float:
    """Dense bf16 tensor peak at a given SM clock: each SM's tcgen05 pipe does one
    128 x 128 x 16 MMA in 64 cycles (8192 flop per clock)."""
    return sms * 8192.0 * sm_mhz * 1e6 / 1e12


def score_flops(B: int, G: int, n_in: int, n_c: int, d: int) -> dict:
    """Algorithmic QK^T flops of the two scoring passes for one chunk of B units.

    pass 1 forms every (row, key) logit a row's normaliser needs: R*n_c context
    pairs plus G*n_in*(n_in+1)/2 causal self pairs; pass 2 re-forms the R*n_c
    context logits.  2*d flops per pair."""
    R = G * n_in
    self_pairs = G * n_in * (n_in + 1) // 2
    return {"pass1": 2.0 * d * B * (R * n_c + self_pairs), "pass2": 2.0 * d * B * R * n_c}
