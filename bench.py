#!/usr/bin/env python
"""KVzip scoring -> global top-r selection -> per-head compaction on B200.

One step = one whole context through the hot path: every reconstruction chunk
scored for all L x H units (two tensor-core passes per chunk), one global
selection over the L x H x n_c scores, one compaction of the kept K/V rows.
Default workload: LLaMA3.1-8B KV shape (32 layers x 8 KV heads, G = 4, d = 128)
with a 131072-token context scored in 64 chunks of 2048 (+16 prompt rows), r = 0.3.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Inputs are synthetic (seeded) and resident in
HBM for ``value`` (workloads whose chunk inputs do not fit are drawn per chunk
between timed launches); ``e2e`` repeats the step from pinned host buffers
through ``pipeline.compress_from_host`` with the uploads and the read-back
inside the timed region.  Under torchrun the context is sharded: each rank
holds H / N KV heads of every layer, scores and compacts them locally, and the
global selection exchanges one histogram per radix round and the tie counts
(strong scaling: one context per step over all ranks); times are the max over
ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_score_reduction_b200 import benchutil as bu  # noqa: E402
from attention_score_reduction_b200 import synth  # noqa: E402

METRIC = "context tokens scored/sec (all layers+heads) @LLaMA3.1-8B 128K; % bf16 TC peak"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per full launch of
# each scorer pass on the 128K LLaMA3.1-8B workload, from an ncu capture of the
# current kernels on one layer (8 units) scaled to the launch's 256 units (each
# unit streams its own keys, so traffic grows with the units).  Only passes
# whose kernel has not changed since their capture are listed.
NCU_TRAFFIC = {("llama8b_128k", 32, "score_pass1_lse"): 10.73e9,
               ("llama8b_128k", 32, "score_pass2_colmax"): 9.49e9}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b_128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--r", type=float, default=None, help="kept fraction (default: first of workload)")
    ap.add_argument("--chunk", type=int, default=None, help="override context rows per chunk")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the layer count (smaller cases for profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-attention table")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the head-level / ablation kernel timings")
    ap.add_argument("--only", choices=["select", "compact"], default=None,
                    help="time one kernel alone on synthetic inputs of the workload's shape "
                         "(a few hundred MB on the device; for profiling)")
    ap.add_argument("--dist-backend", choices=["nccl", "gloo"], default="nccl",
                    help="process-group backend under torchrun (gloo also runs several ranks "
                         "on one GPU, for testing the sharded path)")
    return ap.parse_args()


def workload(args):
    wl = synth.WORKLOADS[args.workload]
    if args.chunk:
        wl = wl.with_(m=args.chunk)
    if args.layers:
        wl = wl.with_(L=args.layers)
    return wl


def shard(wl, rank, world):
    """This rank's part of the context: H / world KV heads of every layer (the
    tensor-parallel layout), or L / world layers when the heads do not divide.
    Each shard draws its own synthetic inputs (a rank salt in the seed)."""
    if world == 1:
        return wl
    salt = wl.cfg_id + bu.rank_salt(rank)
    if wl.H % world == 0:
        return wl.with_(H=wl.H // world, cfg_id=salt)
    if wl.L % world == 0:
        return wl.with_(L=wl.L // world, cfg_id=salt)
    raise SystemExit(f"{world} ranks divide neither the {wl.H} heads nor the {wl.L} layers")


def config_dict(wl, r, resident=True):
    return {"workload": wl.name, "L": wl.L, "H": wl.H, "G": wl.G, "d": wl.d, "n_c": wl.n_c,
            "chunk": wl.m, "prompt_rows": wl.P, "chunks": wl.n_chunks, "r": r,
            "inputs": "synthetic, seeded; " + _recipe(wl),
            "chunk_inputs": "resident in HBM" if resident else "drawn on the device per chunk",
            "l2": "inputs larger than L2 (K_ctx alone is %.1f GB per step)"
                  % (wl.units * wl.n_c * wl.d * 2 / 1e9)}


def _recipe(wl):
    parts = ["Q,K,V ~ N(0,1) bf16" if wl.dtype == "bf16" else "Q,K ~ N(0,1) fp32"]
    if wl.hi_frac:
        parts.append(f"{wl.hi_frac:.0%} of key rows x{wl.hi_scale:g}")
    if wl.sinks:
        parts.append(f"first {wl.sinks} keys x{wl.sink_scale:g}")
    if wl.lognormal_sigma:
        parts.append(f"key rows x lognormal(0,{wl.lognormal_sigma:g})")
    return ", ".join(parts)


# ----------------------------------------------------------------- oracle sample

def oracle_sample(wl, k_ctx_u, k_bits, q_g, ks_u, scores_layer, r):
    """Time the CPU oracle on a bounded sample and extrapolate to one step.

    Scoring sample: one (layer, head) unit, one chunk, one query head (n_in rows
    against all n_c context keys + causal self keys); a step has units x chunks
    x G such pieces.  Selection + compaction sample: one layer (H units); a step
    has L of them.  Returns (seconds per step extrapolated, sample text, threads).
    """
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    s_c, _ = oracle.unit_chunk_scores(q_g, k_ctx_u, ks_u)
    t_score = time.perf_counter() - t0
    assert np.all(s_c > 0)
    t0 = time.perf_counter()
    kk = oracle.keep_count(r, scores_layer.size)
    keep, off, _ = oracle.select(scores_layer.reshape(-1), kk, wl.H)
    kv = np.broadcast_to(k_bits[None], (wl.H,) + k_bits.shape)   # H heads of bf16 rows
    oracle.compact(kv, kv, keep, off)
    t_sel = time.perf_counter() - t0
    pieces = wl.units * wl.n_chunks * wl.G
    step_s = t_score * pieces + t_sel * wl.L
    sample = (f"scoring: 1 unit x 1 chunk x 1 of {wl.G} query heads ({q_g.shape[1]} rows x "
              f"{wl.n_c}+self keys) in {t_score:.2f} s, x{pieces} extrapolated; "
              f"select+compact: 1 layer ({wl.H} heads) in {t_sel:.2f} s, x{wl.L} extrapolated")
    return step_s, sample, threads


def sample_inputs(wl, r):
    """Host float64 / int16 inputs of the oracle sample (chunk 0, unit 0, query head 0)."""
    import numpy as np
    k_ctx = synth.context_keys(wl, units=1)[0]
    q, ks = synth.chunk_qk(wl, 0, units=1)
    q_g = q[0, :1].double().numpy()
    ks_u = ks[0].double().numpy()
    k_u = k_ctx.double().numpy()
    k_bits = k_ctx.view(torch.int16).numpy() if k_ctx.dtype == torch.bfloat16 else k_ctx.numpy()
    rng = np.random.default_rng(0)
    scores_layer = (rng.random((wl.H, wl.n_c)) ** 4).astype(np.float32)
    return k_u, k_bits, q_g, ks_u, scores_layer


def run_reference(args):
    rank, world, _ = bu.dist_env()
    if rank != 0:
        return
    wl = workload(args)
    r = args.r if args.r is not None else wl.r[0]
    import numpy as np
    k_u, k_bits, q_g, ks_u, sl = sample_inputs(wl, r)
    times, sample, threads = [], "", 1
    for i in range(args.warmup + args.steps):
        step_s, sample, threads = oracle_sample(wl, k_u, k_bits, q_g, ks_u, sl, r)
        if i >= args.warmup:
            times.append(step_s)
    step_s = float(np.mean(times))
    value = wl.n_c / step_s
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
           "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": config_dict(wl, r), "impl": "reference",
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------- our arm

def _resident_bytes(wl):
    """Device bytes of K_ctx, V and every chunk's Q and K_self."""
    kv = 2 * wl.units * wl.n_c * wl.d * 2
    per_in = sum(wl.n_in(c) for c in range(wl.n_chunks))
    return kv + wl.units * per_in * wl.d * 2 * (wl.G + 1)


def run_only(args):
    """One kernel alone: kvzip_select on L*H*n_c synthetic scores (skewed like
    attention maxima), or kvzip_compact of one layer's K/V with a random keep
    mask at ratio r.  Inputs exceed L2 (126 MB) at the 128K shape."""
    from attention_score_reduction_b200 import kvzip as kz
    dev = torch.device("cuda", 0)
    wl = workload(args)
    r = args.r if args.r is not None else wl.r[0]
    peaks = bu.load_peaks(os.path.join(ROOT, "MEASURED_PEAKS.json"))
    N = wl.units * wl.n_c
    if args.only == "select":
        s = synth.random_scores(wl.units, wl.n_c, seed=11, device=dev).reshape(-1)
        k = kz.keep_count(r, N)
        keep = torch.empty(N, dtype=torch.uint8, device=dev)
        off = torch.empty(wl.units + 1, dtype=torch.int64, device=dev)
        thr = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.zeros(kz.select_workspace_size(N, wl.units), dtype=torch.uint8, device=dev)
        fn = lambda: kz.select(s, k, wl.units, keep, off, thr, ws)  # noqa: E731
        # the scores' round-1 histogram, as the last chunk's column-max pass would
        # leave it (counted here with torch outside the timed calls)
        hist = torch.bincount((s.view(torch.int32) & 0x7FFFFFFF) >> 19,
                              minlength=kz.SCORE_HIST_BINS).to(torch.int32)
        fn_hist = lambda: kz.select(s, k, wl.units, keep, off, thr, ws, hist=hist)  # noqa: E731
        nbytes = N * 4 + N
    else:
        units = wl.H      # one layer
        k_c = torch.randn(units, wl.n_c, wl.d, device=dev).to(torch.bfloat16)
        v = torch.randn_like(k_c)
        s = synth.random_scores(units, wl.n_c, seed=12, device=dev).reshape(-1)
        kept = kz.keep_count(r, s.numel())
        keep, off, _ = kz.select(s, kept, units)
        k_out = torch.empty(kept, wl.d, dtype=torch.bfloat16, device=dev)
        v_out, pos = torch.empty_like(k_out), torch.empty(kept, dtype=torch.int32, device=dev)
        fn = lambda: kz.compact(k_c, v, keep, off, kept, k_out, v_out, pos)  # noqa: E731
        nbytes = s.numel() + kept * wl.d * 2 * 2 * 2 + kept * 4
    flush = L2Flush(dev)

    def timed(f):
        times = []
        for i in range(args.warmup + args.steps):
            flush(i)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                times.append(e0.elapsed_time(e1))
        ms = sum(times) / len(times)
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": ms, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"]}

    out = {"kernel": args.only, "workload": wl.name, "bytes": nbytes}
    out.update(timed(fn))
    if args.only == "select":   # kvzip_select_hist: the first read replaced by the histogram
        out["given_hist"] = timed(fn_hist)
    out.update({"peak_source": peaks["source"], "l2": "flushed before each launch (256 MB write, then 256 MB read)"})
    print(json.dumps(out))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.only:
        run_only(args)
        return
    rank, world, local = bu.dist_env()
    dev = torch.device("cuda", local % torch.cuda.device_count())
    torch.cuda.set_device(dev)
    group = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {"device_id": dev} if args.dist_backend == "nccl" else {}
        dist.init_process_group(args.dist_backend, timeout=datetime.timedelta(seconds=600), **kw)
        group = dist.group.WORLD
    from attention_score_reduction_b200 import kvzip as kz
    from attention_score_reduction_b200 import pipeline

    wl_ctx = workload(args)            # the whole context
    wl = shard(wl_ctx, rank, world)    # the units this rank scores and compacts
    r = args.r if args.r is not None else wl.r[0]
    free, total = torch.cuda.mem_get_info(dev)
    # Chunk inputs stay resident when they fit with room for the outputs;
    # otherwise each chunk's Q / K_self is drawn on the device just before its
    # launches, outside the timed events (the 170K Gemma3-12B shape: ~100 GB).
    resident = _resident_bytes(wl) < 0.7 * total
    k_ctx, v = synth.context_kv(wl, device=dev)
    chunks = [synth.chunk_qk(wl, c, device=dev) for c in range(wl.n_chunks)] if resident else None
    max_n_in = max(wl.n_in(c) for c in range(wl.n_chunks))
    comp = pipeline.Compressor(wl.units, wl.n_c, wl.d, wl.G, max_n_in, device=dev, group=group,
                               units_global=wl_ctx.units)
    N = wl.units * wl.n_c
    kept = comp.keep_capacity(r)        # rows of this rank's compacted cache (bound)
    k_out = torch.empty(kept, wl.d, dtype=torch.bfloat16, device=dev)
    v_out = torch.empty_like(k_out)
    pos_out = torch.empty(kept, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()

    def chunk(c):
        return chunks[c] if resident else synth.chunk_qk(wl, c, device=dev)

    stream = torch.cuda.current_stream()
    per_launch = []  # (event before, event after, kernel name, flops) per scorer launch, timed steps
    stage_ev = []

    def step(timed: bool):
        comp.reset()
        launches = 0
        for c in range(wl.n_chunks):   # per chunk: pass 1 (row normalisers), then pass 2 (column max)
            q, ks = chunk(c)
            f = bu.score_flops(wl.units, wl.G, q.shape[2], wl.n_c, wl.d)
            for which, name in (("lse", "score_pass1_lse"), ("colmax", "score_pass2_colmax")):
                if timed:
                    e0, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
                    e0.record(stream)
                last = which == "colmax" and c == wl.n_chunks - 1 and comp.score_hist is not None
                kz.score_chunk(q, k_ctx, ks, comp.scores, comp.score_ws, which=which,
                               hist=comp.score_hist if last else None)
                comp.hist_ready = comp.hist_ready or last
                launches += kz.last_launch_count()
                if timed:
                    e1.record(stream)
                    per_launch.append((e0, e1, name,
                                       f["pass1"] if which == "lse" else f["pass2"]))
            del q, ks
        if timed:
            s0, s1, s2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            s0.record(stream)
        comp.select(r)
        launches += kz.last_launch_count()
        if timed:
            s1.record(stream)
        comp.compact(k_ctx, v, kept, k_out, v_out, pos_out)
        launches += kz.last_launch_count()
        if timed:
            s2.record(stream)
            stage_ev.append((s0, s1, s2))
        return launches

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    comp.check_status()

    bu.barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    launches = 0
    with bu.ClockSampler(dev.index) as clk:
        start.record(stream)
        for _ in range(args.steps):
            launches += step(True)
        end.record(stream)
        torch.cuda.synchronize()
    bu.barrier(world)
    comp.check_status()
    clocks = clk.summary()
    sel = [a.elapsed_time(b) for a, b, _ in stage_ev]
    cmp = [b.elapsed_time(c) for _, b, c in stage_ev]
    if resident:
        step_ms = start.elapsed_time(end) / args.steps
        timing = "K whole steps between two events on the launching stream"
    else:
        step_ms = (sum(a.elapsed_time(b) for a, b, _, _ in per_launch) + sum(sel) + sum(cmp)) / args.steps
        timing = ("sum of per-launch events (scorer passes, selection, compaction); each chunk's "
                  "Q / K_self drawn on the device between timed launches")
    ms_per_step = bu.max_over_ranks(step_ms, world, dev)
    value = wl_ctx.n_c / (ms_per_step / 1e3)    # one context per step over all ranks

    # per-kernel device times
    peaks = bu.load_peaks(os.path.join(ROOT, "MEASURED_PEAKS.json"))
    peak_tf = peaks["bf16_tflops_sustained"]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    clock_peak_tf = (bu.clock_peak_tflops(sms, clocks.get("sm_mhz"))
                     if clocks.get("sm_mhz") else None)
    by_kernel = {}
    for a, b, name, flops in per_launch:
        by_kernel.setdefault(name, []).append((a.elapsed_time(b), flops))
    kernels = {}
    for name, rows in by_kernel.items():
        t = sum(ms for ms, _ in rows) / len(rows)
        f = sum(fl for _, fl in rows) / len(rows)
        tf = f / (t * 1e-3) / 1e12
        kernels[name] = {"launches_per_step": len(rows) // args.steps, "ms": t,
                         "tflop_per_launch": f / 1e12, "tflops": tf, "frac_of_peak": tf / peak_tf,
                         "frac_of_burst_peak": tf / peaks["bf16_tflops"],
                         "frac_of_clock_peak": (tf / clock_peak_tf) if clock_peak_tf else None}
    dominant = max(by_kernel, key=lambda n: sum(ms for ms, _ in by_kernel[n]))
    # selection / compaction bytes: scores read once + mask written; kept K and V rows
    # read and written once, positions written, mask read once.
    kept_rows = int(comp.offsets[-1])   # this rank's kept rows (the global k on one GPU)
    sel_bytes = N * 4 + N
    cmp_bytes = N + kept_rows * wl.d * 2 * 2 * 2 + kept_rows * 4
    t_sel, t_cmp = sum(sel) / len(sel), sum(cmp) / len(cmp)
    score_ms = sum(ms for rows in by_kernel.values() for ms, _ in rows) / args.steps
    score_flops = sum(fl for rows in by_kernel.values() for _, fl in rows) / args.steps
    dk = kernels[dominant]
    roofline = {"kernel": dominant, "bound": "tensor", "achieved": dk["tflops"], "peak": peak_tf,
                "unit": "TFLOP/s", "frac": dk["frac_of_peak"],
                "traffic": NCU_TRAFFIC.get((wl.name, wl.L, dominant)),
                "peak_source": f"{peaks['source']} bf16 sustained",
                "flops_per_launch": dk["tflop_per_launch"] * 1e12,
                "frac_of_burst_peak": dk["frac_of_burst_peak"],
                "frac_of_clock_peak": dk["frac_of_clock_peak"],
                "clock_peak_tflops": clock_peak_tf,
                "clock_peak_basis": f"{sms} SMs x 8192 dense bf16 flop/clk x median SM clock"}
    kernels.update({
        "select": {"ms": t_sel, "gbs": sel_bytes / (t_sel * 1e-3) / 1e9,
                   "frac_of_hbm": sel_bytes / (t_sel * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "compact": {"ms": t_cmp, "gbs": cmp_bytes / (t_cmp * 1e-3) / 1e9,
                    "frac_of_hbm": cmp_bytes / (t_cmp * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "select_plus_compact_frac_of_hbm":
            (sel_bytes + cmp_bytes) / ((t_sel + t_cmp) * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "scoring_ms_per_step": score_ms,
        "scoring_pct_bf16_tc_peak": 100.0 * score_flops / (score_ms * 1e-3) / 1e12 / peak_tf,
        "step_pct_bf16_tc_peak": 100.0 * score_flops / (ms_per_step * 1e-3) / 1e12 / peak_tf,
    })

    # ------------------------------------------------------------ decode over the kept cache
    decode = None
    if not args.no_decode:
        decode = run_decode(wl, comp, k_ctx, v, dev, peaks)

    variants = None
    if not args.no_variants:
        variants = run_variants(wl, comp, k_ctx, chunk(0), r, dev, peaks)

    # ------------------------------------------------------------ end to end
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wl, r, comp, k_ctx, v, chunk, kept, world, dev, resident, wl_ctx)

    parallelism = ("one GPU" if world == 1 else
                   f"one context sharded over {world} GPUs: {wl.units} of its {wl_ctx.units} "
                   f"(layer, KV head) units each; scoring and compaction local, global "
                   f"selection by an all-reduce of each radix histogram and an all-gather "
                   f"of tie counts ({args.dist_backend})")
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
           "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic", "config": config_dict(wl_ctx, r, resident),
           "parallelism": parallelism, "timing": timing, "clocks": clocks,
           "gpu_launches": launches, "roofline": roofline, "kernels": kernels,
           "pct_bf16_tc_peak": kernels["step_pct_bf16_tc_peak"], "e2e": e2e,
           "decode_attention": decode, "variants": variants}

    # free device memory before the CPU baseline allocates host buffers
    del chunks, k_ctx, v, comp
    torch.cuda.empty_cache()
    if world == 1 and rank == 0 and not args.no_cpu:
        k_u, k_bits, q_g, ks_u, sl = sample_inputs(workload(args), r)
        step_s, sample, threads = oracle_sample(wl, k_u, k_bits, q_g, ks_u, sl, r)
        out["cpu_baseline"] = {"value": wl.n_c / step_s, "unit": "tokens/s", "cores": threads,
                               "kind": "oracle", "sample": sample}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


class L2Flush:
    """Clears L2 (126 MB) between timed launches: a 256 MB write, then a
    256 MB read of another buffer.  The read evicts the written lines, so
    they are back in HBM before the next launch starts; after a write alone
    the timed kernel would also pay for writing back ~126 MB of dirty lines."""

    def __init__(self, dev):
        self.w = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(64 * 2**20, dtype=torch.int32, device=dev)

    def __call__(self, i):
        self.w.fill_(i & 0xff)
        self.sink = self.r.max()


def _time_ms(fn, flush, iters=10, warm=3):
    ms = 0.0
    for i in range(iters + warm):
        flush(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        if i >= warm:
            ms += e0.elapsed_time(e1)
    return ms / iters


def run_variants(wl, comp, k_ctx, chunk, r, dev, peaks):
    """The ablation and head-level kernels on the bench workload's final scores.

    head_scores and token_scores read the L x H x n_c scores once; expand_keep
    writes the per-head mask from a position mask; select_per_head is the
    uniform-budget selection (same bytes as the global one); score_chunk_sum is
    the sum-aggregation pass 2 of one chunk (tensor cores).  L2 is flushed
    (L2Flush) before every timed launch.
    """
    from attention_score_reduction_b200 import kvzip as kz
    units, n_c = wl.units, wl.n_c
    N = units * n_c
    S = comp.scores
    flush = L2Flush(dev)
    hbm = peaks["hbm_gbs"]
    out = {}

    def bw(name, ms, nbytes):
        g = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"ms": ms, "bytes": nbytes, "gbs": g, "frac_of_hbm": g / hbm}

    hs = torch.empty(units, dtype=torch.float32, device=dev)
    bw("head_scores", _time_ms(lambda: kz.head_scores(S, hs), flush), N * 4 + units * 4)
    tok = torch.empty(n_c, dtype=torch.float32, device=dev)
    bw("token_scores", _time_ms(lambda: kz.token_scores(S, tok), flush), N * 4 + n_c * 4)
    kt = kz.keep_count(r, n_c)
    keep_pos, pos_off, _ = kz.select(tok, kt, 1)
    bw("expand_keep", _time_ms(lambda: kz.expand_keep(keep_pos, pos_off, units), flush),
       n_c + N + (units + 1) * 8)
    ws = torch.empty(max(int(kz.library().kvzip_select_per_head_workspace_size(units, n_c)), 256),
                     dtype=torch.uint8, device=dev)
    kph = kz.keep_count(r, n_c)
    bw("select_per_head", _time_ms(lambda: kz.select_per_head(S, kph, ws), flush), N * 4 + N)
    q, ks = chunk
    tmp = torch.zeros_like(S)
    sws = kz.new_score_workspace(units, wl.G, q.shape[2], dev)

    # kvzip_score_chunk_sum runs both passes; timed whole against both passes' flops
    ms = _time_ms(lambda: kz.score_chunk_sum(q, k_ctx, ks, tmp, sws), flush, iters=3, warm=1)
    f = bu.score_flops(units, wl.G, q.shape[2], n_c, wl.d)
    tf = (f["pass1"] + f["pass2"]) / (ms * 1e-3) / 1e12
    out["score_chunk_sum"] = {"ms": ms, "tflop": (f["pass1"] + f["pass2"]) / 1e12, "tflops": tf,
                              "frac_of_peak": tf / peaks["bf16_tflops_sustained"]}
    del tmp
    return out


def run_decode(wl, comp, k_ctx, v, dev, peaks, ratios=(1.0, 0.8, 0.6, 0.4, 0.2), iters=20):
    """Decode-attention latency over layer 0's cache kept at each ratio.

    The analogue of the rebuttal's decoding-efficiency table (latency and cache
    size against the kept ratio): layer 0's H heads are ranked by the scores of
    the last step, compacted at ratio r, and one decoding step of attention
    (G query heads per KV head) reads the kept rows.  L2 is flushed (L2Flush)
    before every timed launch.  ``ms`` times the call captured once in a
    CUDA graph and replayed (its two kernels, no host work inside the events);
    ``call_ms`` times the plain Python call, host argument checks, tensor-map
    encoding and launches included.
    """
    from attention_score_reduction_b200 import kvzip as kz
    H, n_c, d, G = wl.H, wl.n_c, wl.d, wl.G
    s0 = comp.scores[:H].contiguous().view(-1)
    k0, v0 = k_ctx[:H].contiguous(), v[:H].contiguous()
    g = torch.Generator(device=dev)
    g.manual_seed(synth.BASE_SEED + 5)
    q = torch.randn(H, G, d, generator=g, device=dev).to(torch.bfloat16)
    flush = L2Flush(dev)
    ws = torch.zeros(kz.decode_workspace_size(H, G, d), dtype=torch.uint8, device=dev)
    out = torch.empty(H, G, d, dtype=torch.float32, device=dev)
    rows = []
    for r in ratios:
        kept = kz.keep_count(r, s0.numel())
        keep, off, _ = kz.select(s0, kept, H)
        ko, vo, _ = kz.compact(k0, v0, keep, off, kept, want_pos=False)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            kz.decode_attention(q, ko, vo, off, out, ws)
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(graph):
            kz.decode_attention(q, ko, vo, off, out, ws)
        times = {"graph": 0.0, "call": 0.0}
        for mode in times:
            for i in range(iters + 3):
                flush(i)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                if mode == "graph":
                    graph.replay()
                else:
                    kz.decode_attention(q, ko, vo, off, out, ws)
                e1.record()
                torch.cuda.synchronize()
                if i >= 3:
                    times[mode] += e0.elapsed_time(e1) / iters
        del graph
        ms = times["graph"]
        nbytes = kept * d * 2 * 2 + q.numel() * 2 + out.numel() * 4
        rows.append((r, ms, kept * d * 2 * 2, nbytes / (ms * 1e-3) / 1e9, times["call"]))
    full = rows[0][1]
    return {"workload": f"layer 0: {H} KV heads x G={G}, d={d}, {n_c} positions, one decoding step",
            "r": [x[0] for x in rows], "ms": [x[1] for x in rows],
            "call_ms": [x[4] for x in rows],
            "kv_bytes": [x[2] for x in rows], "gbs": [x[3] for x in rows],
            "frac_of_hbm": [x[3] / peaks["hbm_gbs"] for x in rows],
            "speedup_vs_full": [full / x[1] for x in rows], "l2": "flushed before each launch (256 MB write, then 256 MB read)"}


def _pinned_like(t):
    """Page-locked host copy of a device tensor (registered in place, no size rounding)."""
    h = torch.empty(t.shape, dtype=t.dtype)
    h.copy_(t)
    err = torch.cuda.cudart().cudaHostRegister(h.data_ptr(), h.numel() * h.element_size(), 0)
    if int(err) != 0:
        raise RuntimeError(f"cudaHostRegister failed ({int(err)})")
    return h


def _unpin(ts):
    for h in ts:
        torch.cuda.cudart().cudaHostUnregister(h.data_ptr())


def run_e2e(args, wl, r, comp, k_ctx, v, chunk, kept, world, dev, resident, wl_ctx):
    """Same step from pinned host memory: uploads, scoring, selection, compaction
    and the read-back of the compacted cache all inside the timed region.

    The host holds K_ctx, V and as many distinct chunk inputs as a host-memory
    budget allows (all of them on a single-GPU run with enough RAM); when it
    holds fewer, chunks reuse host buffers cyclically, so every chunk is still
    uploaded in full each step.  When the chunk inputs are not resident on the
    device they stream through a ring of three device buffers."""
    import psutil
    from attention_score_reduction_b200 import pipeline
    steps = args.e2e_steps or max(1, args.steps)
    q0, ks0 = chunk(0)
    per_chunk = q0.numel() * q0.element_size() + ks0.numel() * ks0.element_size()
    fixed = 2 * k_ctx.numel() * k_ctx.element_size() + 2 * kept * wl.d * 2
    budget = 0.6 * psutil.virtual_memory().available / world
    if budget < fixed + per_chunk:
        return {"skipped": f"host RAM: {fixed / 1e9:.1f} GB of pinned K/V and output needed, "
                           f"{budget / 1e9:.1f} GB budget"}
    n_host = int(max(1, min(wl.n_chunks, (budget - fixed) // max(per_chunk, 1))))
    k_h, v_h = _pinned_like(k_ctx), _pinned_like(v)
    q_h, ks_h = [], []
    for c in range(n_host):
        q, ks = chunk(c)
        q_h.append(_pinned_like(q))
        ks_h.append(_pinned_like(ks))
        del q, ks
    qs = [q_h[c % n_host] for c in range(wl.n_chunks)]
    kss = [ks_h[c % n_host] for c in range(wl.n_chunks)]
    if resident:
        ring = [chunk(c) for c in range(wl.n_chunks)]
    else:   # three device slots of the largest chunk's size
        ring = [(torch.empty_like(q0), torch.empty_like(ks0)) for _ in range(3)]
    del q0, ks0
    bufs = {"k_ctx": k_ctx, "v": v, "q": [q for q, _ in ring], "ks": [ks for _, ks in ring]}
    host_out = {"k": torch.empty(kept, wl.d, dtype=torch.bfloat16),
                "v": torch.empty(kept, wl.d, dtype=torch.bfloat16),
                "pos": torch.empty(kept, dtype=torch.int32),
                "offsets": torch.empty(wl.units + 1, dtype=torch.int64)}
    for t in host_out.values():
        torch.cuda.cudart().cudaHostRegister(t.data_ptr(), t.numel() * t.element_size(), 0)
    stream = torch.cuda.current_stream()
    h2d = d2h = 0
    pipeline.compress_from_host(comp, k_h, v_h, qs, kss, r, bufs, host_out)  # warm-up
    torch.cuda.synchronize()
    bu.barrier(world)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        _, _, h2d, d2h = pipeline.compress_from_host(comp, k_h, v_h, qs, kss, r, bufs, host_out)
    end.record(stream)
    torch.cuda.synchronize()
    bu.barrier(world)
    comp.check_status()
    assert int(host_out["offsets"][-1]) <= kept
    ms = bu.max_over_ranks(start.elapsed_time(end), world, dev) / steps
    _unpin([k_h, v_h] + q_h + ks_h + list(host_out.values()))
    return {"value": wl_ctx.n_c / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "steps": steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "host_chunk_buffers": n_host, "device_chunk_buffers": len(ring)}


if __name__ == "__main__":
    main()
