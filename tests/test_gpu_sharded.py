"""Sharded global selection (kvzip_select_shard_*) on the GPU.

A context's heads are split into contiguous runs, one per rank.  The ranks'
histograms are summed and their tie counts gathered between the kernel calls;
the concatenated masks, per-rank offsets and the threshold must equal the
oracle's selection over the whole array, bit for bit.

The first test plays two or three ranks inside one process (each with its own
workspace; the sums are done here).  The second runs two real processes on
cuda:0 that exchange through a gloo process group with
``attention_score_reduction_b200.sharded``.  No kernel waits on another
rank: every exchange happens on the host between launches.
"""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kz():
    from attention_score_reduction_b200 import build
    build.build()
    from attention_score_reduction_b200 import kvzip
    return kvzip


def _run_ranks(kz, parts, k, given=None):
    """The shard protocol for several ranks in one process.  ``given``: per
    rank, its round-1 histogram, used instead of its first histogram pass."""
    dev = parts[0].device
    wss = [kz.shard_workspace(p.numel(), p.shape[0], dev) for p in parts]
    thr = [torch.full((1,), -1.0, device=dev) for _ in parts]
    for ws in wss:
        kz.shard_begin(k, ws)
    for r in range(3):
        hists = []
        for i, (p, ws) in enumerate(zip(parts, wss)):
            if r == 0 and given is not None:
                hists.append(given[i].to(torch.int64, copy=True))
                continue
            h = torch.full((kz.shard_bins(r),), -5, dtype=torch.int64, device=dev)
            kz.shard_hist(p.reshape(-1), r, h, ws)
            hists.append(h)
        tot = torch.stack(hists).sum(0)
        for ws, t in zip(wss, thr):
            kz.shard_pick(tot, r, t, ws)
    ties = []
    for p, ws in zip(parts, wss):
        n = torch.full((1,), -5, dtype=torch.int64, device=dev)
        kz.shard_ties(p.reshape(-1), n, ws)
        ties.append(n)
    tie_counts = torch.cat(ties)
    out = []
    for rank, (p, ws) in enumerate(zip(parts, wss)):
        keep = torch.full((p.numel(),), 9, dtype=torch.uint8, device=dev)
        off = torch.full((p.shape[0] + 1,), -1, dtype=torch.int64, device=dev)
        kz.shard_mask(p.reshape(-1), p.shape[0], tie_counts, rank, keep, off, ws)
        out.append((keep, off))
    torch.cuda.synchronize()
    return out, [float(t.item()) for t in thr]


CASES = [  # (heads per rank, n_c, levels)
    ((128, 128), 16384, 0),     # LLaMA3.1-8B 16K score shape split over two GPUs
    ((3, 5), 3000, 8),          # uneven split, tie-heavy
    ((2, 6), 1001, 2),          # ragged n_c, two values: ties straddle the ranks
    ((4, 4, 4), 640, 1),        # three ranks, every score equal
    ((5, 3), 97, 0),
]


@pytest.mark.parametrize("heads,n_c,levels", CASES)
def test_shard_protocol_matches_global_selection(kz, heads, n_c, levels):
    from attention_score_reduction_b200 import synth
    s = synth.random_scores(sum(heads), n_c, seed=n_c + levels, levels=levels)
    N = s.numel()
    sd = s.cuda()
    parts, h0 = [], 0
    for h in heads:
        parts.append(sd[h0:h0 + h].contiguous())
        h0 += h
    for k in (0, 1, oracle.keep_count(0.3, N), oracle.keep_count(0.5, N), N):
        out, thr = _run_ranks(kz, parts, k)
        keep_ref, off_ref, thr_ref = oracle.select(s.reshape(-1).numpy(), k, sum(heads))
        keep = np.concatenate([o[0].cpu().numpy() for o in out])
        assert np.array_equal(keep, keep_ref), (heads, levels, k)
        base, h0 = 0, 0
        for (kp, off), h in zip(out, heads):
            off = off.cpu().numpy()
            assert np.array_equal(off + base, off_ref[h0:h0 + h + 1])
            base += int(off[-1])
            h0 += h
        if k:
            assert all(t == thr_ref for t in thr)


def test_shard_protocol_with_round1_histograms_from_the_scorer(kz):
    """Each rank's round-1 histogram counted by its last chunk's pass 2
    (kvzip_score_colmax_hist) replaces its first histogram pass; the result is
    still the global selection."""
    g = torch.Generator().manual_seed(21)
    B, G, n_in, n_c, d = 6, 4, 80, 900, 128
    q = torch.randn(B, G, n_in, d, generator=g).to(torch.bfloat16).cuda()
    k_ctx = torch.randn(B, n_c, d, generator=g).to(torch.bfloat16).cuda()
    ks = torch.randn(B, n_in, d, generator=g).to(torch.bfloat16).cuda()
    parts, given = [], []
    for h0, h1 in ((0, 2), (2, 6)):   # two ranks, uneven
        S = torch.zeros(h1 - h0, n_c, device="cuda")
        hist = kz.new_score_hist()
        kz.score_chunk(q[h0:h1].contiguous(), k_ctx[h0:h1].contiguous(), ks[h0:h1].contiguous(),
                       S, hist=hist)
        parts.append(S)
        given.append(hist)
    s_all = torch.cat([p.reshape(-1) for p in parts]).cpu().numpy()
    for r in (0.3, 0.5):
        k = oracle.keep_count(r, s_all.size)
        out, thr = _run_ranks(kz, parts, k, given)
        keep_ref, off_ref, thr_ref = oracle.select(s_all, k, B)
        assert np.array_equal(np.concatenate([o[0].cpu().numpy() for o in out]), keep_ref)
        assert all(t == thr_ref for t in thr)


def test_shard_protocol_signed_zero(kz):
    """-0.0 ranks as 0.0 on every rank, as in the one-GPU selection."""
    g = np.random.default_rng(3)
    s = g.choice(np.array([0.0, 0.25], np.float32), size=(6, 700), p=[0.7, 0.3])
    s[(s == 0) & (g.random(s.shape) < 0.5)] = np.float32(-0.0)
    sd = torch.from_numpy(s).cuda()
    parts = [sd[:2].contiguous(), sd[2:].contiguous()]
    for r in (0.2, 0.5):
        k = oracle.keep_count(r, s.size)
        out, thr = _run_ranks(kz, parts, k)
        keep_ref, off_ref, thr_ref = oracle.select(s.reshape(-1), k, 6)
        assert np.array_equal(np.concatenate([o[0].cpu().numpy() for o in out]), keep_ref)
        assert all(t == thr_ref for t in thr)


def _gloo_worker(rank, world, port, q, heads, n_c, levels, r_keep):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        from attention_score_reduction_b200 import sharded, synth
        s = synth.random_scores(sum(heads), n_c, seed=n_c + levels, levels=levels)
        h0 = sum(heads[:rank])
        mine = s[h0:h0 + heads[rank]].contiguous().cuda()
        k = oracle.keep_count(r_keep, s.numel())
        keep, off, thr = sharded.select_sharded(mine, k)
        torch.cuda.synchronize()
        q.put((rank, keep.cpu().numpy(), off.cpu().numpy(), float(thr.item())))
    finally:
        dist.destroy_process_group()


def test_two_processes_gloo_exchange_on_one_gpu(kz):
    """Two processes, each holding half of a LLaMA3.1-8B 16K context's heads
    (tie-heavy scores), select globally through gloo collectives."""
    from attention_score_reduction_b200 import synth
    heads, n_c, levels, r_keep = (128, 128), 16384, 16, 0.3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_gloo_worker, args=(r, 2, port, q, heads, n_c, levels, r_keep))
             for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        rank, keep, off, thr = q.get(timeout=300)
        res[rank] = (keep, off, thr)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    s = synth.random_scores(sum(heads), n_c, seed=n_c + levels, levels=levels).numpy()
    k = oracle.keep_count(r_keep, s.size)
    keep_ref, off_ref, thr_ref = oracle.select(s.reshape(-1), k, sum(heads))
    assert np.array_equal(np.concatenate([res[0][0], res[1][0]]), keep_ref)
    assert np.array_equal(res[0][1], off_ref[:129])
    assert np.array_equal(res[1][1] + res[0][1][-1], off_ref[128:])
    assert res[0][2] == res[1][2] == thr_ref
