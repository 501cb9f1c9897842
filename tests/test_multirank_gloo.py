"""Host logic of multi-GPU runs, on CPU with gloo and two ranks: each rank
compresses its own context (distinct seeds), and the reported time is the
max over ranks."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_score_reduction_b200 import benchutil as bu
        from attention_score_reduction_b200 import synth
        r, w, lr = bu.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        wl = synth.WORKLOADS["tiny_fp32"]
        if r:
            wl = wl.with_(cfg_id=wl.cfg_id + bu.rank_salt(r))
        k = synth.context_keys(wl)
        digest = float(k.double().sum())
        got = bu.max_over_ranks(10.0 + rank, world)
        allk = [None] * world
        dist.all_gather_object(allk, digest)
        bu.barrier(world)
        q.put((rank, got, allk))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_contexts():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, allk in res:
        assert got == 11.0                       # max over ranks of 10 + rank
        assert allk[0] != allk[1]                # each rank has its own context


def test_clock_summary_parsing():
    from attention_score_reduction_b200 import benchutil as bu
    rows = [["0", "1965", "1965", "700.1", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"],
            ["0", "1800", "1965", "990.0", "0x4", "Not Active", "Not Active", "Not Active", "Active"],
            ["0", "1700", "1965", "1000.0", "0x4", "Not Active", "Not Active", "Not Active", "Active"]]
    s = bu.summarize_clock_rows(rows)
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_score_flops_counts_pairs():
    from attention_score_reduction_b200 import benchutil as bu
    f = bu.score_flops(B=2, G=3, n_in=5, n_c=7, d=4)
    R = 15
    assert f["pass2"] == 2 * 4 * 2 * R * 7
    assert f["pass1"] == 2 * 4 * 2 * (R * 7 + 3 * 5 * 6 // 2)


def _shard_worker(rank, world, port, q, heads, n_c, levels, ks, given=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_score_reduction_b200 import sharded, synth
        from tests import shard_fake
        s = synth.random_scores(sum(heads), n_c, seed=7 + levels, levels=levels)
        h0 = sum(heads[:rank])
        mine = s[h0:h0 + heads[rank]].contiguous()
        hist = None
        if given:   # this rank's round-1 histogram, as its last chunk's pass 2 would count it
            import numpy as np
            u = mine.reshape(-1).numpy().view(np.uint32)
            hist = torch.from_numpy(np.bincount((u & 0x7FFFFFFF) >> 19, minlength=8192))
        out = []
        for k in ks:
            keep, off, thr = sharded.select_sharded(mine, k, backend=shard_fake, round1_hist=hist)
            out.append((keep.numpy().copy(), off.numpy().copy(), float(thr.item())))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("heads,n_c,levels,given", [((3, 5), 300, 0, False), ((4, 4), 257, 8, False),
                                                    ((2, 6), 100, 2, False), ((5, 3), 64, 1, False),
                                                    ((3, 5), 300, 0, True), ((4, 4), 257, 8, True)])
def test_sharded_selection_exchange_matches_global(heads, n_c, levels, given):
    """Two gloo ranks, each holding a run of heads (uneven splits), run the
    sharded selection's exchange (histogram all-reduce per radix round, tie
    count all-gather); the concatenated masks, the per-rank offsets and the
    threshold equal the oracle's global selection, including tie-heavy arrays
    where the ties at the threshold straddle the two ranks.  With ``given``,
    each rank passes its round-1 histogram instead of running the first
    histogram pass."""
    import numpy as np

    import oracle
    from attention_score_reduction_b200 import synth
    N = sum(heads) * n_c
    ks = [0, 1, oracle.keep_count(0.3, N), oracle.keep_count(0.5, N), N - 1, N]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 30500 + (os.getpid() % 1000) + 7 * levels
    port += 3 if given else 0
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q, heads, n_c, levels, ks, given))
             for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    s = synth.random_scores(sum(heads), n_c, seed=7 + levels, levels=levels).numpy()
    for i, k in enumerate(ks):
        keep_ref, off_ref, thr_ref = oracle.select(s.reshape(-1), k, sum(heads))
        keep = np.concatenate([res[0][i][0], res[1][i][0]])
        assert np.array_equal(keep, keep_ref), (k, levels)
        off0, off1 = res[0][i][1], res[1][i][1]
        assert np.array_equal(off0, off_ref[:heads[0] + 1])
        assert np.array_equal(off1 + off0[-1], off_ref[heads[0]:])
        assert res[0][i][2] == res[1][i][2] == thr_ref
