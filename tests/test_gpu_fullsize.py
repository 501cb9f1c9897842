"""Full-size parity in the launch configuration the benchmark times.

LLaMA3.1-8B KV shape, 128K context: one kvzip_score_chunk call over all 256
(layer, head) units with n_c = 131072 context keys and n_in = 16 + 2048 rows.
The oracle cannot materialise all units, so sampled units are checked in
full (every one of their 131072 scores): S for a unit is the max over query
heads g of the oracle's scores for that head's rows alone (rows of different
query heads never interact before the max).  Selection runs on the full
33.5M-score array and must be bit-exact; compaction is checked on sampled
heads against the source rows.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

RTOL = 2e-3


@pytest.fixture(scope="module")
def kz():
    from attention_score_reduction_b200 import build
    build.build()
    from attention_score_reduction_b200 import kvzip
    return kvzip


@pytest.fixture(scope="module")
def full(kz):
    from attention_score_reduction_b200 import synth
    wl = synth.WORKLOADS["llama8b_128k"]
    dev = torch.device("cuda", 0)
    k_ctx, v = synth.context_kv(wl, device=dev)
    return wl, k_ctx, v


def _oracle_unit(q_b, k_b, ks_b):
    f = lambda t: t.double().numpy()  # noqa: E731
    k64, ks64 = f(k_b), f(ks_b)
    out = None
    for g in range(q_b.shape[0]):
        s, _ = oracle.unit_chunk_scores(f(q_b[g:g + 1]), k64, ks64)
        out = s if out is None else np.maximum(out, s)
    return out


@pytest.mark.parametrize("chunk,units", [(0, (0, 255)), (63, (137,))])
def test_fullsize_scores_sampled_units(kz, full, chunk, units):
    from attention_score_reduction_b200 import synth
    wl, k_ctx, _ = full
    q, ks = synth.chunk_qk(wl, chunk, device=k_ctx.device)
    assert q.shape == (256, 4, 2064, 128)
    S = torch.zeros(wl.units, wl.n_c, device=k_ctx.device)
    ws = kz.new_score_workspace(wl.units, wl.G, q.shape[2])
    kz.score_chunk(q, k_ctx, ks, S, ws)
    assert kz.workspace_status(ws) == kz.OK
    for b in units:
        want = _oracle_unit(q[b].cpu(), k_ctx[b].cpu(), ks[b].cpu())
        got = S[b].cpu().double().numpy()
        err = float(np.max(np.abs(got - want) / want))
        assert err <= RTOL, (chunk, b, err)


def test_fullsize_select_and_compact(kz, full):
    """Global selection over 32 x 8 x 131072 scores (from the GPU's chunk-0
    scores) is bit-exact at r = 0.3 and 0.5, read twice (kvzip_select) and
    read once given the round-1 histogram that chunk 0's pass 2 counted
    (kvzip_select_hist); compacted rows of sampled heads equal their source
    rows."""
    from attention_score_reduction_b200 import synth
    wl, k_ctx, v = full
    q, ks = synth.chunk_qk(wl, 0, device=k_ctx.device)
    S = torch.zeros(wl.units, wl.n_c, device=k_ctx.device)
    hist = kz.new_score_hist(k_ctx.device)
    kz.score_chunk(q, k_ctx, ks, S, hist=hist)
    del q, ks
    s_host = S.reshape(-1).cpu().numpy()
    u = s_host.view(np.uint32)
    assert np.array_equal(hist.cpu().numpy().astype(np.int64),
                          np.bincount((u & 0x7FFFFFFF) >> 19, minlength=8192))
    for r in (0.3, 0.5):
        k = kz.keep_count(r, S.numel())
        keep_ref, off_ref, thr_ref = oracle.select(s_host, k, wl.units)
        keep_h, off_h_given, thr_h = kz.select(S.reshape(-1), k, wl.units, hist=hist)
        assert np.array_equal(off_h_given.cpu().numpy(), off_ref)
        assert np.array_equal(keep_h.cpu().numpy(), keep_ref)
        assert float(thr_h.item()) == thr_ref
        del keep_h
        keep, off, thr = kz.select(S.reshape(-1), k, wl.units)
        assert np.array_equal(off.cpu().numpy(), off_ref)
        assert np.array_equal(keep.cpu().numpy(), keep_ref)
        assert float(thr.item()) == thr_ref
        ko, vo, pos = kz.compact(k_ctx, v, keep, off, k)
        off_h = off_ref
        for h in (0, 77, 255):
            a, b = int(off_h[h]), int(off_h[h + 1])
            js = np.nonzero(keep_ref.reshape(wl.units, wl.n_c)[h])[0]
            assert np.array_equal(pos[a:b].cpu().numpy(), js)
            idx = torch.from_numpy(js).to(k_ctx.device)
            assert torch.equal(ko[a:b], k_ctx[h].index_select(0, idx))
            assert torch.equal(vo[a:b], v[h].index_select(0, idx))
        assert ko.shape[0] == k


def test_fullsize_row_normalisers_every_row_tile(kz, full):
    """Pass 1 at full size, every one of the 8256 query rows of sampled units:
    the row normalisers (log-sum-exp over 131072 context keys and the row's
    causal self keys) against the oracle's, for units in the middle of the
    launch grid.  This covers every 256-row CTA tile of the unit, including the
    ones in the middle of the row grid and the ragged last tile (rows 8192 to
    8255).  A normaliser error of e shifts every probability of its row by a
    factor exp(e), so the bound is the score tolerance itself."""
    from attention_score_reduction_b200 import synth
    wl, k_ctx, _ = full
    q, ks = synth.chunk_qk(wl, 31, device=k_ctx.device)
    S = torch.zeros(wl.units, wl.n_c, device=k_ctx.device)
    ws = kz.new_score_workspace(wl.units, wl.G, q.shape[2])
    kz.score_chunk(q, k_ctx, ks, S, ws, which="lse")
    assert kz.workspace_status(ws) == kz.OK
    lse = kz.read_lse(ws, wl.units, wl.G, q.shape[2]).cpu().double().numpy()
    f = lambda t: t.double().numpy()  # noqa: E731
    for b in (37, 200):
        k64, ks64 = f(k_ctx[b].cpu()), f(ks[b].cpu())
        want = np.concatenate([oracle.unit_chunk_scores(f(q[b, g:g + 1].cpu()), k64, ks64)[1]
                               for g in range(wl.G)])
        assert want.shape == (8256,)
        err = np.abs(lse[b] - want)
        assert float(err.max()) <= RTOL, (b, float(err.max()), int(err.argmax()))
