"""Selection given the scores' round-1 histogram.

The column-max half of a context's last chunk can count every score it leaves
in S in the selection's first radix round (kvzip_score_colmax_hist: bins of
the top 13 bits of |s|), and the selection then skips its own first read of
the scores (kvzip_select_hist).  Checked here:

- the histogram equals a plain count of the final scores' bins, for the
  tensor-core scorer (d = 128 and 256) and the fp32 scorer;
- the selection given it equals the oracle's bit for bit, ties, -0.0 and +inf
  included, in one launch;
- a histogram that does not describe the scores (another array's, one score
  moved out of the threshold's bin, fewer than k scores) keeps nothing, writes
  zero offsets and a +inf threshold, and leaves KVZIP_ERR_INVALID_ARG in the
  status word; the next call on the same workspace is exact again.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kz():
    from attention_score_reduction_b200 import build
    build.build()
    from attention_score_reduction_b200 import kvzip
    return kvzip


def bins(s):
    """Round-1 bin counts of |s|: the top 13 bits of the float's magnitude."""
    u = np.ascontiguousarray(np.asarray(s, dtype=np.float32).reshape(-1)).view(np.uint32)
    return np.bincount((u & 0x7FFFFFFF) >> 19, minlength=8192).astype(np.int64)


def inputs(seed, B, G, n_in, n_c, d, dtype):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, G, n_in, d, generator=g).to(dtype)
    k = torch.randn(B, n_c, d, generator=g)
    k[:, :: 37] *= 3.0
    return q, k.to(dtype), torch.randn(B, n_in, d, generator=g).to(dtype)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 256),
                                     (torch.float32, 128)], ids=["bf16_d128", "bf16_d256", "f32"])
def test_last_chunk_histogram_counts_the_final_scores(kz, dtype, d):
    B, G, n_in, n_c = 3, 4, 150, 1000
    q0, k, ks0 = inputs(1, B, G, n_in, n_c, d, dtype)
    q1, _, ks1 = inputs(2, B, G, n_in, n_c, d, dtype)
    k = k.cuda()
    S = torch.zeros(B, n_c, device="cuda")
    ws = kz.new_score_workspace(B, G, n_in)
    kz.score_chunk(q0.cuda(), k, ks0.cuda(), S, ws)
    hist = kz.new_score_hist()
    kz.score_chunk(q1.cuda(), k, ks1.cuda(), S, ws, hist=hist)      # both halves
    assert kz.workspace_status(ws) == kz.OK
    assert np.array_equal(hist.cpu().numpy().astype(np.int64), bins(S.cpu().numpy()))
    # the column-max half alone on scores that are already final counts them all again
    hist2 = kz.new_score_hist()
    kz.score_chunk(q1.cuda(), k, ks1.cuda(), S, ws, which="colmax", hist=hist2)
    assert torch.equal(hist2, hist)


def _scores(kind, n_heads, n_c, seed):
    from attention_score_reduction_b200 import synth
    if kind == "uniform":
        return synth.random_scores(n_heads, n_c, seed=seed).numpy()
    if kind == "levels":
        return synth.random_scores(n_heads, n_c, seed=seed, levels=8).numpy()
    g = np.random.default_rng(seed)
    if kind == "signed_zero":
        s = g.choice(np.array([0.0, 0.125, 0.5], np.float32), size=(n_heads, n_c),
                     p=[0.6, 0.25, 0.15])
        s[(s == 0) & (g.random(s.shape) < 0.5)] = np.float32(-0.0)
        return s
    s = g.random((n_heads, n_c), dtype=np.float32)   # "inf": 5% +inf
    s[g.random(s.shape) < 0.05] = np.inf
    return s


@pytest.mark.parametrize("kind,n_heads,n_c,r", [
    ("uniform", 8, 1000, 0.3), ("uniform", 256, 4096, 0.3), ("levels", 8, 1000, 0.3),
    ("levels", 3, 20000, 0.5), ("signed_zero", 12, 5000, 0.5), ("inf", 12, 5000, 0.03),
    ("inf", 12, 5000, 0.3), ("uniform", 5, 777, 1.0), ("uniform", 5, 777, 0.0)])
def test_select_given_histogram_matches_oracle(kz, kind, n_heads, n_c, r):
    s = _scores(kind, n_heads, n_c, seed=n_c + n_heads)
    N = s.size
    k = kz.keep_count(r, N)
    sd = torch.from_numpy(s).reshape(-1).cuda()
    hist = torch.from_numpy(bins(s).astype(np.int32)).cuda()
    ws = torch.zeros(kz.select_workspace_size(N, n_heads), dtype=torch.uint8, device="cuda")
    keep, off, thr = kz.select(sd, k, n_heads, workspace=ws, hist=hist)
    assert kz.last_launch_count() == 1
    keep_ref, off_ref, thr_ref = oracle.select(s.reshape(-1), k, n_heads)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert float(thr.item()) == thr_ref
    assert kz.workspace_status(ws) == kz.OK


def _true_bin(h, k):
    """The round-1 bin that holds the k-th largest score (scanning from the top)."""
    c = np.cumsum(h[::-1])
    return len(h) - 1 - int(np.searchsorted(c, k))


def test_select_given_a_wrong_histogram_keeps_nothing(kz):
    n_heads, n_c, r = 16, 3000, 0.3
    s = _scores("uniform", n_heads, n_c, seed=4)
    N = s.size
    k = kz.keep_count(r, N)
    sd = torch.from_numpy(s).reshape(-1).cuda()
    h = bins(s)
    b1 = _true_bin(h, k)
    moved = h.copy()                  # one score of the threshold's bin moved below it
    moved[b1] -= 1
    moved[b1 - 1] += 1
    wrong = {"other_scores": bins(_scores("uniform", n_heads, n_c, seed=5) * 0.5),
             "one_score_moved": moved,
             "fewer_than_k": np.zeros_like(h)}
    ws = torch.zeros(kz.select_workspace_size(N, n_heads), dtype=torch.uint8, device="cuda")
    for name, hw in wrong.items():
        hist = torch.from_numpy(hw.astype(np.int32)).cuda()
        keep, off, thr = kz.select(sd, k, n_heads, workspace=ws, hist=hist)
        assert not bool(keep.any()), name
        assert off.tolist() == [0] * (n_heads + 1), name
        assert float(thr.item()) == float("inf"), name
        assert kz.workspace_status(ws) == kz.ERR_INVALID_ARG, name
    # the same workspace, the true histogram: exact again
    keep, off, thr = kz.select(sd, k, n_heads, workspace=ws,
                               hist=torch.from_numpy(h.astype(np.int32)).cuda())
    keep_ref, off_ref, _ = oracle.select(s.reshape(-1), k, n_heads)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert kz.workspace_status(ws) == kz.OK
