"""Selection and aggregation variants the pages report as ablations, against
the oracle: sum aggregation (scores within 2e-3), token-level scores,
position-mask expansion and uniform per-head budgets (bit-exact)."""
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


def f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


@pytest.mark.parametrize("shape", [(2, 4, 100, 300, 128), (1, 5, 200, 777, 128), (2, 2, 150, 500, 256)])
def test_sum_aggregation(kz, shape):
    from tests.test_gpu_parity import make_inputs
    B, G, n_in, n_c, d = shape
    q, k, ks = make_inputs(sum(shape) + 1, B, G, n_in, n_c, d)
    S0 = torch.rand(B, n_c, generator=torch.Generator().manual_seed(3))
    want = f64(S0).copy()
    oracle.score_chunk_sum(f64(q), f64(k), f64(ks), want)
    S = S0.cuda()
    kz.score_chunk_sum(q.cuda(), k.cuda(), ks.cuda(), S)
    got = S.cpu().double().numpy()
    assert float(np.max(np.abs(got - want) / want)) <= 2e-3


@pytest.mark.parametrize("n_heads,n_c", [(256, 4096), (3, 1001), (1, 5)])
def test_token_scores(kz, n_heads, n_c):
    from attention_score_reduction_b200 import synth
    s = synth.random_scores(n_heads, n_c, seed=n_c)
    got = kz.token_scores(s.cuda()).cpu().numpy()
    assert np.array_equal(got, oracle.token_scores(s.numpy()).astype(np.float32))


def test_token_level_pipeline(kz):
    """Token-level eviction end to end: max over heads, select positions, one
    mask for every head, compaction -- bit-exact against the oracle chain."""
    from attention_score_reduction_b200 import synth
    n_heads, n_c, d = 6, 2000, 128
    s = synth.random_scores(n_heads, n_c, seed=17, levels=16)
    g = torch.Generator().manual_seed(5)
    K = torch.randn(n_heads, n_c, d, generator=g).to(torch.bfloat16)
    V = torch.randn(n_heads, n_c, d, generator=g).to(torch.bfloat16)
    tok_ref = oracle.token_scores(s.numpy())
    kpos = oracle.keep_count(0.3, n_c)
    keep_pos_ref, off_pos_ref, _ = oracle.select(tok_ref.astype(np.float32), kpos, 1)
    keep_ref, off_ref = oracle.expand_keep(keep_pos_ref, n_heads)
    tok = kz.token_scores(s.cuda())
    keep_pos, off_pos, _ = kz.select(tok, kpos, 1)
    assert np.array_equal(keep_pos.cpu().numpy(), keep_pos_ref)
    keep, off = kz.expand_keep(keep_pos, off_pos, n_heads)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    ko, vo, pos = kz.compact(K.cuda(), V.cuda(), keep, off, int(off_ref[-1]))
    ko_ref, vo_ref, pos_ref = oracle.compact(K.view(torch.int16).numpy(), V.view(torch.int16).numpy(),
                                             keep_ref, off_ref)
    assert np.array_equal(ko.cpu().view(torch.int16).numpy(), ko_ref)
    assert np.array_equal(pos.cpu().numpy(), pos_ref)


@pytest.mark.parametrize("n_heads,n_c,levels,r", [(8, 5000, 0, 0.3), (8, 5000, 6, 0.3),
                                                  (5, 1001, 2, 0.5), (3, 777, 0, 0.0),
                                                  (3, 777, 0, 1.0), (256, 16384, 0, 0.3)])
def test_select_per_head(kz, n_heads, n_c, levels, r):
    from attention_score_reduction_b200 import synth
    s = synth.random_scores(n_heads, n_c, seed=n_c + levels, levels=levels)
    k_h = oracle.keep_count(r, n_c)
    keep_ref, off_ref = oracle.select_per_head(s.reshape(-1).numpy(), k_h, n_heads)
    keep, off = kz.select_per_head(s.cuda(), k_h)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)


@pytest.mark.parametrize("n_heads,n_c", [(256, 16384), (7, 1001), (3, 4), (1, 5)])
def test_head_scores(kz, n_heads, n_c):
    """Head-level scores max_j S[h][j] (rebuttal, head-level scores): bit-exact,
    from aligned rows (16-byte loads) and from a view that starts 4 bytes in."""
    from attention_score_reduction_b200 import synth
    s = synth.random_scores(n_heads, n_c, seed=n_c + 3)
    want = oracle.head_scores(s.numpy(), 1, n_heads).reshape(-1).astype(np.float32)
    got = kz.head_scores(s.cuda()).cpu().numpy()
    assert np.array_equal(got, want)
    flat = torch.zeros(n_heads * n_c + 1, device="cuda")
    flat[1:] = s.reshape(-1).cuda()
    got2 = kz.head_scores(flat[1:].view(n_heads, n_c)).cpu().numpy()
    assert np.array_equal(got2, want)


def test_token_scores_and_select_from_unaligned_views(kz):
    """The 16-byte paths are taken only for aligned rows: token scores from a view
    that starts 4 bytes into its buffer, and a selection mask written at an odd
    address, go through the scalar kernels and give the same bits."""
    from attention_score_reduction_b200 import synth
    n_heads, n_c = 12, 4096
    s = synth.random_scores(n_heads, n_c, seed=23, levels=5)
    flat = torch.zeros(n_heads * n_c + 1, device="cuda")
    flat[1:] = s.reshape(-1).cuda()
    view = flat[1:].view(n_heads, n_c)
    assert np.array_equal(kz.token_scores(view).cpu().numpy(),
                          oracle.token_scores(s.numpy()).astype(np.float32))
    k = kz.keep_count(0.3, s.numel())
    keep_ref, off_ref, _ = oracle.select(s.reshape(-1).numpy(), k, n_heads)
    buf = torch.zeros(n_heads * n_c + 4, dtype=torch.uint8, device="cuda")
    keep_view = buf[1:1 + n_heads * n_c]            # mask bytes off 4-byte alignment
    kz.select(s.reshape(-1).cuda(), k, n_heads, keep=keep_view)   # scores must be aligned
    assert np.array_equal(keep_view.cpu().numpy(), keep_ref)
