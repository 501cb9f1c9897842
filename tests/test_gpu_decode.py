"""Decode attention over the compacted per-head cache against the oracle.

The GPU path multiplies bf16 values in fp32 and accumulates the softmax and
the weighted V rows in fp32; the oracle works in float64.  Outputs are convex
combinations of V rows (|v| ~ 1), so fp32 rounding leaves errors near 1e-6;
the bound below (1e-4 absolute + 1e-4 relative) fails on any indexing,
masking or merge mistake by orders of magnitude.
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


def _case(seed, n_heads, n_c, d, G, r, empty_head=None):
    from attention_score_reduction_b200 import synth
    g = torch.Generator().manual_seed(seed)
    K = torch.randn(n_heads, n_c, d, generator=g).to(torch.bfloat16)
    V = torch.randn(n_heads, n_c, d, generator=g).to(torch.bfloat16)
    s = synth.random_scores(n_heads, n_c, seed=seed)
    if empty_head is not None:
        s[empty_head] = 0.0           # lowest scores: this head keeps nothing
    k = oracle.keep_count(r, s.numel())
    keep, off, _ = oracle.select(s.reshape(-1).numpy(), k, n_heads)
    ko, vo, _ = oracle.compact(K.view(torch.int16).numpy(), V.view(torch.int16).numpy(), keep, off)
    ko = torch.from_numpy(ko).view(torch.bfloat16)
    vo = torch.from_numpy(vo).view(torch.bfloat16)
    q = torch.randn(n_heads, G, d, generator=g).to(torch.bfloat16)
    return q, ko, vo, off


def _check(kz, q, ko, vo, off):
    want = oracle.decode_attention(q.double().numpy(), ko.double().numpy(), vo.double().numpy(), off)
    got = kz.decode_attention(q.cuda(), ko.cuda(), vo.cuda(), torch.from_numpy(off).cuda())
    got = got.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    assert np.allclose(got, want, rtol=1e-4, atol=1e-4), np.abs(got - want).max()


@pytest.mark.parametrize("G", [1, 2, 4, 5, 8])
@pytest.mark.parametrize("d", [128, 256])
def test_decode_matches_oracle(kz, G, d):
    q, ko, vo, off = _case(G * 100 + d, n_heads=6, n_c=3000, d=d, G=G, r=0.3)
    _check(kz, q, ko, vo, off)


def test_decode_ragged_empty_and_single_row_heads(kz):
    q, ko, vo, off = _case(7, n_heads=5, n_c=701, d=128, G=4, r=0.2, empty_head=2)
    assert off[3] == off[2]                              # head 2 keeps nothing
    _check(kz, q, ko, vo, off)
    # a head with exactly one kept row returns that row's V
    off1 = np.array([0, 1], dtype=np.int64)
    _check(kz, q[:1], ko[:1], vo[:1], off1)


def test_decode_nothing_kept(kz):
    q = torch.randn(3, 4, 128).to(torch.bfloat16)
    off = torch.zeros(4, dtype=torch.int64)
    empty = torch.empty(0, 128, dtype=torch.bfloat16)
    got = kz.decode_attention(q.cuda(), empty.cuda(), empty.cuda(), off.cuda())
    assert torch.count_nonzero(got) == 0


def test_decode_long_heads(kz):
    """LLaMA3.1-8B layer shape at r = 0.3 of 16K keys: about 4900 kept rows per head."""
    q, ko, vo, off = _case(11, n_heads=8, n_c=16384, d=128, G=4, r=0.3)
    _check(kz, q, ko, vo, off)


def test_decode_head_range_outside_the_buffer_reads_nothing(kz):
    """offsets whose last head runs past the packed rows (n_rows, taken from
    the tensors' shape): that head gives zeros and reads no row, the others
    are exact.  The debug build also records the failed range check."""
    q, ko, vo, off = _case(13, n_heads=4, n_c=900, d=128, G=4, r=0.3)
    want = oracle.decode_attention(q.double().numpy(), ko.double().numpy(), vo.double().numpy(), off)
    bad = off.copy()
    bad[-1] = off[-1] + 40
    got = kz.decode_attention(q.cuda(), ko.cuda(), vo.cuda(), torch.from_numpy(bad).cuda())
    got = got.cpu().double().numpy()
    assert np.allclose(got[:3], want[:3], rtol=1e-4, atol=1e-4)
    assert not np.any(got[3])
    lib = kz.library()
    if lib.kvzip_debug_checks() == 1:
        assert lib.kvzip_debug_bounds_status() == kz.ERR_BOUNDS   # reads and clears the flag


def test_decode_buffer_with_spare_rows(kz):
    """A packed buffer longer than offsets[n_heads] (spare rows after the last
    head, as when it was sized for a larger budget): same result."""
    q, ko, vo, off = _case(17, n_heads=3, n_c=1200, d=256, G=2, r=0.4)
    pad = torch.randn(77, 256).to(torch.bfloat16)
    _check(kz, q, torch.cat([ko, pad]), torch.cat([vo, pad]), off)
