"""kvzip_select_noalloc: the selection entry point for callers that cannot
allocate device memory (its scratch is a static array inside the library).

Called through the C ABI directly (ctypes), twice in a row on different score
arrays, and compared with kvzip_select (which takes a caller workspace): the
keep mask, offsets and threshold must be identical, as selection is exact.
This file is collected last so that a failure here never hides another test.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from attention_score_reduction_b200 import build
    build.build()
    from attention_score_reduction_b200 import kvzip
    L = ctypes.CDLL(kvzip.LIB_PATH)
    L.kvzip_select_noalloc.restype = ctypes.c_int
    L.kvzip_select_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p]
    return L, kvzip


def _noalloc(L, s, k, n_heads):
    N = s.numel()
    keep = torch.full((N,), 7, dtype=torch.uint8, device=s.device)
    off = torch.full((n_heads + 1,), -1, dtype=torch.int64, device=s.device)
    thr = torch.zeros(1, dtype=torch.float32, device=s.device)
    st = L.kvzip_select_noalloc(ctypes.c_void_p(s.data_ptr()), N, k, n_heads,
                                ctypes.c_void_p(keep.data_ptr()), ctypes.c_void_p(off.data_ptr()),
                                ctypes.c_void_p(thr.data_ptr()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, keep, off, thr


def test_noalloc_select_matches_workspace_select_twice(lib):
    L, kz = lib
    from attention_score_reduction_b200 import synth
    cases = [(256, 16384, 0, 0.3),    # LLaMA3.1-8B 16K score shape
             (24, 9000, 4, 0.5),      # tie-heavy, ragged segments
             (384, 174080, 0, 0.3),   # Gemma3-12B 170K score shape (48 x 8 heads)
             (40, 5000, 0, 0.0)]      # k = 0: the histogram rounds are skipped
    for n_heads, n_c, levels, r in cases:
        s = synth.random_scores(n_heads, n_c, seed=n_c, levels=levels).reshape(-1).cuda()
        k = kz.keep_count(r, s.numel())
        keep_ref, off_ref, thr_ref = kz.select(s, k, n_heads)
        st, keep, off, thr = _noalloc(L, s, k, n_heads)
        torch.cuda.synchronize()
        assert st == kz.OK
        # the multi-launch radix selection: 11 kernels, 3 when nothing is kept
        assert kz.last_launch_count() == (11 if k else 3)
        assert torch.equal(keep, keep_ref)
        assert torch.equal(off, off_ref)
        assert torch.equal(thr, thr_ref)
        assert int(off[-1]) == k
        if k == 0:
            assert not bool(keep.any()) and float(thr.item()) == float("inf")


def test_noalloc_select_signed_zero_and_inf(lib):
    """The multi-launch selection ranks -0.0 as 0.0 and +inf above every finite
    score, like the one-launch selection."""
    L, kz = lib
    import numpy as np
    g = np.random.default_rng(9)
    s = g.choice(np.array([0.0, 0.125, np.inf], np.float32), size=(8, 3000), p=[0.6, 0.3, 0.1])
    s[(s == 0) & (g.random(s.shape) < 0.5)] = np.float32(-0.0)
    sd = torch.from_numpy(s).reshape(-1).cuda()
    for r in (0.05, 0.3, 0.7):
        k = kz.keep_count(r, sd.numel())
        keep_ref, off_ref, thr_ref = kz.select(sd, k, 8)
        st, keep, off, thr = _noalloc(L, sd, k, 8)
        torch.cuda.synchronize()
        assert st == kz.OK
        assert torch.equal(keep, keep_ref) and torch.equal(off, off_ref)
        assert torch.equal(thr, thr_ref)


def test_noalloc_select_rejects_oversize(lib):
    L, kz = lib
    s = torch.zeros(4, dtype=torch.float32, device="cuda")
    # 2^30 scores in one head need more than the static scratch holds; rejected
    # on the host before any launch (the pointer is never dereferenced).
    st = L.kvzip_select_noalloc(ctypes.c_void_p(s.data_ptr()), 1 << 30, 10, 1,
                                ctypes.c_void_p(s.data_ptr()), ctypes.c_void_p(s.data_ptr()),
                                None, None)
    assert st == kz.ERR_UNSUPPORTED
