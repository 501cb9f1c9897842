"""The scoring kernels' bounded waits.

With the test hook on, the loader warp of every CTA issues no copies, so the
MMA warp's first wait (on the operand tiles) never completes: after the wait
limit (10 ms here) the CTA records KVZIP_ERR_TIMEOUT in the workspace, raises
its abort flag so the other warps stop waiting, frees TMEM and returns.  The
host reads the status; the CUDA context stays usable, and with the hook off
and the default limit restored the same call succeeds and matches the oracle.
Nothing here faults or hangs a GPU: every wait in the kernels is bounded by
the device timer.
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


def test_timeout_reported_and_context_survives(kz):
    g = torch.Generator().manual_seed(5)
    B, G, n_in, n_c, d = 4, 4, 300, 4096, 128
    q = torch.randn(B, G, n_in, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, n_c, d, generator=g).to(torch.bfloat16)
    ks = torch.randn(B, n_in, d, generator=g).to(torch.bfloat16)
    qd, kd, ksd = q.cuda(), k.cuda(), ks.cuda()
    ws = kz.new_score_workspace(B, G, n_in)
    S = torch.zeros(B, n_c, device="cuda")
    kz.set_wait_timeout_ns(10_000_000)
    kz.set_test_stall(True)
    try:
        kz.score_chunk(qd, kd, ksd, S, ws)
        status = kz.workspace_status(ws)
    finally:
        kz.set_test_stall(False)
        kz.set_wait_timeout_ns(0)
    assert status == kz.ERR_TIMEOUT
    assert torch.count_nonzero(S) == 0                # aborted CTAs write no scores
    assert kz.workspace_status(ws) == kz.OK          # reading clears the status
    kz.score_chunk(qd, kd, ksd, S, ws)
    assert kz.workspace_status(ws) == kz.OK
    want = np.zeros((B, n_c))
    oracle.score_chunk(q.double().numpy(), k.double().numpy(), ks.double().numpy(), want)
    got = S.cpu().double().numpy()
    assert float(np.max(np.abs(got - want) / want)) <= 2e-3


def test_selection_grid_barrier_timeout_reported_and_next_call_exact(kz):
    """The selection kernel's blocks meet at grid barriers whose waits are
    bounded.  With the test hook on, its first block returns before the first
    barrier, so every other block's wait runs out (10 ms here): the status word
    of the selection workspace reports KVZIP_ERR_TIMEOUT and the kernel ends.
    With the hook off the same call on the same workspace is bit-exact."""
    from attention_score_reduction_b200 import synth
    n_heads, n_c = 64, 8192                      # 524288 scores: well over one block
    s = synth.random_scores(n_heads, n_c, seed=3).reshape(-1).cuda()
    k = kz.keep_count(0.3, s.numel())
    ws = torch.zeros(kz.select_workspace_size(s.numel(), n_heads), dtype=torch.uint8,
                     device="cuda")
    kz.set_wait_timeout_ns(10_000_000)
    kz.set_test_stall(True)
    try:
        kz.select(s, k, n_heads, workspace=ws)
        status = kz.workspace_status(ws)
    finally:
        kz.set_test_stall(False)
        kz.set_wait_timeout_ns(0)
    assert status == kz.ERR_TIMEOUT
    assert kz.workspace_status(ws) == kz.OK      # reading clears the status
    keep, off, thr = kz.select(s, k, n_heads, workspace=ws)
    assert kz.workspace_status(ws) == kz.OK
    keep_ref, off_ref, thr_ref = oracle.select(s.cpu().numpy(), k, n_heads)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert float(thr.item()) == thr_ref
