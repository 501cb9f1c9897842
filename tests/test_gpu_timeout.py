"""The scoring kernels' bounded waits: with a 1 ns limit every CTA gives up on
its first pipeline wait, drains its in-flight copies and MMAs, frees TMEM and
returns; the host reads KVZIP_ERR_TIMEOUT from the workspace.  The CUDA
context stays usable: with the default limit restored the same call succeeds
and matches the oracle.  Nothing here faults or hangs a GPU: every wait in
the kernels is bounded by the device timer."""
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
    kz.set_wait_timeout_ns(1)
    try:
        kz.score_chunk(qd, kd, ksd, S, ws)
        status = kz.workspace_status(ws)
    finally:
        kz.set_wait_timeout_ns(0)
    assert status == kz.ERR_TIMEOUT
    assert kz.workspace_status(ws) == kz.OK          # reading clears it
    S.zero_()
    kz.score_chunk(qd, kd, ksd, S, ws)
    assert kz.workspace_status(ws) == kz.OK
    want = np.zeros((B, n_c))
    oracle.score_chunk(q.double().numpy(), k.double().numpy(), ks.double().numpy(), want)
    got = S.cpu().double().numpy()
    assert float(np.max(np.abs(got - want) / want)) <= 2e-3
