"""Multi-chunk scoring through the C ABI (kvzip_score_context) against the
oracle's score_context.

Every chunk of a context is scored into one running maximum (blog post
section 4.5).  The one call must match the oracle to the same 2e-3 relative
bound as the per-chunk calls and give the same bits as calling
kvzip_score_chunk chunk by chunk, for ragged contexts, ragged last chunks,
rows of a tile spanning several query heads, many units, d = 256 and fp32.
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


def f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


def make_context(seed, B, G, n_c, d, n_ins, hi_frac=0.02, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, n_c, d, generator=g)
    k = k * torch.where(torch.rand(B, n_c, 1, generator=g) < hi_frac, 3.0, 1.0)
    k[:, : min(4, n_c)] *= 5.0  # sinks
    chunks = []
    for n_in in n_ins:
        q = torch.randn(B, G, n_in, d, generator=g)
        ks = torch.randn(B, n_in, d, generator=g)
        ks = ks * torch.where(torch.rand(B, n_in, 1, generator=g) < hi_frac, 3.0, 1.0)
        chunks.append((q.to(dtype), ks.to(dtype)))
    return k.to(dtype), chunks


def oracle_context(k, chunks):
    return oracle.score_context([f64(q) for q, _ in chunks], [f64(ks) for _, ks in chunks], f64(k))


CONTEXT_SHAPES = [  # (B, G, n_c, d, n_in per chunk)
    (2, 4, 300, 128, (100, 100, 37)),          # ragged tails, ragged last chunk
    (3, 2, 1000, 128, (17, 17)),               # a row tile spans several query heads
    (2, 5, 777, 128, (200, 200, 120)),         # G = 5 (Qwen2.5-14B grouping)
    (1, 4, 2048, 128, (528, 528, 528, 528)),   # tile multiples, four chunks
    (1, 1, 1, 128, (1, 1)),                    # one key, one row per chunk
    (64, 4, 1536, 128, (272, 272)),            # more CTAs than SMs in both passes
    (300, 1, 64, 128, (8, 8, 8)),              # many short items
    (2, 2, 500, 256, (150, 150)),              # head dim 256
    (1, 4, 2048, 128, (16,)),                  # one chunk
]


@pytest.mark.parametrize("shape", CONTEXT_SHAPES,
                         ids=lambda s: "B%d_G%d_nc%d_d%d_" % s[:4] + "-".join(map(str, s[4])))
def test_score_context_matches_oracle(kz, shape):
    B, G, n_c, d, n_ins = shape
    k, chunks = make_context(B * 7 + n_c + d + len(n_ins), B, G, n_c, d, n_ins)
    want = oracle_context(k, chunks)
    kd = k.cuda()
    dch = [(q.cuda(), ks.cuda()) for q, ks in chunks]
    S = torch.zeros(B, n_c, device="cuda")
    ws = kz.new_context_workspace(B, G, max(n_ins))
    kz.score_context(dch, kd, S, ws)
    assert kz.workspace_status(ws) == kz.OK
    assert kz.last_launch_count() == 2 * len(n_ins)   # two passes per chunk
    got = S.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    err = float(np.max(np.abs(got - want) / want))
    assert err <= RTOL, err


def test_context_call_equals_chunk_calls(kz):
    """One kvzip_score_context call gives the same bits as kvzip_score_chunk
    per chunk in order (bf16 and the fp32 CUDA-core path)."""
    for dtype in (torch.bfloat16, torch.float32):
        B, G, n_c, d, n_ins = 5, 4, 3000, 128, (300, 300, 131)
        k, chunks = make_context(11, B, G, n_c, d, n_ins, dtype=dtype)
        kd = k.cuda()
        dch = [(q.cuda(), ks.cuda()) for q, ks in chunks]
        S_ctx = torch.zeros(B, n_c, device="cuda")
        kz.score_context(dch, kd, S_ctx)
        S_chunk = torch.zeros(B, n_c, device="cuda")
        for q, ks in dch:
            kz.score_chunk(q, kd, ks, S_chunk)
        assert torch.equal(S_ctx, S_chunk), dtype


def test_context_running_max_over_existing_scores(kz):
    """The call merges into scores that already hold values (a checkpointed run)."""
    B, G, n_c, d, n_ins = 2, 4, 700, 128, (64, 64)
    k, chunks = make_context(12, B, G, n_c, d, n_ins)
    g = torch.Generator().manual_seed(13)
    S0 = torch.rand(B, n_c, generator=g, dtype=torch.float64) * 0.02
    want = np.maximum(f64(S0), oracle_context(k, chunks))
    S = S0.float().cuda()
    kz.score_context([(q.cuda(), ks.cuda()) for q, ks in chunks], k.cuda(), S)
    got = S.cpu().double().numpy()
    assert float(np.max(np.abs(got - want) / want)) <= RTOL


def test_context_timeout_reported_and_context_survives(kz):
    """With the loaders held back, every CTA of every chunk gives up after
    10 ms, the call reports KVZIP_ERR_TIMEOUT through the status word and no
    score is written; afterwards the same call succeeds."""
    B, G, n_c, d, n_ins = 4, 4, 4096, 128, (300, 300)
    k, chunks = make_context(14, B, G, n_c, d, n_ins)
    kd = k.cuda()
    dch = [(q.cuda(), ks.cuda()) for q, ks in chunks]
    ws = kz.new_context_workspace(B, G, max(n_ins))
    S = torch.zeros(B, n_c, device="cuda")
    kz.set_wait_timeout_ns(10_000_000)
    kz.set_test_stall(True)
    try:
        kz.score_context(dch, kd, S, ws)
        status = kz.workspace_status(ws)
    finally:
        kz.set_test_stall(False)
        kz.set_wait_timeout_ns(0)
    assert status == kz.ERR_TIMEOUT
    assert torch.count_nonzero(S) == 0
    assert kz.workspace_status(ws) == kz.OK
    kz.score_context(dch, kd, S, ws)
    assert kz.workspace_status(ws) == kz.OK
    want = oracle_context(k, chunks)
    got = S.cpu().double().numpy()
    assert float(np.max(np.abs(got - want) / want)) <= RTOL


def test_context_rejects_bad_arguments(kz):
    B, G, n_c, d = 1, 2, 128, 128
    k, chunks = make_context(15, B, G, n_c, d, (32, 400))
    kd = k.cuda()
    dch = [(q.cuda(), ks.cuda()) for q, ks in chunks]
    S = torch.zeros(B, n_c, device="cuda")
    small = kz.new_context_workspace(B, G, 32)   # too small for the 400-row chunk
    assert kz.context_workspace_size(B, G, 400) > small.numel()
    with pytest.raises(kz.KvzipError):
        kz.score_context(dch, kd, S, small)
