"""Multi-chunk scoring through the C ABI (kvzip_score_context and
kvzip_score_pipeline_step) against the oracle's score_context.

Every chunk of a context is scored into one running maximum (blog post
section 4.5).  With bf16 and d = 128 the steps after the first run pass 1 of
chunk c and pass 2 of chunk c - 1 in one kernel; the result must match the
oracle to the same 2e-3 relative bound as the per-chunk calls, for ragged
contexts, ragged last chunks, rows of a tile spanning several query heads,
more work items than SMs, and the unfused shapes (d = 256, one chunk).
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


def make_context(seed, B, G, n_c, d, n_ins, hi_frac=0.02):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, n_c, d, generator=g)
    k = k * torch.where(torch.rand(B, n_c, 1, generator=g) < hi_frac, 3.0, 1.0)
    k[:, : min(4, n_c)] *= 5.0  # sinks
    chunks = []
    for n_in in n_ins:
        q = torch.randn(B, G, n_in, d, generator=g)
        ks = torch.randn(B, n_in, d, generator=g)
        ks = ks * torch.where(torch.rand(B, n_in, 1, generator=g) < hi_frac, 3.0, 1.0)
        chunks.append((q.to(torch.bfloat16), ks.to(torch.bfloat16)))
    return k.to(torch.bfloat16), chunks


def oracle_context(k, chunks):
    return oracle.score_context([f64(q) for q, _ in chunks], [f64(ks) for _, ks in chunks], f64(k))


CONTEXT_SHAPES = [  # (B, G, n_c, d, n_in per chunk)
    (2, 4, 300, 128, (100, 100, 37)),          # ragged tails, ragged last chunk
    (3, 2, 1000, 128, (17, 17)),               # a row tile spans several query heads
    (2, 5, 777, 128, (200, 200, 120)),         # G = 5 (Qwen2.5-14B grouping)
    (1, 4, 2048, 128, (528, 528, 528, 528)),   # tile multiples, three fused steps
    (1, 1, 1, 128, (1, 1)),                    # one key, one row per chunk
    (64, 4, 1536, 128, (272, 272)),            # several items of both passes per CTA
    (300, 1, 64, 128, (8, 8, 8)),              # many short items
    (2, 2, 500, 256, (150, 150)),              # d = 256: passes run back to back
    (1, 4, 2048, 128, (16,)),                  # one chunk: nothing to pipeline
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
    n_launch = kz.last_launch_count()
    fused = d == 128 and len(n_ins) > 1
    # fused: one launch per step (first and last step run a single pass)
    assert n_launch == (len(n_ins) + 1 if fused else 2 * len(n_ins))
    got = S.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    err = float(np.max(np.abs(got - want) / want))
    assert err <= RTOL, err


def test_pipeline_steps_equal_context_call(kz):
    """Driving the steps by hand gives the same bits as kvzip_score_context, and
    both agree with chunk-by-chunk kvzip_score_chunk to fp32 rounding."""
    B, G, n_c, d, n_ins = 5, 4, 3000, 128, (300, 300, 300)
    k, chunks = make_context(11, B, G, n_c, d, n_ins)
    kd = k.cuda()
    dch = [(q.cuda(), ks.cuda()) for q, ks in chunks]
    S_ctx = torch.zeros(B, n_c, device="cuda")
    kz.score_context(dch, kd, S_ctx)
    ws = kz.new_context_workspace(B, G, max(n_ins))
    S_step = torch.zeros(B, n_c, device="cuda")
    for step in range(len(dch) + 1):
        nxt = dch[step] if step < len(dch) else None
        prev = dch[step - 1] if step > 0 else None
        kz.score_pipeline_step(step, nxt, prev, kd, S_step, ws)
    assert kz.workspace_status(ws) == kz.OK
    assert torch.equal(S_ctx, S_step)
    S_chunk = torch.zeros(B, n_c, device="cuda")
    for q, ks in dch:
        kz.score_chunk(q, kd, ks, S_chunk)
    rel = ((S_ctx - S_chunk).abs() / S_chunk).max().item()
    assert rel <= 1e-3, rel


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


def test_pipeline_timeout_reported_and_context_survives(kz):
    """The fused step's bounded waits: with the loaders held back, every CTA
    gives up after 10 ms, reports KVZIP_ERR_TIMEOUT and writes no scores;
    afterwards the same steps succeed."""
    B, G, n_c, d, n_ins = 4, 4, 4096, 128, (300, 300)
    k, chunks = make_context(14, B, G, n_c, d, n_ins)
    kd = k.cuda()
    dch = [(q.cuda(), ks.cuda()) for q, ks in chunks]
    ws = kz.new_context_workspace(B, G, max(n_ins))
    S = torch.zeros(B, n_c, device="cuda")
    kz.score_pipeline_step(0, dch[0], None, kd, S, ws)   # chunk 0 normalisers
    assert kz.workspace_status(ws) == kz.OK
    kz.set_wait_timeout_ns(10_000_000)
    kz.set_test_stall(True)
    try:
        kz.score_pipeline_step(1, dch[1], dch[0], kd, S, ws)
        status = kz.workspace_status(ws)
    finally:
        kz.set_test_stall(False)
        kz.set_wait_timeout_ns(0)
    assert status == kz.ERR_TIMEOUT
    assert torch.count_nonzero(S) == 0
    assert kz.workspace_status(ws) == kz.OK
    S.zero_()
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
    small = kz.new_context_workspace(B, G, 32)   # slots too small for the 400-row chunk
    assert kz.context_workspace_size(B, G, 400) > small.numel()
    with pytest.raises(kz.KvzipError):
        kz.score_context(dch, kd, S, small)
