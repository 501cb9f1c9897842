"""Bitwise repeatability of both scorer passes at full size.

Pass 1 writes each query row's normaliser from one thread's own running sum,
and pass 2 gives every context key to exactly one thread, which updates its
score with a plain read-max-write: no atomics and no order-dependent
reductions.  So the same inputs must give the same bits on every launch.  A
race anywhere in the tile pipeline (an accumulator read before its MMA
finished, an operand tile overwritten while an MMA still reads it, an A tile
in tensor memory that an MMA reads before it was stored) would show up as
bits that differ between runs at unpredictable positions.

Each case scores the same chunk three times, each time into freshly zeroed
scores with a fresh zeroed workspace, and compares the row normalisers and
the scores bit for bit, at the workload's full size in the launch
configuration the benchmark times.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

REPEATS = 3


@pytest.fixture(scope="module")
def kz():
    from attention_score_reduction_b200 import build
    build.build()
    from attention_score_reduction_b200 import kvzip
    return kvzip


def _repeat_chunk(kz, q, k_ctx, ks, units, G):
    n_in = q.shape[2]
    off, stride = kz.lse_layout(G, n_in)
    runs = []
    for _ in range(REPEATS):
        S = torch.zeros(units, k_ctx.shape[1], dtype=torch.float32, device=k_ctx.device)
        ws = kz.new_score_workspace(units, G, n_in, k_ctx.device)
        kz.score_chunk(q, k_ctx, ks, S, ws)
        assert kz.workspace_status(ws) == kz.OK
        lse = ws[off:off + units * stride * 4].clone()
        runs.append((lse, S))
        del ws
    lse0, s0 = runs[0]
    assert bool((s0 > 0).any())
    for i, (lse, S) in enumerate(runs[1:], start=1):
        assert torch.equal(lse, lse0), f"row normalisers differ between run 0 and run {i}"
        if not torch.equal(S, s0):
            diff = (S != s0).nonzero()
            raise AssertionError(f"scores differ between run 0 and run {i} at "
                                 f"{diff.shape[0]} positions, first {diff[:4].tolist()}")


def test_llama8b_128k_chunks_repeat_bitwise(kz):
    """LLaMA3.1-8B shape, 128K context, all 256 units, chunks 0, 31 and 63."""
    from attention_score_reduction_b200 import synth
    wl = synth.WORKLOADS["llama8b_128k"]
    dev = torch.device("cuda", 0)
    k_ctx = synth.context_keys(wl, device=dev)
    for c in (0, 31, 63):
        q, ks = synth.chunk_qk(wl, c, device=dev)
        _repeat_chunk(kz, q, k_ctx, ks, wl.units, wl.G)
        del q, ks
    del k_ctx
    torch.cuda.empty_cache()


def test_gemma12b_170k_chunks_repeat_bitwise(kz):
    """Gemma3-12B shape (d = 256, A tiles in tensor memory in both passes),
    170K context, all 384 units, chunk size 2048: first, middle and last chunk."""
    from attention_score_reduction_b200 import synth
    wl = synth.WORKLOADS["gemma12b_170k"]
    dev = torch.device("cuda", 0)
    k_ctx = synth.context_keys(wl, device=dev)
    for c in (0, 42, wl.n_chunks - 1):
        q, ks = synth.chunk_qk(wl, c, device=dev)
        _repeat_chunk(kz, q, k_ctx, ks, wl.units, wl.G)
        del q, ks
    del k_ctx
    torch.cuda.empty_cache()
