"""Full-size parity for the other workload shapes (one chunk each, every unit
scored in one launch; sampled units checked in full against the oracle):

* LLaMA3.1-8B shape, 16K context (32 x 8 units, G = 4, d = 128);
* Qwen2.5-14B shape, 120K context (48 x 8 units, G = 5, d = 128, keys with a
  lognormal(0, 0.5) per-row norm);
* Gemma3-12B shape, 170K context (48 x 8 units, G = 2, d = 256), chunk sizes
  1024, 2048 and 4096 (the last chunk at 4096 is ragged: 2048 rows).

The oracle handles one query head of one unit at a time (rows of different
query heads only meet in the final max), so a unit's reference is the max
over its G query heads.
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


def _oracle_unit(q_b, k_b, ks_b):
    f = lambda t: t.double().numpy()  # noqa: E731
    k64, ks64 = f(k_b), f(ks_b)
    out = None
    for g in range(q_b.shape[0]):
        s, _ = oracle.unit_chunk_scores(f(q_b[g:g + 1]), k64, ks64)
        out = s if out is None else np.maximum(out, s)
    return out


def _run(kz, wl, chunk, units):
    from attention_score_reduction_b200 import synth
    dev = torch.device("cuda", 0)
    k_ctx = synth.context_keys(wl, device=dev)
    q, ks = synth.chunk_qk(wl, chunk, device=dev)
    S = torch.zeros(wl.units, wl.n_c, device=dev)
    ws = kz.new_score_workspace(wl.units, wl.G, q.shape[2])
    kz.score_chunk(q, k_ctx, ks, S, ws)
    assert kz.workspace_status(ws) == kz.OK
    for b in units:
        want = _oracle_unit(q[b].cpu(), k_ctx[b].cpu(), ks[b].cpu())
        got = S[b].cpu().double().numpy()
        err = float(np.max(np.abs(got - want) / want))
        assert err <= RTOL, (wl.name, chunk, b, err)
    del k_ctx, q, ks, S
    torch.cuda.empty_cache()


def test_llama8b_16k(kz):
    from attention_score_reduction_b200 import synth
    _run(kz, synth.WORKLOADS["llama8b_16k"], chunk=7, units=(0, 200))


def test_qwen14b_120k(kz):
    from attention_score_reduction_b200 import synth
    _run(kz, synth.WORKLOADS["qwen14b_120k"], chunk=30, units=(383,))


@pytest.mark.parametrize("m,chunk", [(1024, 0), (2048, 84), (4096, 42)])
def test_gemma12b_170k_chunk_sweep(kz, m, chunk):
    from attention_score_reduction_b200 import synth
    wl = synth.WORKLOADS["gemma12b_170k"].with_(m=m)
    if m == 4096:
        assert wl.n_chunks == 43 and wl.n_in(chunk) == 16 + 2048     # ragged last chunk
    _run(kz, wl, chunk=chunk, units=(191,))
