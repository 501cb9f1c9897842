"""pipeline.compress_from_host: the same compression from pinned host buffers.

A small multi-layer context with more chunks than device chunk buffers, so
the uploads reuse a ring of two device slots (each upload waits until the
scorer is done with the slot's previous chunk).  The context keys arrive in
runs of units (1, 3 and 4 runs: the first chunk is scored run by run) and V
in pieces behind the later chunks.  The packed cache, positions and offsets
read back to the host must equal the device-resident path's
(Compressor.compress) bit for bit, and the scores must too: same kernels.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _pinned(t):
    return t.contiguous().pin_memory()


@pytest.mark.parametrize("key_slices", [1, 3, 4])
def test_host_pipeline_matches_device_path_with_buffer_ring(key_slices):
    from attention_score_reduction_b200 import build
    build.build()
    from attention_score_reduction_b200 import pipeline, synth
    wl = synth.Workload("host_ring", L=2, H=4, G=4, d=128, n_c=3000, m=700, r=(0.3,),
                        hi_frac=0.01, sinks=4, cfg_id=91)
    dev = torch.device("cuda", 0)
    k_ctx, v = synth.context_kv(wl)
    chunks = [synth.chunk_qk(wl, c) for c in range(wl.n_chunks)]
    assert len(chunks) == 5 and chunks[-1][0].shape[2] != chunks[0][0].shape[2]   # ragged last
    max_n_in = max(q.shape[2] for q, _ in chunks)

    ref = pipeline.Compressor(wl.units, wl.n_c, wl.d, wl.G, max_n_in, device=dev)
    out_ref = ref.compress(k_ctx.to(dev), v.to(dev), [(q.to(dev), ks.to(dev)) for q, ks in chunks],
                           r=0.3)
    torch.cuda.synchronize()
    ref.check_status()

    comp = pipeline.Compressor(wl.units, wl.n_c, wl.d, wl.G, max_n_in, device=dev)
    q0, ks0 = chunks[0]
    ring = [(torch.empty(wl.units, wl.G, max_n_in, wl.d, dtype=q0.dtype, device=dev),
             torch.empty(wl.units, max_n_in, wl.d, dtype=ks0.dtype, device=dev)) for _ in range(2)]
    bufs = {"k_ctx": torch.empty_like(k_ctx, device=dev), "v": torch.empty_like(v, device=dev),
            "q": [q for q, _ in ring], "ks": [ks for _, ks in ring]}
    kept = out_ref.kept
    host_out = {"k": torch.empty(kept, wl.d, dtype=torch.bfloat16).pin_memory(),
                "v": torch.empty(kept, wl.d, dtype=torch.bfloat16).pin_memory(),
                "pos": torch.empty(kept, dtype=torch.int32).pin_memory(),
                "offsets": torch.empty(wl.units + 1, dtype=torch.int64).pin_memory()}
    for _ in range(2):   # twice: the second pass reuses every buffer
        out, host_out, h2d, d2h = pipeline.compress_from_host(
            comp, _pinned(k_ctx), _pinned(v), [_pinned(q) for q, _ in chunks],
            [_pinned(ks) for _, ks in chunks], 0.3, bufs, host_out, key_slices=key_slices)
        torch.cuda.synchronize()
        comp.check_status()
        assert torch.equal(comp.scores, ref.scores)
        assert out.kept == kept
        assert torch.equal(host_out["offsets"], out_ref.offsets.cpu())
        assert torch.equal(host_out["k"].view(torch.int16), out_ref.k.cpu().view(torch.int16))
        assert torch.equal(host_out["v"].view(torch.int16), out_ref.v.cpu().view(torch.int16))
        assert torch.equal(host_out["pos"], out_ref.pos.cpu())
    in_bytes = sum(t.numel() * t.element_size() for t in (k_ctx, v)) + \
        sum(q.numel() * q.element_size() + ks.numel() * ks.element_size() for q, ks in chunks)
    assert h2d == in_bytes
    assert d2h == kept * wl.d * 2 * 2 + kept * 4 + (wl.units + 1) * 8


def test_host_pipeline_single_chunk_context():
    """One chunk: it is both the first chunk (scored run by run as the keys
    land) and the last (its runs count the round-1 histogram); V goes up whole."""
    from attention_score_reduction_b200 import build
    build.build()
    from attention_score_reduction_b200 import pipeline, synth
    wl = synth.Workload("host_one", L=1, H=4, G=2, d=128, n_c=500, m=600, r=(0.3,),
                        hi_frac=0.01, sinks=4, cfg_id=92)
    assert wl.n_chunks == 1
    dev = torch.device("cuda", 0)
    k_ctx, v = synth.context_kv(wl)
    q, ks = synth.chunk_qk(wl, 0)
    ref = pipeline.Compressor(wl.units, wl.n_c, wl.d, wl.G, q.shape[2], device=dev)
    out_ref = ref.compress(k_ctx.to(dev), v.to(dev), [(q.to(dev), ks.to(dev))], r=0.3)
    comp = pipeline.Compressor(wl.units, wl.n_c, wl.d, wl.G, q.shape[2], device=dev)
    bufs = {"k_ctx": torch.empty_like(k_ctx, device=dev), "v": torch.empty_like(v, device=dev),
            "q": [torch.empty_like(q, device=dev)], "ks": [torch.empty_like(ks, device=dev)]}
    out, _, h2d, _ = pipeline.compress_from_host(comp, _pinned(k_ctx), _pinned(v), [_pinned(q)],
                                                 [_pinned(ks)], 0.3, bufs)
    torch.cuda.synchronize()
    comp.check_status()
    assert torch.equal(comp.scores, ref.scores)
    assert torch.equal(out.offsets, out_ref.offsets)
    assert torch.equal(out.k.view(torch.int16), out_ref.k.view(torch.int16))
    assert torch.equal(out.pos, out_ref.pos)
    assert h2d == sum(t.numel() * t.element_size() for t in (k_ctx, v, q, ks))
