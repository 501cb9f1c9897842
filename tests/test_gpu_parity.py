"""CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Scores: max relative error <= 2e-3 (bf16 inputs converted exactly, products in
fp32 on the tensor cores / CUDA cores, fp32 log-sum-exp; the oracle works in
float64).  Selection and compaction run on identical score arrays and must be
bit-exact: same keep mask, offsets, threshold, compacted bytes and positions.
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


def make_inputs(seed, B, G, n_in, n_c, d, dtype=torch.bfloat16, hi_frac=0.02):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, G, n_in, d, generator=g)
    k = torch.randn(B, n_c, d, generator=g)
    ks = torch.randn(B, n_in, d, generator=g)
    if hi_frac > 0:
        k = k * torch.where(torch.rand(B, n_c, 1, generator=g) < hi_frac, 3.0, 1.0)
        ks = ks * torch.where(torch.rand(B, n_in, 1, generator=g) < hi_frac, 3.0, 1.0)
    k[:, : min(4, n_c)] *= 5.0  # sinks
    return q.to(dtype), k.to(dtype), ks.to(dtype)


def oracle_scores(q, k, ks, S0):
    S = f64(S0).copy()
    oracle.score_chunk(f64(q), f64(k), f64(ks), S)
    return S


def max_rel(got, want):
    return float(np.max(np.abs(got - want) / want))


SCORE_SHAPES = [  # (B, G, n_in, n_c, d)
    (2, 4, 100, 300, 128),    # ragged context tail, one ragged query tile
    (1, 1, 1, 1, 128),        # one row, one key
    (3, 2, 17, 1000, 128),    # n_in < tile: a CTA's rows span several query heads
    (2, 5, 200, 777, 128),    # G = 5 (Qwen2.5-14B grouping), ragged everywhere
    (1, 4, 528, 2048, 128),   # R and n_c multiples of the tiles
    (1, 4, 129, 2048, 128),   # R = 516: crosses a 256-row CTA boundary by 4
    (2, 2, 150, 500, 256),    # head dim 256
    (1, 3, 129, 129, 256),
]


@pytest.mark.parametrize("shape", SCORE_SHAPES, ids=lambda s: "B%d_G%d_nin%d_nc%d_d%d" % s)
def test_score_chunk_bf16_matches_oracle(kz, shape):
    B, G, n_in, n_c, d = shape
    q, k, ks = make_inputs(sum(shape), B, G, n_in, n_c, d)
    S0 = torch.zeros(B, n_c)
    want = oracle_scores(q, k, ks, S0)
    S = S0.cuda()
    ws = kz.new_score_workspace(B, G, n_in)
    kz.score_chunk(q.cuda(), k.cuda(), ks.cuda(), S, ws)
    assert kz.workspace_status(ws) == kz.OK
    got = S.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    err = max_rel(got, want)
    assert err <= RTOL, err
    # row normalisers of pass 1 against the oracle's
    lse = kz.read_lse(ws, B, G, n_in).cpu().double().numpy()
    for b in range(B):
        _, lse_ref = oracle.unit_chunk_scores(f64(q[b]), f64(k[b]), f64(ks[b]))
        assert np.max(np.abs(lse[b] - lse_ref)) < 1e-3


def test_score_chunk_merges_running_max(kz):
    """Non-zero incoming scores: the result is max(old, chunk score) elementwise."""
    B, G, n_in, n_c, d = 2, 4, 64, 500, 128
    q, k, ks = make_inputs(7, B, G, n_in, n_c, d)
    g = torch.Generator().manual_seed(8)
    S0 = torch.rand(B, n_c, generator=g) * 0.02
    want = oracle_scores(q, k, ks, S0)
    S = S0.cuda()
    kz.score_chunk(q.cuda(), k.cuda(), ks.cuda(), S)
    assert max_rel(S.cpu().double().numpy(), want) <= RTOL


def test_score_chunk_f32_tiny_workload(kz):
    """The tiny single-head fp32 workload: G=4, d=128, n_c=2048, one chunk of
    16 prompt + 496 context rows, 1% of keys scaled x3."""
    from attention_score_reduction_b200 import synth
    wl = synth.WORKLOADS["tiny_fp32"]
    k = synth.context_keys(wl)
    q, ks = synth.chunk_qk(wl, 0)
    assert q.dtype == torch.float32 and q.shape == (1, 4, 512, 128)
    S0 = torch.zeros(1, wl.n_c)
    want = oracle_scores(q, k, ks, S0)
    S = S0.cuda()
    kz.score_chunk(q.cuda(), k.cuda(), ks.cuda(), S)
    assert max_rel(S.cpu().double().numpy(), want) <= RTOL


def test_score_is_idempotent_and_order_free(kz):
    """Re-scoring a chunk leaves scores unchanged; chunk order does not matter."""
    B, G, d, n_c = 2, 2, 128, 400
    _, k, _ = make_inputs(11, B, G, 1, n_c, d)
    chunks = [make_inputs(20 + c, B, G, 90 + 30 * c, 1, d)[0::2] for c in range(3)]
    kd = k.cuda()
    S1 = torch.zeros(B, n_c, device="cuda")
    for q, ks in chunks:
        kz.score_chunk(q.cuda(), kd, ks.cuda(), S1)
    snap = S1.clone()
    kz.score_chunk(chunks[1][0].cuda(), kd, chunks[1][1].cuda(), S1)
    assert torch.equal(S1, snap)
    S2 = torch.zeros(B, n_c, device="cuda")
    for q, ks in reversed(chunks):
        kz.score_chunk(q.cuda(), kd, ks.cuda(), S2)
    assert torch.equal(S1, S2)
    want = oracle.score_context([f64(q) for q, _ in chunks], [f64(ks) for _, ks in chunks], f64(k))
    assert max_rel(S1.cpu().double().numpy(), want) <= RTOL


# ------------------------------------------------------------------ selection

SELECT_CASES = [  # (n_heads, n_c, levels, r)
    (8, 1000, 0, 0.3),
    (8, 1000, 8, 0.3),       # tie-heavy: 8 distinct values
    (3, 20000, 2, 0.5),      # two values: half the array ties at the threshold
    (5, 777, 0, 0.0),
    (5, 777, 0, 1.0),
    (1, 9000, 0, 0.3),       # one head, two mask blocks
    (256, 4096, 0, 0.3),
    (16, 333, 1, 0.42),      # every score equal
]


@pytest.mark.parametrize("case", SELECT_CASES, ids=lambda c: "H%d_nc%d_lv%d_r%.2f" % c)
def test_select_bit_exact(kz, case):
    from attention_score_reduction_b200 import synth
    n_heads, n_c, levels, r = case
    s = synth.random_scores(n_heads, n_c, seed=n_c + levels, levels=levels)
    N = s.numel()
    k = kz.keep_count(r, N)
    keep, off, thr = kz.select(s.reshape(-1).cuda(), k, n_heads)
    keep_ref, off_ref, thr_ref = oracle.select(s.reshape(-1).numpy(), k, n_heads)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert float(thr.item()) == thr_ref


def test_select_config_shape_scores(kz):
    """LLaMA3.1-8B-shaped 16K context (32 x 8 heads x 16384), r = 0.3."""
    from attention_score_reduction_b200 import synth
    s = synth.random_scores(256, 16384, seed=5)
    k = kz.keep_count(0.3, s.numel())
    keep, off, thr = kz.select(s.reshape(-1).cuda(), k, 256)
    keep_ref, off_ref, thr_ref = oracle.select(s.reshape(-1).numpy(), k, 256)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert float(thr.item()) == thr_ref
    assert int(off[-1]) == k == 1258292


def test_select_no_scores(kz):
    """N = 0: every head keeps nothing and the threshold is +inf, written by one
    enqueued kernel (the call does not synchronise)."""
    n_heads = 5
    s = torch.empty(0, dtype=torch.float32, device="cuda")
    keep = torch.empty(0, dtype=torch.uint8, device="cuda")
    off = torch.full((n_heads + 1,), -7, dtype=torch.int64, device="cuda")
    thr = torch.zeros(1, dtype=torch.float32, device="cuda")
    nws = kz.select_workspace_size(0, n_heads)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    st = kz.library().kvzip_select(None, 0, 0, n_heads, None, off.data_ptr(), thr.data_ptr(),
                                   ws.data_ptr(), nws, torch.cuda.current_stream().cuda_stream)
    assert st == kz.OK and kz.last_launch_count() == 1
    torch.cuda.synchronize()
    assert off.tolist() == [0] * (n_heads + 1)
    assert float(thr.item()) == float("inf")
    del keep, s


def _signed_zero_scores(n_heads, n_c, seed):
    """Scores in {0.0, -0.0, 0.125, 0.5}: -0.0 equals 0.0, so at r = 0.5 the
    threshold is 0 and the zeros of both signs tie, ranked by index."""
    g = np.random.default_rng(seed)
    s = g.choice(np.array([0.0, 0.125, 0.5], np.float32), size=(n_heads, n_c),
                 p=[0.6, 0.25, 0.15])
    s[(s == 0) & (g.random(s.shape) < 0.5)] = np.float32(-0.0)
    assert np.signbit(s).any()
    return s


def _inf_scores(n_heads, n_c, seed):
    """Uniform scores with 5% +inf: at r = 0.03 the threshold is +inf (the
    k-th largest lies in the infinity bin), at r = 0.3 it is finite."""
    g = np.random.default_rng(seed)
    s = g.random((n_heads, n_c), dtype=np.float32)
    s[g.random(s.shape) < 0.05] = np.inf
    return s


@pytest.mark.parametrize("make,rs", [(_signed_zero_scores, (0.3, 0.5, 0.9)),
                                     (_inf_scores, (0.03, 0.3))], ids=["signed_zero", "inf"])
def test_select_signed_zero_and_inf(kz, make, rs):
    """Scores compare by value: -0.0 ranks as 0.0 (not by its raw bits, which
    would rank it above every score), and +inf above every finite score, for
    the global selection, the uniform per-head budgets and head/token scores."""
    n_heads, n_c = 12, 5000
    s = make(n_heads, n_c, seed=n_c)
    sd = torch.from_numpy(s).cuda()
    for r in rs:
        k = kz.keep_count(r, s.size)
        keep, off, thr = kz.select(sd.reshape(-1), k, n_heads)
        keep_ref, off_ref, thr_ref = oracle.select(s.reshape(-1), k, n_heads)
        assert np.array_equal(keep.cpu().numpy(), keep_ref), r
        assert np.array_equal(off.cpu().numpy(), off_ref), r
        assert float(thr.item()) == thr_ref
        k_h = oracle.keep_count(r, n_c)
        keep_h, off_h = kz.select_per_head(sd, k_h)
        keep_h_ref, off_h_ref = oracle.select_per_head(s.reshape(-1), k_h, n_heads)
        assert np.array_equal(keep_h.cpu().numpy(), keep_h_ref), r
        assert np.array_equal(off_h.cpu().numpy(), off_h_ref), r
    assert np.array_equal(kz.head_scores(sd).cpu().numpy(),
                          oracle.head_scores(s, 1, n_heads).reshape(-1).astype(np.float32))
    assert np.array_equal(kz.token_scores(sd).cpu().numpy(),
                          oracle.token_scores(s).astype(np.float32))


# ------------------------------------------------------------------ compaction

@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("n_heads,n_c,r", [(6, 5000, 0.3), (2, 100, 0.5), (4, 4096, 1.0),
                                           (3, 9001, 0.01), (2, 64, 0.0)])
def test_compact_bit_exact(kz, d, n_heads, n_c, r):
    from attention_score_reduction_b200 import synth
    g = torch.Generator().manual_seed(n_c + d)
    K = torch.randn(n_heads, n_c, d, generator=g).to(torch.bfloat16)
    V = torch.randn(n_heads, n_c, d, generator=g).to(torch.bfloat16)
    s = synth.random_scores(n_heads, n_c, seed=n_heads * 7 + n_c)
    k = kz.keep_count(r, s.numel())
    keep_ref, off_ref, _ = oracle.select(s.reshape(-1).numpy(), k, n_heads)
    ko_ref, vo_ref, pos_ref = oracle.compact(K.view(torch.int16).numpy(),
                                             V.view(torch.int16).numpy(), keep_ref, off_ref)
    keep = torch.from_numpy(keep_ref).cuda()
    off = torch.from_numpy(off_ref).cuda()
    ko, vo, pos = kz.compact(K.cuda(), V.cuda(), keep, off, k)
    assert np.array_equal(ko.cpu().view(torch.int16).numpy(), ko_ref)
    assert np.array_equal(vo.cpu().view(torch.int16).numpy(), vo_ref)
    assert np.array_equal(pos.cpu().numpy(), pos_ref)


# ------------------------------------------------------------------ whole path

def test_small_context_end_to_end(kz):
    """Score every chunk of a small multi-layer context, select globally,
    compact: scores within tolerance of the oracle; selection and compaction
    bit-exact on the GPU's own score array."""
    from attention_score_reduction_b200 import synth
    wl = synth.Workload("small", L=2, H=2, G=4, d=128, n_c=600, m=256, r=(0.3,), hi_frac=0.01,
                        sinks=4, cfg_id=90)
    k_ctx, v = synth.context_kv(wl)
    qs, kss = zip(*[synth.chunk_qk(wl, c) for c in range(wl.n_chunks)])
    S = torch.zeros(wl.units, wl.n_c, device="cuda")
    kd = k_ctx.cuda()
    for q, ks in zip(qs, kss):
        kz.score_chunk(q.cuda(), kd, ks.cuda(), S)
    want = oracle.score_context([f64(q) for q in qs], [f64(k) for k in kss], f64(k_ctx))
    assert max_rel(S.cpu().double().numpy(), want) <= RTOL
    k = kz.keep_count(0.3, S.numel())
    keep, off, thr = kz.select(S.reshape(-1), k, wl.units)
    s_host = S.reshape(-1).cpu().numpy()
    keep_ref, off_ref, thr_ref = oracle.select(s_host, k, wl.units)
    assert np.array_equal(keep.cpu().numpy(), keep_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    ko, vo, pos = kz.compact(kd, v.cuda(), keep, off, k)
    ko_ref, vo_ref, pos_ref = oracle.compact(k_ctx.view(torch.int16).numpy(),
                                             v.view(torch.int16).numpy(), keep_ref, off_ref)
    assert np.array_equal(ko.cpu().view(torch.int16).numpy(), ko_ref)
    assert np.array_equal(vo.cpu().view(torch.int16).numpy(), vo_ref)
    assert np.array_equal(pos.cpu().numpy(), pos_ref)


# ------------------------------------------------------------------ head scores

@pytest.mark.parametrize("n_heads,n_c", [(256, 16384), (3, 40000), (5, 7), (1, 1)])
def test_head_scores_bit_exact(kz, n_heads, n_c):
    from attention_score_reduction_b200 import synth
    s = synth.random_scores(n_heads, n_c, seed=n_heads + n_c)
    got = kz.head_scores(s.cuda()).cpu().numpy()
    L = 1
    want = oracle.head_scores(s.numpy(), L, n_heads)[0]
    assert np.array_equal(got, want.astype(np.float32))


@pytest.mark.parametrize("jump", [45.0, 70.0, 100.0, 126.0, 130.0, 200.0])
def test_score_chunk_late_dominant_key(kz, jump):
    """A context key far down the sequence outscores every earlier key by `jump`
    in log2 units (all query rows share one direction, the key is a multiple of
    it), from well inside to far past the range of fp32 exponentials taken
    against any earlier maximum (2^126 is the largest power of two the
    polynomial exponentials reach, 2^128 overflows).  The online maximum must
    rescale the row sum exactly.  Scores above 1e-30 match the oracle to 2e-3,
    the rest are below 1e-30 (probabilities below 2^-126 flush to zero)."""
    B, G, n_in, n_c, d = 2, 2, 40, 2000, 128
    g = torch.Generator().manual_seed(int(jump))
    u = torch.randn(d, generator=g)
    q = (u.repeat(B, G, n_in, 1) + 0.05 * torch.randn(B, G, n_in, d, generator=g)).to(torch.bfloat16)
    k = torch.randn(B, n_c, d, generator=g)
    ks = torch.randn(B, n_in, d, generator=g)
    c = 1.4426950408889634 / np.sqrt(d)
    beta = jump / (c * float(u @ u))
    # two keys: the polynomial takes the first 4 of every 16 accumulator columns
    # (tiles and chunks start on multiples of 16), so key 1488 lands on the
    # polynomial and key 1500 on MUFU
    k[:, 1488] = beta * u
    k[:, 1500] = beta * u
    k, ks = k.to(torch.bfloat16), ks.to(torch.bfloat16)
    want = oracle_scores(q, k, ks, torch.zeros(B, n_c))
    S = torch.zeros(B, n_c, device="cuda")
    ws = kz.new_score_workspace(B, G, n_in)
    kz.score_chunk(q.cuda(), k.cuda(), ks.cuda(), S, ws)
    assert kz.workspace_status(ws) == kz.OK
    got = S.cpu().double().numpy()
    assert np.all(np.isfinite(got))
    assert got[:, [1488, 1500]].min() > 0.49
    big = want > 1e-30
    assert float(np.max(np.abs(got[big] - want[big]) / want[big])) <= RTOL
    if (~big).any():
        assert float(np.max(np.abs(got[~big]))) <= 1e-30
