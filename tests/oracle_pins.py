"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each pin takes an oracle module ``o`` and raises AssertionError when the
oracle disagrees with a closed form, an invariant, a brute-force computation
on tiny inputs, or a value printed on the KVzip pages.  The same pins run
against deliberately broken copies of the oracle (tests/test_oracle_pins.py)
to show that each plausible mistake is caught by at least one of them.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _inputs(seed, B, G, n_in, n_c, d, chunks=1):
    r = _rng(seed)
    k_ctx = r.standard_normal((B, n_c, d))
    qs = [r.standard_normal((B, G, n_in, d)) for _ in range(chunks)]
    kss = [r.standard_normal((B, n_in, d)) for _ in range(chunks)]
    return qs, kss, k_ctx


# ---------------------------------------------------------------- scoring pins

def pin_row_sums_and_range(o):
    """Softmax rows sum to 1 (1e-12) and every score lies in (0, 1]."""
    qs, kss, k_ctx = _inputs(1, 2, 3, 9, 20, 8, chunks=2)
    scale = 1 / math.sqrt(8)
    for q, ks in zip(qs, kss):
        for b in range(2):
            p = o.softmax_rows(o.chunk_logits(q[b], k_ctx[b], ks[b], scale))
            assert np.allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    S = o.score_context(qs, kss, k_ctx)
    assert np.all(S > 0) and np.all(S <= 1.0 + 1e-15)


def pin_uniform_queries(o):
    """Q = 0: row (g, i) is uniform over n_c + i + 1 keys, so S[j] = 1/(n_c + 1)
    (the row i = 0 wins) and lse_i = log(n_c + i + 1)."""
    for (G, n_in, n_c, d, chunks) in [(1, 5, 7, 4, 1), (3, 6, 11, 8, 2), (2, 17, 33, 16, 3)]:
        r = _rng(2)
        k_ctx = r.standard_normal((1, n_c, d)) * 3
        qs = [np.zeros((1, G, n_in, d)) for _ in range(chunks)]
        kss = [r.standard_normal((1, n_in, d)) for _ in range(chunks)]
        S = o.score_context(qs, kss, k_ctx)
        assert np.allclose(S, 1.0 / (n_c + 1), rtol=1e-13, atol=0)
        _, lse = o.unit_chunk_scores(qs[0][0], k_ctx[0], kss[0][0])
        i = np.tile(np.arange(n_in), G)
        assert np.allclose(lse, np.log(n_c + i + 1), rtol=1e-13, atol=1e-13)


def pin_logistic(o):
    """n_c = 1, n_in = 1, G = 1: S = sigmoid(s - s') with s = q.k / sqrt(d),
    s' = q.k_self / sqrt(d) (the single row sees one context key and itself)."""
    r = _rng(3)
    for d in (4, 64, 128):
        for _ in range(5):
            q = r.standard_normal((1, 1, 1, d))
            k = r.standard_normal((1, 1, d))
            ks = r.standard_normal((1, 1, d))
            s = float(q[0, 0, 0] @ k[0, 0]) / math.sqrt(d)
            sp = float(q[0, 0, 0] @ ks[0, 0]) / math.sqrt(d)
            S = o.score_context([q], [ks], k)
            want = 1.0 / (1.0 + math.exp(sp - s))
            assert abs(S[0, 0] - want) <= 1e-14, (S[0, 0], want)


def pin_dominant_key(o):
    """A context key far larger than the rest and aligned with one query row
    takes essentially all of that row's mass: S -> 1 for that key, while a
    mean over rows would stay near 1/rows."""
    r = _rng(4)
    G, n_in, n_c, d = 2, 8, 30, 16
    q = r.standard_normal((1, G, n_in, d))
    k = r.standard_normal((1, n_c, d))
    ks = r.standard_normal((1, n_in, d))
    u = q[0, 1, 5] / np.linalg.norm(q[0, 1, 5])
    k[0, 17] = 400.0 * u
    S = o.score_context([q], [ks], k)
    assert S[0, 17] > 1 - 1e-12, S[0, 17]


def _bruteforce_pure_python(qs, kss, k_ctx, scale):
    """Dense, unchunked: every row of every chunk in one matrix whose columns
    are the n_c context keys followed by the self keys of *all* chunks; a row
    of chunk c at position i sees context keys and chunk c's self keys 0..i
    (block-diagonal causal mask).  Global column max over all rows."""
    B, n_c, d = k_ctx.shape
    out = [[0.0] * n_c for _ in range(B)]
    for b in range(B):
        cols = [list(map(float, k_ctx[b, j])) for j in range(n_c)]
        owner = [(-1, j) for j in range(n_c)]
        for c, ks in enumerate(kss):
            for jp in range(ks.shape[1]):
                cols.append(list(map(float, ks[b, jp])))
                owner.append((c, jp))
        for c, q in enumerate(qs):
            G, n_in = q.shape[1], q.shape[2]
            for g in range(G):
                for i in range(n_in):
                    row = list(map(float, q[b, g, i]))
                    logit = []
                    for col, (oc, jp) in zip(cols, owner):
                        visible = oc == -1 or (oc == c and jp <= i)
                        if visible:
                            logit.append(scale * sum(x * y for x, y in zip(row, col)))
                        else:
                            logit.append(None)
                    mx = max(v for v in logit if v is not None)
                    z = sum(math.exp(v - mx) for v in logit if v is not None)
                    for j in range(n_c):
                        p = math.exp(logit[j] - mx) / z
                        if p > out[b][j]:
                            out[b][j] = p
    return np.array(out)


def pin_bruteforce_unchunked(o):
    """Chunked running max == one dense unchunked matrix over all chunks' rows
    with a block-diagonal causal self mask, on tiny inputs (pure Python)."""
    cases = [  # (G, n_in, n_c, d, chunks)
        (1, 8, 24, 4, 3),
        (2, 11, 16, 16, 2),
        (4, 6, 20, 8, 2),
        (2, 19, 40, 128, 2),
    ]
    for seed, (G, n_in, n_c, d, chunks) in enumerate(cases):
        qs, kss, k_ctx = _inputs(10 + seed, 2, G, n_in, n_c, d, chunks)
        k_ctx[:, :3] *= 3.0
        want = _bruteforce_pure_python(qs, kss, k_ctx, 1 / math.sqrt(d))
        got = o.score_context(qs, kss, k_ctx)
        assert np.allclose(got, want, rtol=1e-12, atol=0), np.abs(got / want - 1).max()


def pin_invariants(o):
    """Chunk order, query-head order and duplicated query heads leave S
    unchanged; permuting the context keys permutes S; re-scoring a chunk is
    idempotent."""
    qs, kss, k_ctx = _inputs(20, 2, 3, 10, 25, 8, chunks=3)
    S = o.score_context(qs, kss, k_ctx)
    # chunk order
    S2 = o.score_context(qs[::-1], kss[::-1], k_ctx)
    assert np.array_equal(S, S2)
    # query-head permutation and duplication
    perm = [2, 0, 1]
    S3 = o.score_context([q[:, perm] for q in qs], kss, k_ctx)
    assert np.allclose(S, S3, rtol=1e-14, atol=0)
    S4 = o.score_context([np.concatenate([q, q[:, :1]], axis=1) for q in qs], kss, k_ctx)
    assert np.allclose(S, S4, rtol=1e-14, atol=0)
    # key permutation
    pk = _rng(21).permutation(25)
    S5 = o.score_context(qs, kss, k_ctx[:, pk])
    assert np.allclose(S5, S[:, pk], rtol=1e-13, atol=0)
    # idempotent re-scoring
    S6 = S.copy()
    o.score_chunk(qs[1], k_ctx, kss[1], S6)
    assert np.array_equal(S6, S)


def pin_rows_see_own_prefix(o):
    """Changing a self key j' changes only rows i >= j': checked through the
    lse of each row (rows i < j' keep their lse exactly)."""
    r = _rng(30)
    G, n_in, n_c, d = 2, 9, 12, 8
    q = r.standard_normal((G, n_in, d))
    k = r.standard_normal((n_c, d))
    ks = r.standard_normal((n_in, d))
    _, lse0 = o.unit_chunk_scores(q, k, ks)
    jp = 4
    ks2 = ks.copy()
    ks2[jp] += 5.0
    _, lse1 = o.unit_chunk_scores(q, k, ks2)
    i = np.tile(np.arange(n_in), G)
    assert np.array_equal(lse0[i < jp], lse1[i < jp])
    assert np.all(lse0[i >= jp] != lse1[i >= jp])


# -------------------------------------------------------------- selection pins

def pin_keep_count(o):
    """k = ceil(r N): equals the exact decimal product for the workloads'
    ratios and sizes (e.g. r = 0.3 of 2048 keys keeps 615)."""
    cases = [(0.3, 2048), (0.3, 4194304), (0.3, 33554432), (0.5, 33554432),
             (0.25, 47185920), (0.3, 66846720), (0.0, 100), (1.0, 100), (0.7, 10)]
    for r, N in cases:
        exact = Fraction(str(r)) * N
        want = math.ceil(exact)
        assert o.keep_count(r, N) == want, (r, N, o.keep_count(r, N), want)
    assert o.keep_count(0.3, 2048) == 615


def _check_selection(s, k, n_heads, keep, offsets, threshold):
    s = np.asarray(s).reshape(-1)
    N = s.size
    kept = np.nonzero(keep)[0]
    dropped = np.nonzero(keep == 0)[0]
    assert kept.size == k
    if k and dropped.size:
        # every kept score is >= every dropped score
        assert s[kept].min() >= s[dropped].max()
        # ties at the boundary: kept ones have lower flat index than dropped ones
        tau = s[kept].min()
        tk = kept[s[kept] == tau]
        td = dropped[s[dropped] == tau]
        if td.size:
            assert tk.max() < td.min()
    if k:
        assert threshold == s[kept].min()
    else:
        assert threshold == math.inf
    cnt = keep.reshape(n_heads, -1).sum(axis=1)
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), cnt)
    assert offsets[-1] == k


def pin_select_properties(o):
    """The kept set is the unique set of size k with every kept score >= every
    dropped one and ties kept lowest-index first; offsets are the exclusive
    scan of per-head counts.  Random and tie-heavy arrays, r in {0, .3, .5, 1}."""
    r = _rng(40)
    for levels in (0, 8, 2, 1):
        for n_heads, n_c in [(4, 50), (7, 33), (1, 200)]:
            s = r.random((n_heads, n_c)) ** 4
            if levels:
                s = (np.floor(s * levels) + 1) / levels
            s = s.astype(np.float32)
            for frac in (0.0, 0.3, 0.5, 1.0):
                k = o.keep_count(frac, s.size)
                keep, offsets, thr = o.select(s.reshape(-1), k, n_heads)
                _check_selection(s, k, n_heads, keep, offsets, thr)
    keep, offsets, _ = o.select(np.ones(12, np.float32), 12, 3)
    assert keep.all()


def pin_select_bruteforce(o):
    """Tiny arrays: the kept set equals the best-of-all-subsets answer under the
    order (higher score, then lower index) found by exhaustive search."""
    from itertools import combinations
    r = _rng(41)
    for trial in range(6):
        n_heads, n_c = 2, 4
        code = np.floor(r.random(n_heads * n_c) * 3).astype(np.int64)   # 0, 1, 2
        s = (code / 3).astype(np.float32)
        for k in range(0, 9):
            best = None
            for sub in combinations(range(8), k):
                # preference: larger total score first (exact, in integer codes),
                # then the lexicographically smaller sorted index list
                key = (sum(int(code[i]) for i in sub), tuple(-i for i in sorted(sub)))
                if best is None or key > best[0]:
                    best = (key, sub)
            keep, _, _ = o.select(s, k, n_heads)
            assert set(np.nonzero(keep)[0].tolist()) == set(best[1]), (s, k)


# ------------------------------------------------------------- compaction pins

def pin_select_signed_zero_and_inf(o):
    """Scores compare by value (the ordering reading): -0.0 equals 0.0, so the
    zeros of both signs tie and go lowest index first, and +inf ranks above
    every finite score.  Exhaustive search over all subsets of 8 scores whose
    value codes are exact integers (-0.0 and 0.0 both code 0, +inf codes 9)."""
    from itertools import combinations
    s = np.array([0.0, -0.0, 0.5, np.inf, -0.0, 0.25, 0.0, np.inf], dtype=np.float32)
    code = {0.0: 0, 0.25: 1, 0.5: 2}
    c = [9 if np.isinf(x) else code[float(abs(x))] for x in s]
    for k in range(0, 9):
        best = None
        for sub in combinations(range(8), k):
            key = (sum(c[i] for i in sub), tuple(-i for i in sorted(sub)))
            if best is None or key > best[0]:
                best = (key, sub)
        keep, off, thr = o.select(s, k, 2)
        assert set(np.nonzero(keep)[0].tolist()) == set(best[1]), k
        if k:
            assert thr == min(s[list(best[1])])   # -0.0 == 0.0
        assert off[-1] == k


def pin_compact(o):
    """Compacted rows equal the source rows byte for byte; positions ascend in
    each head; kept bytes = k * d * 2 (bf16) * 2 (K and V)."""
    r = _rng(50)
    n_heads, n_c, d = 5, 37, 8
    k = r.integers(0, 2**16, size=(n_heads, n_c, d), dtype=np.uint16)  # bf16 bit patterns
    v = r.integers(0, 2**16, size=(n_heads, n_c, d), dtype=np.uint16)
    s = r.random(n_heads * n_c).astype(np.float32)
    kk = o.keep_count(0.4, s.size)
    keep, offsets, _ = o.select(s, kk, n_heads)
    ko, vo, pos = o.compact(k, v, keep, offsets)
    assert ko.nbytes + vo.nbytes == kk * d * 2 * 2
    for h in range(n_heads):
        seg = pos[offsets[h]:offsets[h + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.array_equal(seg, np.nonzero(keep.reshape(n_heads, n_c)[h])[0])
        assert np.array_equal(ko[offsets[h]:offsets[h + 1]], k[h, seg])
        assert np.array_equal(vo[offsets[h]:offsets[h + 1]], v[h, seg])


def pin_kv_size_table(o):
    """The rebuttal's decoding table: KV cache size is linear in the kept ratio
    (32.7 GB at ratio 1 -> 26.2, 19.6, 13.1, 6.5).  Compaction bytes from the
    oracle, scaled to 32.7 GB at ratio 1, reproduce every printed size to the
    printed 0.1 GB."""
    with open(os.path.join(GOLDEN, "kv_size_vs_ratio.json")) as f:
        g = json.load(f)
    r = _rng(51)
    n_heads, n_c, d = 8, 1000, 4
    s = r.random(n_heads * n_c).astype(np.float32)
    k = np.zeros((n_heads, n_c, d), np.uint16)
    full = None
    for ratio, gb in zip(g["ratio"], g["kv_cache_gb"]):
        kk = o.keep_count(ratio, s.size)
        keep, offsets, _ = o.select(s, kk, n_heads)
        ko, vo, _ = o.compact(k, k, keep, offsets)
        nbytes = ko.nbytes + vo.nbytes
        if full is None:
            full = nbytes
        assert round(32.7 * nbytes / full, 1) == gb, (ratio, 32.7 * nbytes / full, gb)


# --------------------------------------------------------- decode attention pins

def pin_decode_closed_forms(o):
    """Decode attention: a head with one kept row returns that row's V; zero
    queries average the head's V rows; an empty head returns zeros; a
    dominant aligned key returns its V row."""
    r = _rng(60)
    d, G = 8, 3
    K = r.standard_normal((7, d))
    V = r.standard_normal((7, d))
    offsets = np.array([0, 1, 1, 4, 7])          # heads of 1, 0, 3, 3 rows
    q = r.standard_normal((4, G, d))
    out = o.decode_attention(q, K, V, offsets)
    assert np.allclose(out[0], V[0], rtol=0, atol=1e-14)
    assert np.all(out[1] == 0)
    out0 = o.decode_attention(np.zeros((4, G, d)), K, V, offsets)
    assert np.allclose(out0[2], V[1:4].mean(axis=0), rtol=0, atol=1e-14)
    assert np.allclose(out0[3], V[4:7].mean(axis=0), rtol=0, atol=1e-14)
    K2 = K.copy()
    K2[5] = 200.0 * q[3, 1] / np.linalg.norm(q[3, 1])
    out2 = o.decode_attention(q, K2, V, offsets)
    assert np.allclose(out2[3, 1], V[5], rtol=0, atol=1e-9)


def pin_decode_matches_dense_over_kept(o):
    """Decode attention over the compacted cache equals dense attention over
    the full cache with evicted keys masked out (pure-Python loops)."""
    r = _rng(61)
    n_heads, n_c, d, G = 3, 9, 4, 2
    K = r.standard_normal((n_heads, n_c, d))
    V = r.standard_normal((n_heads, n_c, d))
    s = r.random(n_heads * n_c).astype(np.float32)
    kk = o.keep_count(0.5, s.size)
    keep, offsets, _ = o.select(s, kk, n_heads)
    ko, vo, _ = o.compact(K, V, keep, offsets)
    q = r.standard_normal((n_heads, G, d))
    got = o.decode_attention(q, ko, vo, offsets)
    keep = keep.reshape(n_heads, n_c)
    for h in range(n_heads):
        for g in range(G):
            ls = [(sum(float(a) * float(b) for a, b in zip(q[h, g], K[h, j])) / math.sqrt(d), j)
                  for j in range(n_c) if keep[h, j]]
            if not ls:
                assert np.all(got[h, g] == 0)
                continue
            mx = max(x for x, _ in ls)
            z = sum(math.exp(x - mx) for x, _ in ls)
            want = [sum(math.exp(x - mx) / z * float(V[h, j, t]) for x, j in ls) for t in range(d)]
            assert np.allclose(got[h, g], want, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------- variant pins

def pin_sum_aggregation(o):
    """Sum aggregation: Q = 0 gives S[j] = G * sum_i 1/(n_c + i + 1) (each row
    is uniform over its n_c + i + 1 keys); column sums plus the self-key mass
    account for every row's probability 1 (pure-Python check on a tiny case)."""
    G, n_in, n_c, d = 3, 7, 11, 4
    r = _rng(70)
    k = r.standard_normal((1, n_c, d))
    ks = r.standard_normal((1, n_in, d))
    S = np.zeros((1, n_c))
    o.score_chunk_sum(np.zeros((1, G, n_in, d)), k, ks, S)
    want = G * sum(1.0 / (n_c + i + 1) for i in range(n_in))
    assert np.allclose(S, want, rtol=1e-13, atol=0)
    q = r.standard_normal((G, n_in, d))
    cs = o.unit_chunk_colsums(q, k[0], ks[0])
    self_mass = 0.0
    for g in range(G):
        for i in range(n_in):
            lg = [float(q[g, i] @ k[0, j]) / 2.0 for j in range(n_c)] + \
                 [float(q[g, i] @ ks[0, jp]) / 2.0 for jp in range(i + 1)]
            mx = max(lg)
            z = sum(math.exp(x - mx) for x in lg)
            self_mass += sum(math.exp(x - mx) for x in lg[n_c:]) / z
    assert abs(cs.sum() + self_mass - G * n_in) < 1e-12


def pin_uniform_budgets(o):
    """Uniform budgets keep exactly k_h per head, each head's kept set being its
    own top k_h with ties taken lowest position first (the defining property,
    checked head by head)."""
    r = _rng(71)
    S = (np.floor(r.random((4, 30)) * 6) / 6).astype(np.float32)
    keep, off = o.select_per_head(S.reshape(-1), 9, 4)
    assert np.array_equal(off, [0, 9, 18, 27, 36])
    for h in range(4):
        kh = keep.reshape(4, 30)[h]
        _check_selection(S[h], 9, 1, kh, np.array([0, 9]), S[h][kh == 1].min())


def _planted_scores(L, H, n_c, cells, seed):
    """Background scores in [0, 0.5) with hand-placed larger values at the given
    (l, h, j) cells.  Pure-Python lists, no array reductions."""
    r = _rng(seed)
    S = [[[0.5 * float(r.random()) for _ in range(n_c)] for _ in range(H)] for _ in range(L)]
    for (l, h, j), val in cells.items():
        S[l][h][j] = val
    return S


def pin_head_scores(o):
    """Head-level scores (rebuttal, answer on the head-level scores used for the
    DuoAttention comparison: the maximum over the sequence axis of the
    L x H x n_c score tensor).  L = 3, H = 2, n_c = 5 with one planted maximum
    per head at a hand-chosen position; the expected value of head (l, h) is the
    value planted there, written out by hand, and a pure-Python triple loop over
    (l, h, j) agrees."""
    L, H, n_c = 3, 2, 5
    planted = {(0, 0, 4): 0.91, (0, 1, 0): 0.62, (1, 0, 2): 0.97,
               (1, 1, 1): 0.55, (2, 0, 0): 0.88, (2, 1, 3): 0.73}
    S = _planted_scores(L, H, n_c, planted, seed=72)
    want = [[0.91, 0.62], [0.97, 0.55], [0.88, 0.73]]
    loop = [[max(S[l][h][j] for j in range(n_c)) for h in range(H)] for l in range(L)]
    assert loop == want
    got = o.head_scores(np.array(S), L, H)
    assert np.shape(got) == (L, H), np.shape(got)
    for l in range(L):
        for h in range(H):
            assert float(got[l][h]) == want[l][h], (l, h, got[l][h])


def pin_token_scores(o):
    """Token-level scores (blog post section 4.3.3: one score per position, the
    maximum over all layers and heads).  Each position's maximum is planted in
    a different (layer, head), including heads other than the first and layers
    other than the first, so a maximum over layers only or over heads only
    misses some of them.  Input as [L, H, n_c] and as [L*H, n_c]."""
    L, H, n_c = 3, 2, 6
    planted = {(2, 1, 0): 0.93, (0, 1, 1): 0.81, (1, 0, 2): 0.77,
               (0, 0, 3): 0.99, (2, 0, 4): 0.66, (1, 1, 5): 0.58}
    S = _planted_scores(L, H, n_c, planted, seed=73)
    want = [0.93, 0.81, 0.77, 0.99, 0.66, 0.58]
    loop = [max(S[l][h][j] for l in range(L) for h in range(H)) for j in range(n_c)]
    assert loop == want
    for arr in (np.array(S), np.array(S).reshape(L * H, n_c)):
        got = o.token_scores(arr)
        assert np.shape(got) == (n_c,), np.shape(got)
        assert [float(x) for x in got] == want


def pin_expand_keep(o):
    """A position mask shared by all heads (token-level eviction, blog post
    section 4.3.3) becomes one identical row per head, and head h's packed rows
    start after h full copies of the kept positions.  Checked by loops against
    hand-written expectations."""
    n_heads, n_c = 4, 7
    kp = [0, 1, 0, 0, 1, 1, 0]                       # kept positions 1, 4, 5
    keep, off = o.expand_keep(np.array(kp, np.uint8), n_heads)
    keep = np.asarray(keep).reshape(-1)
    assert keep.size == n_heads * n_c
    for h in range(n_heads):
        for j in range(n_c):
            assert int(keep[h * n_c + j]) == kp[j], (h, j)
    assert [int(x) for x in off] == [0, 3, 6, 9, 12]


SCORING_PINS = [pin_row_sums_and_range, pin_uniform_queries, pin_logistic, pin_dominant_key,
                pin_bruteforce_unchunked, pin_invariants, pin_rows_see_own_prefix]
SELECT_PINS = [pin_keep_count, pin_select_properties, pin_select_bruteforce, pin_select_signed_zero_and_inf]
COMPACT_PINS = [pin_compact, pin_kv_size_table]
DECODE_PINS = [pin_decode_closed_forms, pin_decode_matches_dense_over_kept]
VARIANT_PINS = [pin_sum_aggregation, pin_uniform_budgets, pin_head_scores, pin_token_scores,
                pin_expand_keep]
ALL_PINS = SCORING_PINS + SELECT_PINS + COMPACT_PINS + DECODE_PINS + VARIANT_PINS
