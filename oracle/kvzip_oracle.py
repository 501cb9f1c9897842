"""Plain float64 CPU oracle of KVzip's importance scoring, global top-r
selection and per-head compaction.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.

Sources (web pages on "KVzip: Query-Agnostic KV Cache Compression with Context
Reconstruction", Kim et al.):

* blog post (jjl357.github.io), section 4.1 "Method Overview": prefill gives
  K_c, V_c in R^{n_c x d}; the model is then run on "repeat prompt + context".
* same post, section 4.3.1 "Reconstruction Attention": for layer l and head h,
  queries Q_{l,h} in R^{G x n_in x d} attend to the cached context keys,
  A = Softmax(Q K^T) (the post prints no 1/sqrt(d); standard scaled attention
  is used, with the scale as a parameter).
* same post, section 4.3.2 "Importance Score": S_{l,h}[j] = max over g, i of
  A_{l,h}[g, i, j].
* same post, section 4.5 "Chunked Scoring" and the rebuttal's answer on
  position IDs (paperhub.cn OpenReview rebuttal, first question): the context
  is reconstructed chunk by chunk and chunk scores are merged; each chunk's
  reconstruction continues after the prefilled tokens.
* rebuttal, answer on FLOPs ("2x attention FLOPs relative to prefilling"):
  every chunk attends the whole prefilled context plus its own causal keys.
* rebuttal, answer on head-level scores: S has shape L x H x n_c.
* scime.ai summary, "Approach" and the "Measured effects" table row on
  non-uniform head budgets: evict the lowest-scoring pairs once per context,
  ranked globally over (layer, head, position).

Readings taken where the pages are silent or garbled (each is listed in the
design notes):

1. scale = 1/sqrt(d) unless given.
2. G is the GQA group size: query rows of one KV head are (g, i) pairs,
   row index rho = g * n_in + i.
3. A chunk's row i (prompt or context row) sees all n_c prefilled keys and its
   own chunk's keys 0..i (causal, diagonal included); never another chunk's.
4. Prompt rows take part in the softmax and in the max; only the n_c context
   keys are scored, the chunk's own keys never are.
5. The softmax normaliser includes the causal self keys.
6. Across chunks, S is the running max starting from 0.
7. k = ceil(r * N) computed in IEEE double; among equal scores the lower flat
   index f = (l * H + h) * n_c + j is kept first.
8. Compacted caches are packed head-major, positions ascending in each head.
9. Decoding over a compressed cache attends each query head to its KV head's
   kept rows only (standard softmax attention, scale 1/sqrt(d)); a head with
   no kept rows returns zeros.
10. Sum aggregation (the rebuttal's average-aggregation ablation; sum and
    average rank pairs identically) adds each chunk's column sums of the same
    softmax instead of taking maxima.
11. Uniform head budgets give every head the same k_h = ceil(r * n_c) pairs,
    ranked inside the head with the same tie rule.

Everything is float64 on inputs converted exactly from their storage type
(bf16 and fp32 values are exactly representable in float64).
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def causal_self_mask(G: int, n_in: int) -> np.ndarray:
    """Boolean [G*n_in, n_in]: row rho=(g,i) may see self key j' iff j' <= i.

    Reading 3 (blog post section 4.5 with the rebuttal's FLOP statement): the
    teacher-forced chunk is decoded causally, so token i attends its own
    chunk's keys 0..i.
    """
    i = np.tile(np.arange(n_in), G)            # row -> position inside the chunk
    jp = np.arange(n_in)
    return jp[None, :] <= i[:, None]


def chunk_logits(q, k_ctx, k_self, scale: float) -> np.ndarray:
    """Scaled logits of one (layer, head) unit for one chunk.

    q: [G, n_in, d], k_ctx: [n_c, d], k_self: [n_in, d].
    Returns [G*n_in, n_c + n_in]: columns 0..n_c-1 are the context keys,
    columns n_c.. are the chunk's own keys with the causal mask applied (-inf).
    (Blog post section 4.3.1: A = Softmax(Q K^T), Q in R^{G x n_in x d}.)
    """
    q = _f64(q)
    G, n_in, d = q.shape
    rows = q.reshape(G * n_in, d)
    a_ctx = scale * (rows @ _f64(k_ctx).T)
    a_self = scale * (rows @ _f64(k_self).T)
    a_self[~causal_self_mask(G, n_in)] = -np.inf
    return np.concatenate([a_ctx, a_self], axis=1)


def softmax_rows(a: np.ndarray) -> np.ndarray:
    """Row softmax with max subtraction (rows always hold a finite entry)."""
    m = a.max(axis=1, keepdims=True)
    e = np.exp(a - m)
    return e / e.sum(axis=1, keepdims=True)


def unit_chunk_scores(q, k_ctx, k_self, scale: float | None = None):
    """Chunk scores of one unit: S_c[j] = max over rows of softmax[row, j], j < n_c.

    Returns (S_c [n_c], lse [G*n_in]) where lse is the natural-log normaliser
    of each row (log of the sum of exp over context and visible self keys).
    (Blog post section 4.3.2: S[j] = max_{g,i} A[g,i,j].)
    """
    k_ctx = _f64(k_ctx)
    n_c, d = k_ctx.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    a = chunk_logits(q, k_ctx, k_self, scale)
    m = a.max(axis=1)
    lse = m + np.log(np.exp(a - m[:, None]).sum(axis=1))
    p = softmax_rows(a)
    return p[:, :n_c].max(axis=0), lse


def score_chunk(q, k_ctx, k_self, scores, scale: float | None = None):
    """One chunk for a batch of units, merged into ``scores`` by a running max.

    q: [B, G, n_in, d]; k_ctx: [B, n_c, d]; k_self: [B, n_in, d];
    scores: [B, n_c] float64, updated in place and returned.
    (Blog post section 4.5: chunk scores are merged across chunks.)
    """
    B = len(q)
    for b in range(B):
        s_c, _ = unit_chunk_scores(q[b], k_ctx[b], k_self[b], scale)
        np.maximum(scores[b], s_c, out=scores[b])
    return scores


def score_context(q_chunks, k_self_chunks, k_ctx, scale: float | None = None):
    """Full context scoring: S = max over chunks of the chunk scores, from 0.

    q_chunks[c]: [B, G, n_in_c, d]; k_self_chunks[c]: [B, n_in_c, d]; k_ctx: [B, n_c, d].
    Returns S: [B, n_c] float64 (B = L*H units, flat order l*H + h).
    """
    k_ctx = _f64(k_ctx)
    S = np.zeros(k_ctx.shape[:2], dtype=np.float64)
    for q, ks in zip(q_chunks, k_self_chunks):
        score_chunk(q, k_ctx, ks, S, scale)
    return S


def keep_count(r: float, N: int) -> int:
    """k = ceil(r * N), the product taken in IEEE double (reading 7)."""
    if not (0.0 <= r <= 1.0):
        raise ValueError("r must lie in [0, 1]")
    return int(math.ceil(float(r) * float(N)))


def select(scores, k: int, n_heads: int):
    """Global top-k over all (layer, head, position) scores.

    scores: flat [N] (any float type; compared as given), N = n_heads * n_c.
    Keeps the k highest scores; among equal scores the lower flat index wins
    (reading 7).  Per-head counts are whatever the global ranking leaves in
    each head, i.e. non-uniform head budgets (scime.ai summary, "Measured
    effects" table: uniform head budgets hurt).

    Returns (keep uint8 [N], offsets int64 [n_heads+1], threshold) where
    threshold is the k-th largest score (+inf when k == 0).
    """
    s = np.asarray(scores).reshape(-1)
    N = s.size
    if N % n_heads:
        raise ValueError("N must be a multiple of n_heads")
    if not (0 <= k <= N):
        raise ValueError("k must lie in [0, N]")
    idx = np.arange(N)
    order = np.lexsort((idx, -s.astype(np.float64)))   # score descending, then index ascending
    keep = np.zeros(N, dtype=np.uint8)
    keep[order[:k]] = 1
    cnt = keep.reshape(n_heads, -1).sum(axis=1, dtype=np.int64)
    offsets = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)
    threshold = float(s[order[k - 1]]) if k > 0 else math.inf
    return keep, offsets, threshold


def compact(k, v, keep, offsets):
    """Per-head stream compaction of the kept rows (blog post section 4.1, step 5).

    k, v: [n_heads, n_c, d] (any dtype; rows copied unchanged);
    keep: [n_heads * n_c]; offsets: [n_heads+1].
    Returns (k_out [total, d], v_out [total, d], pos int32 [total]) packed head-major,
    positions ascending inside each head (reading 8).
    """
    k = np.asarray(k)
    v = np.asarray(v)
    n_heads, n_c, d = k.shape
    keep = np.asarray(keep).reshape(n_heads, n_c)
    total = int(offsets[-1])
    k_out = np.zeros((total, d), dtype=k.dtype)
    v_out = np.zeros((total, d), dtype=v.dtype)
    pos = np.zeros(total, dtype=np.int32)
    for h in range(n_heads):
        js = np.nonzero(keep[h])[0]                 # kept positions, ascending
        o = int(offsets[h])
        assert o + js.size == int(offsets[h + 1])
        k_out[o:o + js.size] = k[h, js]
        v_out[o:o + js.size] = v[h, js]
        pos[o:o + js.size] = js
    return k_out, v_out, pos


def head_scores(S, L: int, H: int) -> np.ndarray:
    """Head-level score max_j S[l, h, j] (rebuttal, answer on how head-level
    scores for the DuoAttention comparison were computed)."""
    return _f64(S).reshape(L, H, -1).max(axis=2)


def decode_attention(q, k_packed, v_packed, offsets, scale: float | None = None):
    """One decoding step of attention over the compressed, per-head variable-length
    cache (rebuttal, computational-efficiency table: decoding attention over the
    cache kept at each ratio).

    q: [n_heads, G, d] (the G query heads of each KV head); k_packed, v_packed:
    [total, d] packed head-major; offsets: [n_heads+1].
    Returns o [n_heads, G, d] float64: o[h, g] = softmax(scale * K_h q_g) @ V_h over
    head h's kept rows (reading 9: zeros for an empty head).
    """
    q = _f64(q)
    K = _f64(k_packed)
    V = _f64(v_packed)
    n_heads, G, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((n_heads, G, d))
    for h in range(n_heads):
        a, b = int(offsets[h]), int(offsets[h + 1])
        if b == a:
            continue
        logits = scale * (q[h] @ K[a:b].T)                 # [G, n_h]
        out[h] = softmax_rows(logits) @ V[a:b]
    return out


def unit_chunk_colsums(q, k_ctx, k_self, scale: float | None = None):
    """Sum aggregation for one unit and chunk: sum over rows of softmax[row, j], j < n_c
    (rebuttal, answer on sum/average aggregation; reading 10)."""
    k_ctx = _f64(k_ctx)
    n_c, d = k_ctx.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    p = softmax_rows(chunk_logits(q, k_ctx, k_self, scale))
    return p[:, :n_c].sum(axis=0)


def score_chunk_sum(q, k_ctx, k_self, scores, scale: float | None = None):
    """Sum-aggregation counterpart of score_chunk: scores += chunk column sums."""
    for b in range(len(q)):
        scores[b] += unit_chunk_colsums(q[b], k_ctx[b], k_self[b], scale)
    return scores


def token_scores(S):
    """Token-level importance S[j] = max over (layer, head) of S[l, h, j]
    (blog post section 4.3.3): one score per position, shared by all heads."""
    return _f64(S).reshape(-1, np.asarray(S).shape[-1]).max(axis=0)


def select_per_head(scores, k_h: int, n_heads: int):
    """Uniform head budgets (reading 11): the k_h highest scores inside every
    head, lower position first among equal scores.  Returns (keep, offsets)."""
    s = np.asarray(scores).reshape(n_heads, -1)
    n_c = s.shape[1]
    if not (0 <= k_h <= n_c):
        raise ValueError("k_h must lie in [0, n_c]")
    keep = np.zeros_like(s, dtype=np.uint8)
    for h in range(n_heads):
        order = np.lexsort((np.arange(n_c), -s[h].astype(np.float64)))
        keep[h, order[:k_h]] = 1
    offsets = np.arange(n_heads + 1, dtype=np.int64) * k_h
    return keep.reshape(-1), offsets


def expand_keep(keep_pos, n_heads: int):
    """A position mask shared by all heads, as a per-head mask and offsets."""
    kp = np.asarray(keep_pos).astype(np.uint8).reshape(-1)
    keep = np.tile(kp, n_heads)
    offsets = np.arange(n_heads + 1, dtype=np.int64) * int(kp.sum())
    return keep, offsets
