"""The CPU oracle against its pins, and planted mistakes against the same pins.

A planted mistake lives in a private copy of the oracle module loaded for the
test; the real oracle is never modified.
"""
import importlib.util
import math
import os

import numpy as np
import pytest

import oracle
from tests import oracle_pins as P

ORACLE_FILE = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "kvzip_oracle.py")


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle)


def _fresh_copy():
    spec = importlib.util.spec_from_file_location("kvzip_oracle_mutant", ORACLE_FILE)
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _mut_drop_diagonal(m):
    def mask(G, n_in):
        i = np.tile(np.arange(n_in), G)
        return np.arange(n_in)[None, :] < i[:, None]
    m.causal_self_mask = mask


def _mut_anticausal(m):
    def mask(G, n_in):
        i = np.tile(np.arange(n_in), G)
        return np.arange(n_in)[None, :] >= i[:, None]
    m.causal_self_mask = mask


def _mut_row_order(m):
    # rows taken i-major instead of g-major: the row -> position map is wrong
    def mask(G, n_in):
        i = np.repeat(np.arange(n_in), G)
        return np.arange(n_in)[None, :] <= i[:, None]
    m.causal_self_mask = mask


def _mut_no_self_in_normaliser(m):
    orig = m.chunk_logits

    def logits(q, k_ctx, k_self, scale):
        a = orig(q, k_ctx, k_self, scale)
        a[:, k_ctx.shape[0]:] = -np.inf
        return a
    m.chunk_logits = logits


def _mut_no_scale(m):
    orig = m.chunk_logits
    m.chunk_logits = lambda q, k, ks, scale: orig(q, k, ks, 1.0)


def _mut_mean(m):
    def ucs(q, k_ctx, k_self, scale=None):
        k_ctx = np.asarray(k_ctx, np.float64)
        if scale is None:
            scale = 1 / math.sqrt(k_ctx.shape[1])
        a = m.chunk_logits(q, k_ctx, k_self, scale)
        p = m.softmax_rows(a)
        mx = a.max(axis=1)
        return p[:, :k_ctx.shape[0]].mean(axis=0), mx + np.log(np.exp(a - mx[:, None]).sum(1))
    m.unit_chunk_scores = ucs


def _mut_sum_over_chunks(m):
    def score_chunk(q, k_ctx, k_self, scores, scale=None):
        for b in range(len(q)):
            s_c, _ = m.unit_chunk_scores(q[b], k_ctx[b], k_self[b], scale)
            scores[b] += s_c
        return scores
    m.score_chunk = score_chunk


def _mut_transposed_keys(m):
    orig = m.chunk_logits

    def logits(q, k_ctx, k_self, scale):
        q = np.asarray(q, np.float64)
        # uses the self keys of the wrong end of the chunk (reversed order)
        return orig(q, k_ctx, np.asarray(k_self)[::-1], scale)
    m.chunk_logits = logits


def _mut_floor_count(m):
    m.keep_count = lambda r, N: int(math.floor(r * N))


def _mut_tie_high_index(m):
    orig = m.select

    def select(scores, k, n_heads):
        s = np.asarray(scores).reshape(-1)
        N = s.size
        order = np.lexsort((-np.arange(N), -s.astype(np.float64)))
        keep = np.zeros(N, np.uint8)
        keep[order[:k]] = 1
        cnt = keep.reshape(n_heads, -1).sum(1)
        off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)
        return keep, off, (float(s[order[k - 1]]) if k else math.inf)
    m.select = select


def _mut_uniform_head_budget(m):
    def select(scores, k, n_heads):
        s = np.asarray(scores).reshape(n_heads, -1)
        keep = np.zeros_like(s, dtype=np.uint8)
        per = k // n_heads
        for h in range(n_heads):
            keep[h, np.argsort(-s[h], kind="stable")[:per]] = 1
        keep = keep.reshape(-1)
        cnt = keep.reshape(n_heads, -1).sum(1)
        off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)
        kept = s.reshape(-1)[keep == 1]
        return keep, off, (float(kept.min()) if kept.size else math.inf)
    m.select = select


def _mut_positions_descending(m):
    orig = m.compact

    def compact(k, v, keep, offsets):
        ko, vo, pos = orig(k, v, keep, offsets)
        for h in range(len(offsets) - 1):
            a, b = int(offsets[h]), int(offsets[h + 1])
            ko[a:b], vo[a:b], pos[a:b] = ko[a:b][::-1].copy(), vo[a:b][::-1].copy(), pos[a:b][::-1].copy()
        return ko, vo, pos
    m.compact = compact


def _mut_decode_no_scale(m):
    orig = m.decode_attention
    m.decode_attention = lambda q, k, v, off, scale=None: orig(q, k, v, off, 1.0)


def _mut_decode_wrong_head(m):
    orig = m.decode_attention

    def dec(q, k, v, off, scale=None):
        q = np.asarray(q)
        return orig(q[::-1].copy(), k, v, off, scale)[::-1].copy()
    m.decode_attention = dec


def _mut_sum_without_self(m):
    def colsums(q, k_ctx, k_self, scale=None):
        k_ctx = np.asarray(k_ctx, np.float64)
        if scale is None:
            scale = 1 / math.sqrt(k_ctx.shape[1])
        a = m.chunk_logits(q, k_ctx, k_self, scale)[:, :k_ctx.shape[0]]
        return m.softmax_rows(a).sum(axis=0)
    m.unit_chunk_colsums = colsums


def _mut_per_head_tie_high(m):
    def sph(scores, k_h, n_heads):
        s = np.asarray(scores).reshape(n_heads, -1)
        n_c = s.shape[1]
        keep = np.zeros_like(s, dtype=np.uint8)
        for h in range(n_heads):
            order = np.lexsort((-np.arange(n_c), -s[h].astype(np.float64)))
            keep[h, order[:k_h]] = 1
        return keep.reshape(-1), np.arange(n_heads + 1, dtype=np.int64) * k_h
    m.select_per_head = sph


def _mut_head_scores_wrong_axis(m):
    # maximum over the heads of a layer instead of over the positions of a head
    m.head_scores = lambda S, L, H: np.asarray(S, np.float64).reshape(L, H, -1).max(axis=1)


def _mut_head_scores_heads_major(m):
    # units read as head-major (h * L + l) instead of layer-major (l * H + h)
    m.head_scores = lambda S, L, H: np.asarray(S, np.float64).reshape(H, L, -1).max(axis=2).T


def _mut_token_scores_layers_only(m):
    # maximum over the leading axis only: layers, not layers and heads
    m.token_scores = lambda S: np.asarray(S, np.float64).max(axis=0)


def _mut_token_scores_first_head(m):
    # maximum over the layers of the first head of each layer only
    def tok(S):
        S = np.asarray(S, np.float64)
        n_c = S.shape[-1]
        return S.reshape(-1, n_c)[::2].max(axis=0)
    m.token_scores = tok


def _mut_expand_repeat(m):
    # each position repeated n_heads times instead of the whole mask per head
    def expand(keep_pos, n_heads):
        kp = np.asarray(keep_pos).astype(np.uint8).reshape(-1)
        return np.repeat(kp, n_heads), np.arange(n_heads + 1, dtype=np.int64) * int(kp.sum())
    m.expand_keep = expand


def _mut_expand_offsets_by_n_c(m):
    # head h's rows start at h * n_c (the dense layout) instead of h * kept
    def expand(keep_pos, n_heads):
        kp = np.asarray(keep_pos).astype(np.uint8).reshape(-1)
        return np.tile(kp, n_heads), np.arange(n_heads + 1, dtype=np.int64) * kp.size
    m.expand_keep = expand


def _mut_select_raw_bits(m):
    # scores ranked by their raw float bits as unsigned integers: -0.0 (0x80000000)
    # then outranks every score, and any negative value outranks +inf
    orig = m.select

    def select(scores, k, n_heads):
        s = np.asarray(scores, dtype=np.float32).reshape(-1)
        as_rank = s.view(np.uint32).astype(np.float64)
        keep, off, _ = orig(as_rank, k, n_heads)
        thr = float(s[np.nonzero(keep)[0]][np.argmin(as_rank[keep.astype(bool)])]) if k else math.inf
        return keep, off, thr
    m.select = select


MUTANTS = [_mut_drop_diagonal, _mut_anticausal, _mut_row_order, _mut_no_self_in_normaliser,
           _mut_no_scale, _mut_mean, _mut_sum_over_chunks, _mut_transposed_keys,
           _mut_floor_count, _mut_tie_high_index, _mut_uniform_head_budget,
           _mut_positions_descending, _mut_decode_no_scale, _mut_decode_wrong_head,
           _mut_sum_without_self, _mut_per_head_tie_high, _mut_head_scores_wrong_axis,
           _mut_head_scores_heads_major, _mut_token_scores_layers_only,
           _mut_token_scores_first_head, _mut_expand_repeat, _mut_expand_offsets_by_n_c,
           _mut_select_raw_bits]


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__)
def test_planted_mistake_is_caught(mutate):
    m = _fresh_copy()
    mutate(m)
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(m)
        except AssertionError:
            caught.append(pin.__name__)
        except (ValueError, IndexError, ZeroDivisionError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught {mutate.__name__}"
