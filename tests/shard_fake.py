"""A numpy stand-in for libkvzip's five sharded-selection kernels, used to test
the cross-rank exchange in ``attention_score_reduction_b200.sharded`` on CPU
(gloo ranks, no GPU).  It follows the calls' contract in include/kvzip.h: three
radix rounds on the float bits (13, 10 and 9 bits, most significant first),
each histogram counting only the scores that match the bits fixed so far; then
the scores equal to the threshold are ranked in flat order, ties on earlier
ranks first.  Test infrastructure only."""
from __future__ import annotations

import numpy as np
import torch

_BINS = (8192, 1024, 512)
_SHIFT = (19, 9, 0)
_MASK = (0x0, 0xFFF80000, 0xFFFFFE00)


class _State:
    def __init__(self):
        self.prefix = 0
        self.k_rem = 0
        self.none = False
        self.tau = None
        self.take_eq = 0


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.float32).view(np.uint32)


def shard_bins(r):
    return _BINS[r]


def shard_workspace(N_local, n_heads_local, device=None):
    return _State()


def shard_begin(k, ws, stream=None):
    ws.prefix, ws.k_rem, ws.none, ws.tau, ws.take_eq = 0, int(k), k == 0, None, 0


def shard_hist(flat, r, hist, ws, stream=None):
    b = _bits(flat)
    h = np.zeros(_BINS[r], dtype=np.int64)
    if not ws.none:
        m = (b & np.uint32(_MASK[r])) == np.uint32(ws.prefix)
        d = (b[m] >> np.uint32(_SHIFT[r])) & np.uint32(_BINS[r] - 1)
        h = np.bincount(d.astype(np.int64), minlength=_BINS[r]).astype(np.int64)
    hist.copy_(torch.from_numpy(h))


def shard_pick(hist, r, threshold, ws, stream=None):
    if ws.none:
        return
    h = hist.cpu().numpy()
    above = 0
    for bin_ in range(_BINS[r] - 1, -1, -1):
        if above + int(h[bin_]) >= ws.k_rem:
            ws.prefix |= bin_ << _SHIFT[r]
            ws.k_rem -= above
            break
        above += int(h[bin_])
    if r == 2:
        ws.tau = ws.prefix
        ws.take_eq = ws.k_rem
        if threshold is not None:
            threshold.copy_(torch.tensor([ws.tau], dtype=torch.int64).to(torch.int32)
                            .view(torch.float32))


def shard_ties(flat, n_ties, ws, stream=None):
    c = 0 if ws.none else int(np.count_nonzero(_bits(flat) == np.uint32(ws.tau)))
    n_ties.fill_(c)


def shard_mask(flat, n_heads_local, tie_counts, rank, keep, offsets, ws, stream=None):
    b = _bits(flat)
    if ws.none:
        kp = np.zeros(b.size, np.uint8)
    else:
        tc = tie_counts.cpu().numpy()
        quota = max(0, ws.take_eq - int(tc[:rank].sum()))
        eq = b == np.uint32(ws.tau)
        rank_in = np.cumsum(eq) - 1                  # flat-order rank among this rank's ties
        kp = ((b > np.uint32(ws.tau)) | (eq & (rank_in < quota))).astype(np.uint8)
    keep.copy_(torch.from_numpy(kp))
    cnt = kp.reshape(n_heads_local, -1).sum(axis=1)
    offsets.copy_(torch.from_numpy(np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)))
