"""Global top-r selection when one context's heads are split across ranks.

KVzip ranks all L x H x n_c scores of a context together, which is what gives
non-uniform head budgets (rebuttal: S has shape L x H x n_c; scime.ai summary,
"Measured effects").  In tensor-parallel serving every GPU holds a run of KV
heads, so scoring and compaction stay local and only the selection needs an
exchange.  ``select_sharded`` drives libkvzip's sharded selection calls
(kvzip_select_shard_*) and does that exchange with ``torch.distributed``:

* three radix rounds, each one all-reduce (sum) of a 64-bit histogram of
  8192, 1024 and 512 bins (64, 8 and 4 KB);
* one all-gather of every rank's count of scores equal to the threshold, so
  that ties keep the lowest flat indices of the whole context.

Every rank takes the same collective steps in the same order.  Rank r must
hold the r-th run of heads (ranks in flat-index order).  The result on each
rank is its part of what ``kvzip_select`` gives on the concatenated scores.

On an NCCL group the histograms stay on the device; on a gloo group they are
copied to the host for the exchange and back.  All arithmetic runs in the
library's kernels (``backend`` is the ctypes binding; tests may pass a stand-in
with the same functions to exercise the exchange without a GPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def select_sharded(scores_local: torch.Tensor, k: int, group=None, backend=None,
                   workspace: torch.Tensor | None = None, keep: torch.Tensor | None = None,
                   offsets: torch.Tensor | None = None, threshold: torch.Tensor | None = None,
                   stream=None, round1_hist: torch.Tensor | None = None):
    """Keep the k largest scores of the whole context (k is the GLOBAL count).

    scores_local: this rank's scores [n_heads_local][n_c] float32.
    round1_hist: optionally, the round-1 histogram of exactly these scores
    (SCORE_HIST_BINS counts, as the last chunk's kvzip_score_colmax_hist leaves
    it); it replaces this rank's first histogram pass.  Like the histograms
    the ranks exchange, it is trusted as given.
    Returns (keep uint8 [n_heads_local * n_c], offsets int64 [n_heads_local + 1]
    over this rank's heads, threshold float32 [1] = the k-th largest score of
    the whole context, +inf when k == 0).
    """
    if backend is None:
        from . import kvzip as backend
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    on_host = dist.get_backend(group) == "gloo"
    n_heads_local, n_c = scores_local.shape
    flat = scores_local.reshape(-1)
    dev = flat.device
    if workspace is None:
        workspace = backend.shard_workspace(flat.numel(), n_heads_local, dev)
    if keep is None:
        keep = torch.empty(flat.numel(), dtype=torch.uint8, device=dev)
    if offsets is None:
        offsets = torch.empty(n_heads_local + 1, dtype=torch.int64, device=dev)
    if threshold is None:
        threshold = torch.full((1,), float("inf"), dtype=torch.float32, device=dev)

    backend.shard_begin(k, workspace, stream)
    for r in range(3):
        if r == 0 and round1_hist is not None:
            if round1_hist.numel() != backend.shard_bins(0):
                raise ValueError("round1_hist must hold shard_bins(0) counts")
            # a copy (also when it is int64 already): the all-reduce works in place
            hist = round1_hist.to(torch.int64, copy=True)
        else:
            hist = torch.empty(backend.shard_bins(r), dtype=torch.int64, device=dev)
            backend.shard_hist(flat, r, hist, workspace, stream)
        _all_reduce_sum(hist, group, on_host)
        backend.shard_pick(hist, r, threshold, workspace, stream)
    n_ties = torch.empty(1, dtype=torch.int64, device=dev)
    backend.shard_ties(flat, n_ties, workspace, stream)
    tie_counts = _all_gather_one(n_ties, world, group, on_host)
    backend.shard_mask(flat, n_heads_local, tie_counts, rank, keep, offsets, workspace, stream)
    return keep, offsets, threshold


def _all_reduce_sum(t: torch.Tensor, group, on_host: bool):
    if on_host and t.device.type != "cpu":
        h = t.cpu()
        dist.all_reduce(h, op=dist.ReduceOp.SUM, group=group)
        t.copy_(h)
    else:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def _all_gather_one(t: torch.Tensor, world: int, group, on_host: bool) -> torch.Tensor:
    src = t.cpu() if (on_host and t.device.type != "cpu") else t
    parts = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(parts, src, group=group)
    return torch.cat(parts).to(t.device)
