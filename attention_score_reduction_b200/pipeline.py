"""End-to-end KVzip compression of one context: chunked scoring, global top-r
selection and per-head compaction, through libkvzip.

This is the user-facing call.  ``Compressor`` owns the device buffers for one
context shape and runs the three C-ABI calls on a CUDA stream:

  1. ``kvzip_score_context`` (all chunks but the last) or ``kvzip_score_chunk``
     once per reconstruction chunk (blog post section 4.5: chunked scoring
     keeps memory linear in n_c), merging into the L x H x n_c score tensor by
     a running max.  The last chunk's column-max half is
     ``kvzip_score_colmax_hist``: it also counts the final scores in the
     selection's round-1 histogram;
  2. ``kvzip_select_hist`` once per context (scime.ai summary, "Approach":
     evict the lowest-scoring pairs once, query-agnostically), global over
     (l, h, j), reading the scores once; with several ranks, the sharded
     selection;
  3. ``kvzip_compact`` once, packing the kept K/V rows per head.

``compress_from_host`` is the same path for inputs that start in (pinned)
host memory: the context K/V and each chunk's Q / K_self are uploaded on a
copy stream that runs ahead of the scorer, and the compacted cache is read
back.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import kvzip as kz


@dataclass
class Compressed:
    k: torch.Tensor          # [kept][d]   packed head-major, positions ascending per head
    v: torch.Tensor          # [kept][d]
    pos: torch.Tensor        # [kept] int32 positions within the head
    offsets: torch.Tensor    # [units + 1] int64; head h owns rows offsets[h]:offsets[h+1]
    kept: int                # = offsets[-1]
    threshold: torch.Tensor  # [1] float32, the kept-th largest score


class Compressor:
    """Device state for compressing contexts of one shape.

    units = L * H (layer-major), n_c context keys per unit, head dim d, G
    query heads per KV head, max_n_in = largest chunk (prompt + context rows).

    With a process group (``group``), this rank holds ``units`` of the
    context's ``units_global`` units, ranks in flat-index order; scoring and
    compaction stay local and the selection ranks all units_global * n_c scores
    together through ``sharded.select_sharded``.
    """

    def __init__(self, units: int, n_c: int, d: int, G: int, max_n_in: int, device="cuda",
                 group=None, units_global: int | None = None):
        self.units, self.n_c, self.d, self.G, self.max_n_in = units, n_c, d, G, max_n_in
        self.device = torch.device(device)
        self.group = group
        self.units_global = units_global or units
        N = units * n_c
        self.scores = torch.zeros(units, n_c, dtype=torch.float32, device=self.device)
        self.score_ws = kz.new_context_workspace(units, G, max_n_in, self.device)
        if group is None:
            self.select_ws = torch.zeros(max(kz.select_workspace_size(N, units), 256),
                                         dtype=torch.uint8, device=self.device)
        else:
            self.select_ws = kz.shard_workspace(N, units, self.device)
        self.compact_ws = torch.empty(max(kz.compact_workspace_size(units, n_c), 256),
                                      dtype=torch.uint8, device=self.device)
        self.keep = torch.empty(N, dtype=torch.uint8, device=self.device)
        self.offsets = torch.empty(units + 1, dtype=torch.int64, device=self.device)
        self.threshold = torch.empty(1, dtype=torch.float32, device=self.device)
        # round-1 histogram of the final scores, counted by the last chunk's
        # column-max pass: the one-GPU selection then reads the scores once, and
        # a sharded selection skips its first histogram pass
        self.score_hist = kz.new_score_hist(self.device)
        self.hist_ready = False
        self.unit_ws = {}   # (u0, u1) -> workspace of score_units
        self.launches = 0

    def reset(self):
        self.scores.zero_()
        self.score_hist.zero_()
        self.hist_ready = False

    def score_chunk(self, q, k_ctx, k_self, scale: float = 0.0, stream=None, last: bool = False):
        """One chunk; ``last`` (the context's final chunk) also counts the
        final scores in the selection's round-1 histogram."""
        self._score(q, k_ctx, k_self, self.scores, self.score_ws, scale, stream, last)

    def score_units(self, u0: int, u1: int, q, k_ctx, k_self, scale: float = 0.0, stream=None,
                    last: bool = False):
        """One chunk for units [u0, u1) only (q, k_ctx, k_self hold every unit),
        with a workspace of its own for those units' row normalisers."""
        ws = self.unit_ws.get((u0, u1))
        if ws is None:
            ws = self.unit_ws[(u0, u1)] = kz.new_score_workspace(u1 - u0, self.G, self.max_n_in,
                                                                 self.device)
        self._score(q[u0:u1], k_ctx[u0:u1], k_self[u0:u1], self.scores[u0:u1], ws, scale, stream,
                    last)

    def _score(self, q, k_ctx, k_self, scores, ws, scale, stream, last):
        if last:
            kz.score_chunk(q, k_ctx, k_self, scores, ws, scale, stream, "lse")
            self.launches += kz.last_launch_count()
            kz.score_chunk(q, k_ctx, k_self, scores, ws, scale, stream, "colmax",
                           hist=self.score_hist)
            self.hist_ready = True
        else:
            kz.score_chunk(q, k_ctx, k_self, scores, ws, scale, stream)
        self.launches += kz.last_launch_count()

    def keep_capacity(self, r: float) -> int:
        """Rows this rank's compacted cache can need: the kept count itself on
        one GPU; with shards, at most the global count and at most its scores."""
        k = kz.keep_count(r, self.units_global * self.n_c)
        return k if self.group is None else min(k, self.scores.numel())

    def select(self, r: float, stream=None) -> int:
        """Global top-r selection; returns the kept count (global on one GPU,
        this rank's capacity bound with shards: offsets[-1] holds its count)."""
        if self.group is None:
            kept = kz.keep_count(r, self.scores.numel())
            kz.select(self.scores.view(-1), kept, self.units, self.keep, self.offsets,
                      self.threshold, self.select_ws, stream,
                      hist=self.score_hist if self.hist_ready else None)
            self.launches += kz.last_launch_count()
            return kept
        from . import sharded
        k = kz.keep_count(r, self.units_global * self.n_c)
        given = self.score_hist if self.hist_ready else None
        sharded.select_sharded(self.scores, k, self.group, workspace=self.select_ws,
                               keep=self.keep, offsets=self.offsets, threshold=self.threshold,
                               stream=stream, round1_hist=given)
        # begin, 3 x (histogram, pick), tie count, five-kernel mask; one histogram fewer if given
        self.launches += 13 if given is None else 12
        return self.keep_capacity(r)

    def compact(self, k_ctx, v, kept: int, k_out=None, v_out=None, pos_out=None, stream=None):
        out = kz.compact(k_ctx, v, self.keep, self.offsets, kept, k_out, v_out, pos_out,
                         workspace=self.compact_ws, stream=stream)
        self.launches += kz.last_launch_count()
        return out

    def compress(self, k_ctx, v, chunks, r: float, scale: float = 0.0, stream=None,
                 out=None) -> Compressed:
        """k_ctx, v: [units][n_c][d] bf16 on the device; chunks: iterable of
        (q [units][G][n_in][d], k_self [units][n_in][d]) device tensors."""
        self.reset()
        chunks = list(chunks)
        if len(chunks) > 1:
            kz.score_context(chunks[:-1], k_ctx, self.scores, self.score_ws, scale, stream)
            self.launches += kz.last_launch_count()
        if chunks:
            q_last, ks_last = chunks[-1]
            self.score_chunk(q_last, k_ctx, ks_last, scale=scale, stream=stream, last=True)
        kept = self.select(r, stream)
        k_out, v_out, pos = self.compact(k_ctx, v, kept, *(out or (None, None, None)),
                                         stream=stream)
        return Compressed(k_out, v_out, pos, self.offsets, kept, self.threshold)

    def check_status(self, stream=None):
        for ws in [self.score_ws] + list(self.unit_ws.values()):
            s = kz.workspace_status(ws, stream)
            if s != kz.OK:
                raise kz.KvzipError(s, "scoring kernels")
        if self.group is None:
            s = kz.workspace_status(self.select_ws, stream)
            if s != kz.OK:
                raise kz.KvzipError(s, "selection kernel")


def compress_from_host(comp: Compressor, k_ctx_h, v_h, q_chunks_h, ks_chunks_h, r: float,
                       dev_bufs: dict, host_out: dict | None = None, scale: float = 0.0,
                       key_slices: int = 4):
    """Upload host inputs, compress, and read the compacted cache back.

    k_ctx_h, v_h: pinned host [units][n_c][d]; q_chunks_h / ks_chunks_h: lists of
    pinned host chunk tensors (one per chunk, in order).  ``dev_bufs`` holds
    reusable device tensors: "k_ctx", "v", and lists "q", "ks" of chunk buffers.
    When the lists are shorter than the chunk list they are used as a ring:
    chunk c goes into buffer c % len, and its upload waits until the scorer has
    finished the chunk that last used that buffer.  ``host_out`` (pinned)
    receives "k", "v", "pos", "offsets".  Uploads run on a side stream in the
    order the scorer needs them, each recorded by an event the scorer waits on:
    the first chunk's inputs, then the context keys in ``key_slices`` runs of
    units (the first chunk is scored run by run as its keys arrive), then each
    later chunk's inputs followed by a piece of V, which only compaction needs.
    Returns (Compressed on the device, host_out, bytes_h2d, bytes_d2h).
    """
    main = torch.cuda.current_stream()
    copy = dev_bufs.setdefault("_copy_stream", torch.cuda.Stream())
    n_buf = len(dev_bufs["q"])
    n_chunks = len(q_chunks_h)
    if n_buf == 0 or len(dev_bufs["ks"]) != n_buf or n_chunks != len(ks_chunks_h):
        raise ValueError("need matching lists of chunk inputs and device chunk buffers")
    units = comp.units
    n_sl = max(1, min(key_slices, units)) if n_chunks else 1
    k_runs = [(units * i // n_sl, units * (i + 1) // n_sl) for i in range(n_sl)]
    n_vp = max(1, min(units, n_chunks - 1))           # V pieces, one behind each later chunk
    v_runs = [(units * i // n_vp, units * (i + 1) // n_vp) for i in range(n_vp)]
    copy.wait_stream(main)          # device buffers are free once earlier work is done
    comp.reset()
    h2d = 0
    ev_v = []

    def upload(dst, src_h):
        nonlocal h2d
        dst.copy_(src_h, non_blocking=True)
        h2d += src_h.numel() * src_h.element_size()

    def upload_v(p):
        a, b = v_runs[p]
        with torch.cuda.stream(copy):
            upload(dev_bufs["v"][a:b], v_h[a:b])
            ev = torch.cuda.Event()
            ev.record(copy)
        ev_v.append(ev)

    freed = [None] * n_buf          # event: the scorer is done with this ring slot
    for c, (qh, ksh) in enumerate(zip(q_chunks_h, ks_chunks_h)):
        slot = c % n_buf
        qd, ksd = dev_bufs["q"][slot], dev_bufs["ks"][slot]
        if qd.shape != qh.shape or ksd.shape != ksh.shape:   # a ragged last chunk
            qd = qd.view(-1)[:qh.numel()].view(qh.shape)
            ksd = ksd.view(-1)[:ksh.numel()].view(ksh.shape)
        with torch.cuda.stream(copy):
            if freed[slot] is not None:
                copy.wait_event(freed[slot])
            upload(qd, qh)
            upload(ksd, ksh)
            up = torch.cuda.Event()
            up.record(copy)
        last = c == n_chunks - 1
        if c == 0:                  # the keys, run by run, each scored as it lands
            ev_k = []
            with torch.cuda.stream(copy):
                for a, b in k_runs:
                    upload(dev_bufs["k_ctx"][a:b], k_ctx_h[a:b])
                    ev = torch.cuda.Event()
                    ev.record(copy)
                    ev_k.append(ev)
            main.wait_event(up)
            for (a, b), ev in zip(k_runs, ev_k):
                main.wait_event(ev)
                if n_sl == 1:
                    comp.score_chunk(qd, dev_bufs["k_ctx"], ksd, scale, last=last)
                else:
                    comp.score_units(a, b, qd, dev_bufs["k_ctx"], ksd, scale, last=last)
        else:
            main.wait_event(up)
            comp.score_chunk(qd, dev_bufs["k_ctx"], ksd, scale, last=last)
            if c - 1 < n_vp:
                upload_v(c - 1)
        done = torch.cuda.Event()
        done.record(main)
        freed[slot] = done
    if n_chunks <= 1:
        if not n_chunks:            # no chunks: the keys still go up for compaction
            with torch.cuda.stream(copy):
                upload(dev_bufs["k_ctx"], k_ctx_h)
        upload_v(0)
    for ev in ev_v:
        main.wait_event(ev)
    kept = comp.select(r)
    if comp.group is not None:    # this rank's share of the global count (one small read)
        kept = int(comp.offsets[-1])
    k_out, v_out, pos = comp.compact(dev_bufs["k_ctx"], dev_bufs["v"], kept)
    d2h = 0
    if host_out is not None:
        host_out["k"][:kept].copy_(k_out, non_blocking=True)
        host_out["v"][:kept].copy_(v_out, non_blocking=True)
        host_out["pos"][:kept].copy_(pos, non_blocking=True)
        host_out["offsets"].copy_(comp.offsets, non_blocking=True)
        d2h = (k_out.numel() * 2 + v_out.numel() * 2 + pos.numel() * 4 + comp.offsets.numel() * 8)
    return Compressed(k_out, v_out, pos, comp.offsets, kept, comp.threshold), host_out, h2d, d2h
