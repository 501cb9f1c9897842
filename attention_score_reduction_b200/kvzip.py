"""ctypes binding of libkvzip (include/kvzip.h): argument marshalling only.

Every computation runs in the library's CUDA kernels; torch tensors provide
device memory and the stream.  If the library is missing, importing this
module raises: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# KVZIP_LIBRARY selects another build of the same ABI (e.g. libkvzip_debug.so,
# the build with device bounds checks); by default the in-tree libkvzip.so.
LIB_PATH = os.environ.get("KVZIP_LIBRARY") or os.path.join(_HERE, "libkvzip.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = 0, 1, 2, 3, 4, 5
BF16, F32 = 0, 1


class KvzipError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libkvzip.so not found at {LIB_PATH}; build it with "
            "`python -m attention_score_reduction_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, f32, f64, u64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                       ctypes.c_size_t, ctypes.c_float, ctypes.c_double,
                                       ctypes.c_uint64)
    sig = {
        "kvzip_score_workspace_size": (sz, [i32, i32, i32]),
        "kvzip_score_chunk": (i32, [i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, sz, vp]),
        "kvzip_score_lse": (i32, [i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, sz, vp]),
        "kvzip_score_colmax": (i32, [i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, sz, vp]),
        "kvzip_score_colmax_hist": (i32, [i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, vp,
                                          sz, vp]),
        "kvzip_score_context_workspace_size": (sz, [i32, i32, i32]),
        "kvzip_score_context": (i32, [i32, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, vp,
                                      sz, vp]),
        "kvzip_workspace_status": (i32, [vp, vp]),
        "kvzip_score_lse_layout": (i32, [i32, i32, ctypes.POINTER(sz), ctypes.POINTER(i64)]),
        "kvzip_set_wait_timeout_ns": (None, [u64]),
        "kvzip_set_test_stall": (None, [i32]),
        "kvzip_keep_count": (i64, [f64, i64]),
        "kvzip_select_workspace_size": (sz, [i64, i64]),
        "kvzip_select": (i32, [vp, i64, i64, i64, vp, vp, vp, vp, sz, vp]),
        "kvzip_select_hist": (i32, [vp, i64, i64, i64, vp, vp, vp, vp, vp, sz, vp]),
        "kvzip_select_noalloc": (i32, [vp, i64, i64, i64, vp, vp, vp, vp]),
        "kvzip_select_shard_bins": (i32, [i32]),
        "kvzip_select_shard_workspace_size": (sz, [i64, i64]),
        "kvzip_select_shard_begin": (i32, [i64, vp, sz, vp]),
        "kvzip_select_shard_hist": (i32, [vp, i64, i32, vp, vp, sz, vp]),
        "kvzip_select_shard_pick": (i32, [vp, i32, vp, vp, sz, vp]),
        "kvzip_select_shard_ties": (i32, [vp, i64, vp, vp, sz, vp]),
        "kvzip_select_shard_mask": (i32, [vp, i64, i64, vp, i32, vp, vp, vp, sz, vp]),
        "kvzip_compact_workspace_size": (sz, [i64, i32]),
        "kvzip_compact": (i32, [vp, vp, vp, vp, i64, i32, i32, vp, vp, vp, vp, sz, vp]),
        "kvzip_head_scores": (i32, [vp, i64, i64, vp, vp]),
        "kvzip_score_chunk_sum": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, sz, vp]),
        "kvzip_token_scores": (i32, [vp, i64, i64, vp, vp]),
        "kvzip_expand_keep": (i32, [vp, vp, i64, i64, vp, vp, vp]),
        "kvzip_select_per_head_workspace_size": (sz, [i64, i64]),
        "kvzip_select_per_head": (i32, [vp, i64, i64, i64, vp, vp, vp, sz, vp]),
        "kvzip_decode_workspace_size": (sz, [i64, i32, i32]),
        "kvzip_decode_attention": (i32, [vp, vp, vp, i64, vp, i64, i32, i32, f32, vp, vp, sz, vp]),
        "kvzip_last_launch_count": (i32, []),
        "kvzip_debug_checks": (i32, []),
        "kvzip_debug_bounds_status": (i32, []),
        "kvzip_status_string": (ctypes.c_char_p, [i32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def status_string(s: int) -> str:
    return _lib.kvzip_status_string(int(s)).decode()


def _check(s: int, where: str):
    if s != OK:
        raise KvzipError(s, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev_contig(name, t, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


# ---------------------------------------------------------------- scoring

def score_workspace_size(B: int, G: int, n_in: int) -> int:
    return int(_lib.kvzip_score_workspace_size(B, G, n_in))


def new_score_workspace(B: int, G: int, n_in: int, device=None) -> torch.Tensor:
    """Zero-initialised workspace (the status word must start at 0)."""
    n = score_workspace_size(B, G, n_in)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device or "cuda")


SCORE_HIST_BINS = 8192   # KVZIP_SCORE_HIST_BINS


def new_score_hist(device=None) -> torch.Tensor:
    """A zeroed round-1 histogram for score_chunk(..., hist=) / select(..., hist=)."""
    return torch.zeros(SCORE_HIST_BINS, dtype=torch.int32, device=device or "cuda")


def score_chunk(q: torch.Tensor, k_ctx: torch.Tensor, k_self: torch.Tensor, scores: torch.Tensor,
                workspace: torch.Tensor | None = None, scale: float = 0.0, stream=None,
                which: str = "both", hist: torch.Tensor | None = None):
    """scores[b][j] = max(scores[b][j], max_rho softmax(...)[rho][j]) for one chunk.

    q [B][G][n_in][d], k_ctx [B][n_c][d], k_self [B][n_in][d] (bf16 or fp32,
    same dtype), scores [B][n_c] float32.  ``which`` = "both" (kvzip_score_chunk),
    "lse" (kvzip_score_lse) or "colmax" (kvzip_score_colmax).  With ``hist``
    (int32 [SCORE_HIST_BINS], zeroed) the column-max half is
    kvzip_score_colmax_hist: the resulting scores are counted in their
    round-1 bins.
    """
    if hist is not None:
        _dev_contig("hist", hist, torch.int32)
        if hist.numel() != SCORE_HIST_BINS:
            raise ValueError("hist must hold SCORE_HIST_BINS counts")
        if which == "both":
            score_chunk(q, k_ctx, k_self, scores, workspace, scale, stream, "lse")
            return score_chunk(q, k_ctx, k_self, scores, workspace, scale, stream, "colmax", hist)
        if which != "colmax":
            raise ValueError("hist goes with the column-max half")
    fn = {"both": _lib.kvzip_score_chunk, "lse": _lib.kvzip_score_lse,
          "colmax": _lib.kvzip_score_colmax}[which]
    for n, t in (("q", q), ("k_ctx", k_ctx), ("k_self", k_self)):
        _dev_contig(n, t, q.dtype)
    _dev_contig("scores", scores, torch.float32)
    B, G, n_in, d = q.shape
    n_c = k_ctx.shape[1]
    if k_ctx.shape != (B, n_c, d) or k_self.shape != (B, n_in, d) or scores.shape != (B, n_c):
        raise ValueError("shape mismatch between q, k_ctx, k_self and scores")
    if workspace is None:
        workspace = new_score_workspace(B, G, n_in, q.device)
    if hist is not None:
        s = _lib.kvzip_score_colmax_hist(
            _dtype_code(q), _ptr(q), _ptr(k_ctx), _ptr(k_self), _ptr(scores), B, G, n_in, n_c, d,
            float(scale), _ptr(hist), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream))
        _check(s, "kvzip_score_colmax_hist")
        return scores
    s = fn(_dtype_code(q), _ptr(q), _ptr(k_ctx), _ptr(k_self), _ptr(scores), B, G, n_in, n_c, d,
           float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
           _stream(stream))
    _check(s, "kvzip_score_" + which)
    return scores


def context_workspace_size(B: int, G: int, max_n_in: int) -> int:
    return int(_lib.kvzip_score_context_workspace_size(B, G, max_n_in))


def new_context_workspace(B: int, G: int, max_n_in: int, device=None) -> torch.Tensor:
    """Zero-initialised workspace for score_context (status word + normalisers)."""
    n = context_workspace_size(B, G, max_n_in)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def _chunk_check(q, k_self, k_ctx):
    _dev_contig("q", q, k_ctx.dtype)
    _dev_contig("k_self", k_self, k_ctx.dtype)
    B, G, n_in, d = q.shape
    if k_self.shape != (B, n_in, d) or k_ctx.shape[0] != B or k_ctx.shape[2] != d:
        raise ValueError("shape mismatch between q, k_self and k_ctx")
    return n_in


def score_context(chunks, k_ctx: torch.Tensor, scores: torch.Tensor,
                  workspace: torch.Tensor | None = None, scale: float = 0.0, stream=None):
    """Score every chunk of one context in one call (kvzip_score_context): the
    same running maximum as ``score_chunk`` over the chunks in order.
    ``chunks`` = [(q, k_self), ...] device tensors."""
    _dev_contig("k_ctx", k_ctx)
    _dev_contig("scores", scores, torch.float32)
    B, n_c, d = k_ctx.shape
    if scores.shape != (B, n_c):
        raise ValueError("scores must be [B][n_c]")
    n = len(chunks)
    if n == 0:
        return scores
    G = chunks[0][0].shape[1]
    n_in = [_chunk_check(q, ks, k_ctx) for q, ks in chunks]
    if any(q.shape[1] != G for q, _ in chunks):
        raise ValueError("every chunk must have the same number of query heads")
    if workspace is None:
        workspace = new_context_workspace(B, G, max(n_in), k_ctx.device)
    qa = (ctypes.c_void_p * n)(*[q.data_ptr() for q, _ in chunks])
    ka = (ctypes.c_void_p * n)(*[ks.data_ptr() for _, ks in chunks])
    na = (ctypes.c_int * n)(*n_in)
    s = _lib.kvzip_score_context(
        _dtype_code(k_ctx), n, qa, ka, na, _ptr(k_ctx), _ptr(scores), B, G, n_c, d, float(scale),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(s, "kvzip_score_context")
    return scores


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and return (and clear) the scoring status word (OK or ERR_TIMEOUT)."""
    return int(_lib.kvzip_workspace_status(_ptr(workspace), _stream(stream)))


def set_wait_timeout_ns(ns: int):
    _lib.kvzip_set_wait_timeout_ns(int(ns))


def set_test_stall(on: bool):
    """Timeout-path test hook: the scoring loader issues no copies while on."""
    _lib.kvzip_set_test_stall(1 if on else 0)


def lse_layout(G: int, n_in: int) -> tuple[int, int]:
    """(byte offset, row stride) of the row normalisers inside a scoring workspace."""
    off = ctypes.c_size_t(0)
    stride = ctypes.c_int64(0)
    _check(_lib.kvzip_score_lse_layout(G, n_in, ctypes.byref(off), ctypes.byref(stride)),
           "kvzip_score_lse_layout")
    return int(off.value), int(stride.value)


def read_lse(workspace: torch.Tensor, B: int, G: int, n_in: int) -> torch.Tensor:
    """Natural-log row normalisers the last pass-1 launch left in the workspace,
    [B][G*n_in] (the library stores base-2 values; converted here)."""
    R = G * n_in
    off, stride = lse_layout(G, n_in)
    lse2 = workspace[off:off + B * stride * 4].view(torch.float32).view(B, stride)[:, :R]
    return lse2 * 0.6931471805599453


# ---------------------------------------------------------------- selection

def keep_count(r: float, N: int) -> int:
    k = int(_lib.kvzip_keep_count(float(r), int(N)))
    if k < 0:
        raise ValueError("r must be in [0, 1] and N >= 0")
    return k


def select_workspace_size(N: int, n_heads: int) -> int:
    return int(_lib.kvzip_select_workspace_size(N, n_heads))


def select(scores: torch.Tensor, k: int, n_heads: int, keep: torch.Tensor | None = None,
           offsets: torch.Tensor | None = None, threshold: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None, stream=None, hist: torch.Tensor | None = None):
    """Global top-k keep mask, per-head offsets and the threshold score.

    With ``hist`` (the scores' round-1 histogram, as score_chunk(..., hist=)
    leaves it) this is kvzip_select_hist, which reads the scores once.
    Returns (keep uint8 [N], offsets int64 [n_heads+1], threshold float32 [1]).
    """
    _dev_contig("scores", scores, torch.float32)
    N = scores.numel()
    dev = scores.device
    keep = torch.empty(N, dtype=torch.uint8, device=dev) if keep is None else keep
    offsets = torch.empty(n_heads + 1, dtype=torch.int64, device=dev) if offsets is None else offsets
    threshold = torch.empty(1, dtype=torch.float32, device=dev) if threshold is None else threshold
    if workspace is None:
        workspace = torch.zeros(max(select_workspace_size(N, n_heads), 256), dtype=torch.uint8,
                                device=dev)
    if hist is not None:
        _dev_contig("hist", hist, torch.int32)
        if hist.numel() != SCORE_HIST_BINS:
            raise ValueError("hist must hold SCORE_HIST_BINS counts")
        s = _lib.kvzip_select_hist(_ptr(scores), N, int(k), int(n_heads), _ptr(hist), _ptr(keep),
                                   _ptr(offsets), _ptr(threshold), _ptr(workspace),
                                   workspace.numel(), _stream(stream))
        _check(s, "kvzip_select_hist")
        return keep, offsets, threshold
    s = _lib.kvzip_select(_ptr(scores), N, int(k), int(n_heads), _ptr(keep), _ptr(offsets),
                          _ptr(threshold), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(s, "kvzip_select")
    return keep, offsets, threshold


# ---------------------------------------------------------------- sharded selection

def shard_bins(round_: int) -> int:
    return int(_lib.kvzip_select_shard_bins(int(round_)))


def shard_workspace(N_local: int, n_heads_local: int, device=None) -> torch.Tensor:
    n = int(_lib.kvzip_select_shard_workspace_size(N_local, n_heads_local))
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def shard_begin(k: int, workspace: torch.Tensor, stream=None):
    _check(_lib.kvzip_select_shard_begin(int(k), _ptr(workspace), workspace.numel(),
                                         _stream(stream)), "kvzip_select_shard_begin")


def shard_hist(scores: torch.Tensor, round_: int, hist: torch.Tensor, workspace: torch.Tensor,
               stream=None):
    _dev_contig("scores", scores, torch.float32)
    _dev_contig("hist", hist, torch.int64)
    if hist.numel() != shard_bins(round_):
        raise ValueError("hist must hold kvzip_select_shard_bins(round) counts")
    _check(_lib.kvzip_select_shard_hist(_ptr(scores), scores.numel(), int(round_), _ptr(hist),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "kvzip_select_shard_hist")


def shard_pick(hist: torch.Tensor, round_: int, threshold: torch.Tensor | None,
               workspace: torch.Tensor, stream=None):
    _dev_contig("hist", hist, torch.int64)
    _check(_lib.kvzip_select_shard_pick(_ptr(hist), int(round_), _ptr(threshold),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "kvzip_select_shard_pick")


def shard_ties(scores: torch.Tensor, n_ties: torch.Tensor, workspace: torch.Tensor, stream=None):
    _dev_contig("n_ties", n_ties, torch.int64)
    _check(_lib.kvzip_select_shard_ties(_ptr(scores), scores.numel(), _ptr(n_ties),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "kvzip_select_shard_ties")


def shard_mask(scores: torch.Tensor, n_heads_local: int, tie_counts: torch.Tensor, rank: int,
               keep: torch.Tensor, offsets: torch.Tensor, workspace: torch.Tensor, stream=None):
    _dev_contig("tie_counts", tie_counts, torch.int64)
    _check(_lib.kvzip_select_shard_mask(_ptr(scores), scores.numel(), int(n_heads_local),
                                        _ptr(tie_counts), int(rank), _ptr(keep), _ptr(offsets),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "kvzip_select_shard_mask")


# ---------------------------------------------------------------- compaction

def compact_workspace_size(n_heads: int, n_c: int) -> int:
    return int(_lib.kvzip_compact_workspace_size(n_heads, n_c))


def compact(k: torch.Tensor, v: torch.Tensor, keep: torch.Tensor, offsets: torch.Tensor,
            total: int, k_out: torch.Tensor | None = None, v_out: torch.Tensor | None = None,
            pos_out: torch.Tensor | None = None, want_pos: bool = True,
            workspace: torch.Tensor | None = None, stream=None):
    """Pack kept rows per head.  ``total`` = offsets[-1] (known on the host as k).

    Returns (k_out [total][d], v_out [total][d], pos_out int32 [total] or None).
    """
    _dev_contig("k", k, torch.bfloat16)
    _dev_contig("v", v, torch.bfloat16)
    n_heads, n_c, d = k.shape
    dev = k.device
    k_out = torch.empty(total, d, dtype=k.dtype, device=dev) if k_out is None else k_out
    v_out = torch.empty(total, d, dtype=v.dtype, device=dev) if v_out is None else v_out
    if pos_out is None and want_pos:
        pos_out = torch.empty(total, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(compact_workspace_size(n_heads, n_c), 256), dtype=torch.uint8,
                                device=dev)
    s = _lib.kvzip_compact(_ptr(k), _ptr(v), _ptr(keep), _ptr(offsets), n_heads, n_c, d,
                           _ptr(k_out), _ptr(v_out), _ptr(pos_out), _ptr(workspace),
                           workspace.numel(), _stream(stream))
    _check(s, "kvzip_compact")
    return k_out, v_out, pos_out


# ---------------------------------------------------------------- variants

def score_chunk_sum(q, k_ctx, k_self, scores, workspace=None, scale: float = 0.0, stream=None):
    """scores += per-key sums over query rows of the chunk's softmax (bf16 only)."""
    for n, t in (("q", q), ("k_ctx", k_ctx), ("k_self", k_self)):
        _dev_contig(n, t, torch.bfloat16)
    _dev_contig("scores", scores, torch.float32)
    B, G, n_in, d = q.shape
    n_c = k_ctx.shape[1]
    if workspace is None:
        workspace = new_score_workspace(B, G, n_in, q.device)
    _check(_lib.kvzip_score_chunk_sum(_ptr(q), _ptr(k_ctx), _ptr(k_self), _ptr(scores), B, G,
                                      n_in, n_c, d, float(scale), _ptr(workspace),
                                      workspace.numel(), _stream(stream)),
           "kvzip_score_chunk_sum")
    return scores


def token_scores(scores: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    """max over heads per position; scores [n_heads][n_c] float32 -> [n_c]."""
    _dev_contig("scores", scores, torch.float32)
    n_heads, n_c = scores.shape
    out = torch.empty(n_c, dtype=torch.float32, device=scores.device) if out is None else out
    _check(_lib.kvzip_token_scores(_ptr(scores), n_heads, n_c, _ptr(out), _stream(stream)),
           "kvzip_token_scores")
    return out


def expand_keep(keep_pos: torch.Tensor, pos_offsets: torch.Tensor, n_heads: int, stream=None):
    """Position mask (from select with n_heads = 1) -> per-head mask and offsets."""
    n_c = keep_pos.numel()
    keep = torch.empty(n_heads * n_c, dtype=torch.uint8, device=keep_pos.device)
    offsets = torch.empty(n_heads + 1, dtype=torch.int64, device=keep_pos.device)
    _check(_lib.kvzip_expand_keep(_ptr(keep_pos), _ptr(pos_offsets), n_heads, n_c, _ptr(keep),
                                  _ptr(offsets), _stream(stream)), "kvzip_expand_keep")
    return keep, offsets


def select_per_head(scores: torch.Tensor, k_per_head: int, workspace=None, stream=None):
    """Uniform budgets: top k_per_head of each head; scores [n_heads][n_c] float32."""
    _dev_contig("scores", scores, torch.float32)
    n_heads, n_c = scores.shape
    dev = scores.device
    keep = torch.empty(n_heads * n_c, dtype=torch.uint8, device=dev)
    offsets = torch.empty(n_heads + 1, dtype=torch.int64, device=dev)
    if workspace is None:
        n = int(_lib.kvzip_select_per_head_workspace_size(n_heads, n_c))
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
    _check(_lib.kvzip_select_per_head(_ptr(scores), n_heads, n_c, int(k_per_head), _ptr(keep),
                                      _ptr(offsets), _ptr(workspace), workspace.numel(),
                                      _stream(stream)), "kvzip_select_per_head")
    return keep, offsets


# ---------------------------------------------------------------- head scores

def head_scores(scores: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    """max over positions of each head's scores; scores [n_heads][n_c] float32."""
    _dev_contig("scores", scores, torch.float32)
    n_heads, n_c = scores.shape
    out = torch.empty(n_heads, dtype=torch.float32, device=scores.device) if out is None else out
    _check(_lib.kvzip_head_scores(_ptr(scores), n_heads, n_c, _ptr(out), _stream(stream)),
           "kvzip_head_scores")
    return out


# ---------------------------------------------------------------- decode attention

def decode_workspace_size(n_heads: int, G: int, d: int) -> int:
    return int(_lib.kvzip_decode_workspace_size(n_heads, G, d))


def decode_attention(q: torch.Tensor, k_packed: torch.Tensor, v_packed: torch.Tensor,
                     offsets: torch.Tensor, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, scale: float = 0.0, stream=None):
    """softmax(scale * K_h q) V_h per KV head over its kept rows.

    q [n_heads][G][d] bf16; k_packed / v_packed [total][d] bf16; offsets int64
    [n_heads+1].  Returns out [n_heads][G][d] float32.
    """
    _dev_contig("q", q, torch.bfloat16)
    n_heads, G, d = q.shape
    dev = q.device
    out = torch.empty(n_heads, G, d, dtype=torch.float32, device=dev) if out is None else out
    if workspace is None:
        workspace = torch.zeros(max(decode_workspace_size(n_heads, G, d), 256), dtype=torch.uint8,
                                device=dev)
    kp = k_packed if k_packed.numel() else None
    vp = v_packed if v_packed.numel() else None
    if k_packed.shape != v_packed.shape:
        raise ValueError("k_packed and v_packed must have the same shape")
    n_rows = k_packed.shape[0] if k_packed.numel() else 0
    _check(_lib.kvzip_decode_attention(_ptr(q), _ptr(kp), _ptr(vp), n_rows, _ptr(offsets),
                                       n_heads, G, d, float(scale), _ptr(out), _ptr(workspace),
                                       workspace.numel(), _stream(stream)),
           "kvzip_decode_attention")
    return out


def last_launch_count() -> int:
    return int(_lib.kvzip_last_launch_count())
