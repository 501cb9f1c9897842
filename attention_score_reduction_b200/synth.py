"""Seeded synthetic inputs for KVzip scoring, selection and compaction.

This module only draws random tensors with the shapes and value distributions of
the workloads; it holds none of the method's arithmetic (no attention, no
softmax, no ranking).  Both the CUDA path and the CPU oracle are fed from here.

What the tensors stand in for (KVzip: Query-Agnostic KV Cache Compression with
Context Reconstruction, blog post section 4.1 / 4.3.1; rebuttal answer on
head-level scores for the L x H x n_c score shape):

* ``k_ctx`` / ``v``   -- the prefilled context cache K_c, V_c, per (layer, KV head),
                         layout ``[units][n_c][d]`` with ``units = L * H``.
* ``q``               -- the reconstruction queries of one chunk,
                         ``[units][G][n_in][d]`` with ``n_in = P + m_chunk``
                         (P repeat-prompt rows, then the chunk's context rows).
* ``k_self``          -- the keys the chunk's own tokens produce, ``[units][n_in][d]``.

No model exists here, so every tensor is drawn i.i.d. with the recipe of its
workload (see ``WORKLOADS``): N(0, 1) entries, a fraction of key rows scaled up
("high-norm" keys), optional attention-sink rows at the start of the context,
or a lognormal per-row key norm.  Values are rounded once to the storage dtype.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BASE_SEED = 20251121

# tensor ids that enter the seed
_T_KCTX, _T_V, _T_Q, _T_KSELF = 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    """Shapes and input recipe of one synthetic scoring/eviction job."""

    name: str
    L: int                  # layers
    H: int                  # KV heads per layer
    G: int                  # query heads sharing one KV head (GQA group)
    d: int                  # head dim
    n_c: int                # context length (prefilled keys per head)
    m: int                  # context rows per chunk
    r: tuple = (0.3,)       # kept fractions
    P: int = 16             # repeat-prompt rows per chunk
    dtype: str = "bf16"     # storage dtype of Q / K ("bf16" or "f32")
    hi_frac: float = 0.0    # fraction of key rows scaled by hi_scale
    hi_scale: float = 3.0
    sinks: int = 0          # leading context keys scaled by sink_scale
    sink_scale: float = 5.0
    lognormal_sigma: float = 0.0  # per-row key norm factor exp(N(0, sigma^2))
    cfg_id: int = 0
    max_chunks: int = 0     # 0: reconstruct every chunk; else only the first max_chunks
    notes: str = field(default="", compare=False)

    @property
    def units(self) -> int:
        return self.L * self.H

    @property
    def n_chunks(self) -> int:
        n = (self.n_c + self.m - 1) // self.m
        return min(n, self.max_chunks) if self.max_chunks > 0 else n

    def chunk_rows(self, c: int) -> tuple[int, int]:
        """Context rows [lo, hi) that chunk c reconstructs."""
        lo = c * self.m
        return lo, min(lo + self.m, self.n_c)

    def n_in(self, c: int) -> int:
        lo, hi = self.chunk_rows(c)
        return self.P + (hi - lo)

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The five workloads (shapes of LLaMA3.1-8B, Qwen2.5-14B, Gemma3-12B KV layouts).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", L=1, H=1, G=4, d=128, n_c=2048, m=496,
                          r=(0.3,), dtype="f32", hi_frac=0.01, cfg_id=1, max_chunks=1,
                          notes="one chunk of 16 prompt + 496 context rows; all 2048 keys scored"),
    "llama8b_16k": Workload("llama8b_16k", L=32, H=8, G=4, d=128, n_c=16384, m=2048,
                            r=(0.3,), hi_frac=0.01, sinks=4, cfg_id=2),
    "llama8b_128k": Workload("llama8b_128k", L=32, H=8, G=4, d=128, n_c=131072, m=2048,
                             r=(0.3, 0.5), hi_frac=0.01, sinks=4, cfg_id=3),
    "qwen14b_120k": Workload("qwen14b_120k", L=48, H=8, G=5, d=128, n_c=122880, m=2048,
                             r=(0.25,), lognormal_sigma=0.5, cfg_id=4),
    "gemma12b_170k": Workload("gemma12b_170k", L=48, H=8, G=2, d=256, n_c=174080, m=2048,
                              r=(0.3,), hi_frac=0.02, cfg_id=5,
                              notes="chunk size swept over 1024, 2048, 4096"),
}


def _seed(wl: Workload, tensor: int, chunk: int = 0, salt: int = 0) -> int:
    return (BASE_SEED + 1_000_003 * wl.cfg_id + 7_919 * tensor + 104_729 * chunk
            + 15_485_863 * salt) % (2**63 - 1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _storage(wl: Workload, kind: str) -> torch.dtype:
    if kind == "v":
        return torch.bfloat16
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def _keys(wl: Workload, units: int, n: int, g: torch.Generator, device,
          with_sinks: bool) -> torch.Tensor:
    """N(0,1) key rows with the workload's per-row norm recipe, in float32."""
    k = torch.randn(units, n, wl.d, generator=g, device=device, dtype=torch.float32)
    row = torch.ones(units, n, 1, device=device, dtype=torch.float32)
    if wl.hi_frac > 0.0:
        n_hi = int(round(wl.hi_frac * n))
        if n_hi > 0:
            pick = torch.rand(units, n, generator=g, device=device).argsort(dim=1)[:, :n_hi]
            row.scatter_(1, pick.unsqueeze(-1), wl.hi_scale)
    if wl.lognormal_sigma > 0.0:
        z = torch.randn(units, n, 1, generator=g, device=device, dtype=torch.float32)
        row = row * torch.exp(wl.lognormal_sigma * z)
    if with_sinks and wl.sinks > 0:
        row[:, : min(wl.sinks, n)] = row[:, : min(wl.sinks, n)] * wl.sink_scale
    return k.mul_(row)   # in place: the full-size float32 keys are tens of GB


def context_kv(wl: Workload, device="cpu", units: int | None = None):
    """(k_ctx, v): ``[units][n_c][d]`` each; k in the workload dtype, v in bf16."""
    u = wl.units if units is None else units
    k = _keys(wl, u, wl.n_c, _gen(device, _seed(wl, _T_KCTX)), device, with_sinks=True)
    k = k.to(_storage(wl, "k"))
    v = torch.randn(u, wl.n_c, wl.d, generator=_gen(device, _seed(wl, _T_V)),
                    device=device, dtype=torch.float32)
    return k, v.to(torch.bfloat16)


def context_keys(wl: Workload, device="cpu", units: int | None = None) -> torch.Tensor:
    u = wl.units if units is None else units
    k = _keys(wl, u, wl.n_c, _gen(device, _seed(wl, _T_KCTX)), device, with_sinks=True)
    return k.to(_storage(wl, "k"))


def chunk_qk(wl: Workload, c: int, device="cpu", units: int | None = None):
    """(q, k_self) of chunk c: ``[units][G][n_in][d]`` and ``[units][n_in][d]``."""
    u = wl.units if units is None else units
    n_in = wl.n_in(c)
    q = torch.randn(u, wl.G, n_in, wl.d, generator=_gen(device, _seed(wl, _T_Q, c)),
                    device=device, dtype=torch.float32)
    ks = _keys(wl, u, n_in, _gen(device, _seed(wl, _T_KSELF, c)), device, with_sinks=False)
    return q.to(_storage(wl, "q")), ks.to(_storage(wl, "k"))


def random_scores(n_heads: int, n_c: int, seed: int, levels: int = 0, device="cpu"):
    """Score arrays for selection tests: values in (0, 1], float32.

    ``levels > 0`` quantises them onto that many distinct values, which makes
    ties frequent (every value repeated ~N/levels times).
    """
    g = _gen(device, BASE_SEED + 31 * seed)
    s = torch.rand(n_heads, n_c, generator=g, device=device, dtype=torch.float32)
    s = s.pow(4.0)  # skewed like attention maxima: many small, few large
    if levels > 0:
        s = (torch.floor(s * levels) + 1.0) / levels
    else:
        s = s.clamp_min(1e-12)
    return s
