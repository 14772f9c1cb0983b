"""Seeded synthetic workloads for predicted-query sparse decoding.

The pages measure long chain-of-thought decoding of Qwen3-8B / Qwen3-32B on
AIME-24/25, GPQA-Diamond and MATH-500 (AsyncSpade abstract; research-map
summary, "Experimental setup").  No dataset or weight is used here: these
generators stand in for them with the head geometry of those models, 32k-64k
contexts and high concurrency.  Nothing in this module computes any step of
the method; it only draws numbers and lays them out.

Recipe (every draw is seeded, so both the CUDA path and the oracle see the
same bits):

* K, V: i.i.d. N(0, 1).  For the bf16 workloads K is multiplied by a
  per-(KV head, channel) scale drawn from U(0.5, 2), shared by all sequences
  and tokens, then both are rounded to bf16.
* Contiguous layout: K, V are ``[B, Hkv, T, d]``.  Paged layout: pages of
  ``page_size`` tokens, ``[n_pages, Hkv, page_size, d]``; the page table maps
  each sequence's logical pages onto a random permutation of all physical
  pages (``-1`` past the end of a sequence).
* Ragged lengths: ``T_b ~ U[t_min, t_max]`` (integers), drawn once.
* Query history: an AR(1) series per query head, ``q_0 ~ N(0, 1)``,
  ``q_{s+1} = rho * q_s + 0.1 * N(0, 1)``, ``W + 2`` vectors: the first
  ``W + 1`` fill the history window, the last is the true current query.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    t_max: int               # tokens per sequence (upper bound when ragged)
    t_min: int               # lower bound of the ragged draw (== t_max when fixed)
    kv_dtype: str            # "f32" or "bf16"
    W: int                   # number of lagged queries in the history
    C: int                   # selected tokens per (sequence, KV head)
    windows: Tuple[int, ...]  # pooling windows
    lam: float               # ridge parameter
    rho: float               # AR(1) coefficient of the synthetic query series
    seed: int
    page_size: int = 0       # 0 = contiguous KV layout
    k_channel_scale: bool = True
    description: str = ""

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def ragged(self) -> bool:
        return self.t_min != self.t_max

    @property
    def max_pages(self) -> int:
        return math.ceil(self.t_max / self.page_size) if self.page_size else 0

    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.kv_dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_f32_t512", 1, 4, 2, 64, 512, 512, "f32", 8, 64, (4, 8), 1e-2, 0.9, 0,
                 k_channel_scale=False,
                 description="1 sequence, 4 query / 2 KV heads, d=64, T=512, fp32, C=64"),
        Workload("qwen3_8b_shaped_32k", 8, 32, 8, 128, 32768, 32768, "bf16", 16, 2048, (4, 8, 16), 1e-2, 0.9, 1,
                 description="Qwen3-8B head geometry, batch 8, T=32768, bf16, C=2048"),
        Workload("qwen3_32b_shaped_32k", 16, 64, 8, 128, 32768, 32768, "bf16", 16, 2048, (4, 8, 16), 1e-2, 0.9, 2,
                 description="Qwen3-32B head geometry (GQA group 8), batch 16, T=32768, bf16, C=2048"),
        Workload("longcot_ragged_paged_b64", 64, 32, 8, 128, 65536, 8192, "bf16", 16, 2048, (4, 8, 16), 1e-2, 0.9, 3,
                 page_size=16,
                 description="batch 64, T_b ~ U[8192, 65536], 16-token pages, shuffled page table"),
        Workload("longcot_ragged_paged_b8", 8, 32, 8, 128, 65536, 8192, "bf16", 16, 2048, (4, 8, 16), 1e-2, 0.9, 3,
                 page_size=16,
                 description="the ragged paged workload with 8 sequences (a profiling-size case, ~1.2 GB of K/V)"),
        Workload("qwen3_8b_shaped_b32_8k", 32, 32, 8, 128, 8192, 8192, "bf16", 16, 2048, (4, 8, 16), 1e-2, 0.9, 4,
                 description="Qwen3-8B head geometry, batch 32, T=8192, C=2048 (a profiling-size case with the "
                             "ragged batch's 200+ attention tiles per SM, ~1.1 GB of K/V)"),
        Workload("quest_page_scan_8b_32k", 8, 32, 8, 128, 32768, 32768, "bf16", 16, 2048, (4, 8, 16), 1e-2, 0.9, 1,
                 page_size=16,
                 description="Qwen3-8B shapes for the page-scan comparison path, 16-token pages"),
    ]
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def _cpu_gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _dev_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def sequence_lengths(wl: Workload) -> torch.Tensor:
    """``[B]`` int32 token counts (CPU)."""
    if not wl.ragged:
        return torch.full((wl.batch,), wl.t_max, dtype=torch.int32)
    g = _cpu_gen(wl.seed * 1000 + 11)
    return torch.randint(wl.t_min, wl.t_max + 1, (wl.batch,), generator=g, dtype=torch.int64).to(torch.int32)


def key_channel_scale(wl: Workload) -> torch.Tensor:
    """``[Hkv, d]`` fp32 per-channel key scale (ones when disabled)."""
    if not wl.k_channel_scale:
        return torch.ones(wl.n_kv_heads, wl.head_dim)
    g = _cpu_gen(wl.seed * 1000 + 13)
    return 0.5 + 1.5 * torch.rand(wl.n_kv_heads, wl.head_dim, generator=g)


def kv_cache(wl: Workload, device="cpu", layout: Optional[str] = None) -> dict:
    """Draw the KV cache of a workload.

    ``layout`` is "contiguous" or "paged" (default: paged iff ``wl.page_size``).
    Returns a dict with ``k``, ``v`` (on ``device``), ``seq_lens`` int32 ``[B]``,
    ``page_table`` int32 ``[B, max_pages]`` or None, ``page_size`` and ``t_max``.
    """
    device = torch.device(device)
    layout = layout or ("paged" if wl.page_size else "contiguous")
    dt = wl.torch_dtype()
    B, H, d = wl.batch, wl.n_kv_heads, wl.head_dim
    lens = sequence_lengths(wl)
    scale = key_channel_scale(wl).to(device)
    out = {"seq_lens": lens.to(device), "t_max": wl.t_max}
    if layout == "contiguous":
        T = wl.t_max
        k = torch.empty(B, H, T, d, dtype=dt, device=device)
        v = torch.empty(B, H, T, d, dtype=dt, device=device)
        for b in range(B):
            gk = _dev_gen(wl.seed * 1000 + 100 + b, device)
            gv = _dev_gen(wl.seed * 1000 + 500 + b, device)
            kb = torch.randn(H, T, d, generator=gk, device=device)
            kb.mul_(scale[:, None, :])
            k[b].copy_(kb)
            del kb
            v[b].copy_(torch.randn(H, T, d, generator=gv, device=device))
        out.update(k=k, v=v, page_table=None, page_size=0)
        return out
    P = wl.page_size or 16
    max_pages = math.ceil(wl.t_max / P)
    n_per = [(int(t) + P - 1) // P for t in lens.tolist()]
    n_pages = sum(n_per)
    perm = torch.randperm(n_pages, generator=_cpu_gen(wl.seed * 1000 + 17)).to(torch.int32)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(n_per):
        table[b, :n] = perm[off:off + n]
        off += n
    k = torch.empty(n_pages, H, P, d, dtype=dt, device=device)
    v = torch.empty(n_pages, H, P, d, dtype=dt, device=device)
    chunk = 8192
    gk = _dev_gen(wl.seed * 1000 + 101, device)
    gv = _dev_gen(wl.seed * 1000 + 501, device)
    for p0 in range(0, n_pages, chunk):
        p1 = min(n_pages, p0 + chunk)
        kb = torch.randn(p1 - p0, H, P, d, generator=gk, device=device)
        kb.mul_(scale[None, :, None, :])
        k[p0:p1].copy_(kb)
        del kb
        v[p0:p1].copy_(torch.randn(p1 - p0, H, P, d, generator=gv, device=device))
    out.update(k=k, v=v, page_table=table.to(device), page_size=P, n_pages=n_pages)
    return out


def query_history(wl: Workload, steps: int = 1) -> Tuple[torch.Tensor, torch.Tensor]:
    """AR(1) query series per head (CPU fp32).

    Returns ``qhist [B, Hq, W+1, d]`` (oldest first) and ``q_next
    [steps, B, Hq, d]``: the true queries of the next ``steps`` decode steps.
    """
    g = _cpu_gen(wl.seed * 1000 + 777)
    B, Hq, d = wl.batch, wl.n_q_heads, wl.head_dim
    n = wl.W + 1 + steps
    q = torch.empty(n, B, Hq, d)
    q[0] = torch.randn(B, Hq, d, generator=g)
    for s in range(1, n):
        q[s] = wl.rho * q[s - 1] + 0.1 * torch.randn(B, Hq, d, generator=g)
    qhist = q[: wl.W + 1].permute(1, 2, 0, 3).contiguous()
    return qhist, q[wl.W + 1:].contiguous()


def score_rows(rows: int, T: int, seed: int, kind: str = "normal") -> torch.Tensor:
    """fp32 score rows ``[rows, T]`` for selection tests.

    kinds: "normal" (N(0,1)), "ties" (small integers: heavy ties, with -0.0
    and +0.0 mixed in), "special" (normal values with +-inf, +-0.0, subnormals
    and huge magnitudes planted), "equal" (every score identical).
    """
    g = _cpu_gen(seed)
    if kind == "normal":
        return torch.randn(rows, T, generator=g)
    if kind == "ties":
        s = torch.randint(-3, 4, (rows, T), generator=g).to(torch.float32)
        zero = s == 0
        flip = torch.rand(rows, T, generator=g) < 0.5
        s[zero & flip] = -0.0
        return s
    if kind == "special":
        s = torch.randn(rows, T, generator=g)
        u = torch.rand(rows, T, generator=g)
        s[u < 0.02] = float("inf")
        s[(u >= 0.02) & (u < 0.05)] = float("-inf")
        s[(u >= 0.05) & (u < 0.08)] = 0.0
        s[(u >= 0.08) & (u < 0.11)] = -0.0
        s[(u >= 0.11) & (u < 0.13)] = 1e-40
        s[(u >= 0.13) & (u < 0.15)] = -1e-40
        s[(u >= 0.15) & (u < 0.17)] = 3e38
        s[(u >= 0.17) & (u < 0.19)] = -3e38
        return s
    if kind == "equal":
        return torch.full((rows, T), 0.25)
    raise ValueError(kind)


def random_selection(batch: int, n_kv_heads: int, C: int, seq_lens, seed: int):
    """Random ascending token subsets for attention tests.

    Returns ``idx [B, Hkv, C]`` int32 (ascending, -1 padded) and ``count
    [B, Hkv]`` int32 with ``count = min(C, T_b)``.
    """
    g = _cpu_gen(seed)
    lens = [int(t) for t in torch.as_tensor(seq_lens).tolist()]
    idx = torch.full((batch, n_kv_heads, C), -1, dtype=torch.int32)
    cnt = torch.zeros(batch, n_kv_heads, dtype=torch.int32)
    for b in range(batch):
        n = min(C, lens[b])
        for h in range(n_kv_heads):
            pick = torch.randperm(lens[b], generator=g)[:n].sort().values
            idx[b, h, :n] = pick.to(torch.int32)
            cnt[b, h] = n
    return idx, cnt

