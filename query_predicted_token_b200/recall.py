"""Selection recall: how much of the top-C set chosen with one query the set
chosen with the true next query keeps, and how stable the top-C sets of
successive queries are.

A synthetic analogue of the pages' evidence for query-aware selection (the
research-map summary, "Approach"; the reproduction card, claim C5 on temporal
locality and linear query prediction, the paper's Figs. 4 and 5): for step
t+1, the set chosen with the predicted query q_hat_{t+1} is compared with the
set the true query q_{t+1} would choose, and with the set chosen by reusing
the current query q_t one step late; and the set of step t is compared with
the sets of the 16 steps before it.  The sets come from the library's own scan
and selection kernels; the set intersections, and for the softmax-mass reading
the per-head normalisation of the scan's scores, run on the host (this is
analysis of what the decode path selects, not the decode path).

How a KV head's set is formed from its group's G query heads (reading S2):
  max       one score per token, the maximum over the group (the library's path);
  mean      one score per token from the group's mean query;
  mass      the sum over the group of each head's softmax probabilities;
  per_head  every query head keeps its own top C (recall averaged over heads).
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import _lib as L


def _scan_select(q: torch.Tensor, kv: "L.KV", C: int, stream=None):
    """Top-C sets for ``q [B, Hq, d]`` grouped onto the cache's KV heads (max over the group)."""
    B, Hkv, T = kv.batch, kv.n_kv_heads, kv.t_max
    dev = kv.k.device
    scores = torch.empty(B, Hkv, T, dtype=torch.float32, device=dev)
    L.score_keys(q.float().contiguous(), kv, scores, stream=stream)
    idx = torch.empty(B, Hkv, C, dtype=torch.int32, device=dev)
    cnt = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
    L.select_topk(scores, kv.seq_lens, C, idx, cnt, stream=stream)
    return idx, cnt, scores


def topk_sets(q: torch.Tensor, kv: "L.KV", C: int, stream=None):
    """The top-C token set of every (sequence, KV head) for query ``q [B, Hq, d]``
    (scored as fp32, max over the group): ``(idx [B, Hkv, C], count [B, Hkv])`` on the device."""
    idx, cnt, _ = _scan_select(q, kv, C, stream)
    return idx, cnt


def _heads(q: torch.Tensor, kv: "L.KV"):
    B, Hq, d = q.shape
    return q.float().view(B, kv.n_kv_heads, Hq // kv.n_kv_heads, d)


def topk_sets_reading(q: torch.Tensor, kv: "L.KV", C: int, reading: str):
    """Host copies of the sets under reading ``reading`` of S2: ``(idx, count)`` with
    shape ``[B, Hkv, ...]`` (``per_head``: ``[B, Hkv, G, C]`` and ``[B, Hkv, G]``)."""
    if reading == "max":
        i, c = topk_sets(q, kv, C)
        return i.cpu().numpy(), c.cpu().numpy()
    qh = _heads(q, kv)
    if reading == "mean":
        i, c = topk_sets(qh.mean(dim=2).contiguous(), kv, C)
        return i.cpu().numpy(), c.cpu().numpy()
    G = qh.shape[2]
    per = [_scan_select(qh[:, :, g].contiguous(), kv, C) for g in range(G)]
    if reading == "per_head":
        return (np.stack([p[0].cpu().numpy() for p in per], axis=2),
                np.stack([p[1].cpu().numpy() for p in per], axis=2))
    if reading != "mass":
        raise ValueError(reading)
    # sum over the group of each head's softmax over its candidate tokens j < T_b
    lens = (kv.seq_lens.cpu().numpy() if kv.seq_lens is not None
            else np.full(kv.batch, kv.t_max)).astype(np.int64)
    s = np.stack([p[2].cpu().numpy().astype(np.float64) for p in per], axis=0)   # [G, B, Hkv, T]
    mass = np.zeros(s.shape[1:], dtype=np.float32)
    for b in range(s.shape[1]):
        Tb = int(lens[b])
        x = s[:, b, :, :Tb]
        e = np.exp(x - x.max(axis=-1, keepdims=True))
        mass[b, :, :Tb] = (e / e.sum(axis=-1, keepdims=True)).sum(axis=0)
    dev = kv.k.device
    idx = torch.empty(kv.batch, kv.n_kv_heads, C, dtype=torch.int32, device=dev)
    cnt = torch.empty(kv.batch, kv.n_kv_heads, dtype=torch.int32, device=dev)
    L.select_topk(torch.from_numpy(mass).to(dev), kv.seq_lens, C, idx, cnt)
    return idx.cpu().numpy(), cnt.cpu().numpy()


def overlap(idx_a: np.ndarray, cnt_a: np.ndarray, idx_b: np.ndarray, cnt_b: np.ndarray) -> np.ndarray:
    """Per unit ``|A ∩ B| / |B|`` for index sets ``[..., C]`` with valid counts ``[...]``
    (1.0 where B is empty)."""
    idx_a, idx_b = np.asarray(idx_a), np.asarray(idx_b)
    cnt_a, cnt_b = np.asarray(cnt_a), np.asarray(cnt_b)
    out = np.ones(cnt_b.shape, dtype=np.float64)
    for u in np.ndindex(cnt_b.shape):
        nb = int(cnt_b[u])
        if nb == 0:
            continue
        a = idx_a[u][: int(cnt_a[u])]
        b = idx_b[u][:nb]
        out[u] = np.intersect1d(a, b, assume_unique=True).size / nb
    return out


def recall_report(kv: "L.KV", C: int, q_true: torch.Tensor, sets: Dict[str, torch.Tensor],
                  chosen: Optional[Dict[str, tuple]] = None) -> Dict[str, float]:
    """Mean recall of the true next query's top-C set for each named query in
    ``sets`` (``name -> q [B, Hq, d]``) and each named ready selection in
    ``chosen`` (``name -> (idx, count)``)."""
    ti, tc = topk_sets(q_true, kv, C)
    ti, tc = ti.cpu().numpy(), tc.cpu().numpy()
    out = {}
    for name, q in sets.items():
        i, c = topk_sets(q, kv, C)
        out[name] = float(overlap(i.cpu().numpy(), c.cpu().numpy(), ti, tc).mean())
    for name, (i, c) in (chosen or {}).items():
        out[name] = float(overlap(i.cpu().numpy(), c.cpu().numpy(), ti, tc).mean())
    return out


def reading_recall(kv: "L.KV", C: int, q_true: torch.Tensor, queries: Dict[str, torch.Tensor],
                   readings: Sequence[str] = ("mean", "mass", "per_head")) -> Dict[str, Dict[str, float]]:
    """For each S2 reading, the mean recall of the true next query's set by the set of
    each named query, both formed under that reading."""
    out = {}
    for r in readings:
        ti, tc = topk_sets_reading(q_true, kv, C, r)
        out[r] = {}
        for name, q in queries.items():
            i, c = topk_sets_reading(q, kv, C, r)
            out[r][name] = float(overlap(i, c, ti, tc).mean())
    return out


def window_overlap(kv: "L.KV", C: int, queries: Sequence[torch.Tensor]) -> Dict[str, float]:
    """Temporal locality of the selection: ``queries`` are the true queries of W+1
    successive steps, oldest first; per unit, the overlap of the last step's set with
    each earlier step's set (averaged: "mean") and with their union ("union"), then
    the mean over units."""
    sets = [topk_sets(q, kv, C) for q in queries]
    sets = [(i.cpu().numpy(), c.cpu().numpy()) for i, c in sets]
    last_i, last_c = sets[-1]
    mean = np.mean([overlap(i, c, last_i, last_c) for i, c in sets[:-1]], axis=0)
    union = np.ones(last_c.shape)
    for u in np.ndindex(last_c.shape):
        n = int(last_c[u])
        if n == 0:
            continue
        earlier = np.concatenate([i[u][: int(c[u])] for i, c in sets[:-1]])
        union[u] = np.intersect1d(np.unique(earlier), last_i[u][:n]).size / n
    return {"mean": float(mean.mean()), "union": float(union.mean()), "window": len(queries) - 1}
