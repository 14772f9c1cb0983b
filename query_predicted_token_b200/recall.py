"""Selection recall: how much of the top-C set chosen with one query the set
chosen with the true next query keeps.

A synthetic analogue of the pages' evidence for query-aware selection (the
research-map summary, "Approach"; the reproduction card, claim C5 on temporal
locality and linear query prediction): for step t+1, the set chosen with the
predicted query q_hat_{t+1} is compared with the set the true query q_{t+1}
would choose, and with the set chosen by reusing the current query q_t one step
late.  The sets come from the library's own scan and selection kernels; only
the set intersection runs on the host (this is analysis, not the decode path).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import _lib as L


def topk_sets(q: torch.Tensor, kv: "L.KV", C: int, stream=None):
    """The top-C token set of every (sequence, KV head) for query ``q [B, Hq, d]``
    (scored as fp32): ``(idx [B, Hkv, C] int32, count [B, Hkv] int32)`` on the device."""
    B, Hkv, T = kv.batch, kv.n_kv_heads, kv.t_max
    dev = kv.k.device
    scores = torch.empty(B, Hkv, T, dtype=torch.float32, device=dev)
    L.score_keys(q.float().contiguous(), kv, scores, stream=stream)
    idx = torch.empty(B, Hkv, C, dtype=torch.int32, device=dev)
    cnt = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
    L.select_topk(scores, kv.seq_lens, C, idx, cnt, stream=stream)
    return idx, cnt


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
