"""Oracle for the page-level comparison path (Quest-style) (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU arms may use this.

Pages: the baseline is query-aware page-level sparse decoding whose page
filtering depends on the current query (abstract; summary, "Problem"); its
extra cost is a page-scan term 2 q h (T/P) with P tokens per page (repro card,
"Key finding ...").  The pages do not spell out the page score; this oracle
uses the per-page, per-channel key minimum and maximum and the upper bound
they imply for the logit of any key in the page:

Q1  meta: kmin_c, kmax_c over the (valid) tokens of each page.
Q2  page score u_p = max over the group's query heads of
    sum_c max(q_c kmin_c, q_c kmax_c) / sqrt(d), with the current query.
Q3  the ceil(C / P) pages with the highest score are kept (lowest page index
    on ties); their tokens j < T_b are attended, in ascending order.

Pins (tests/test_oracle_quest.py): the bound is >= every true logit of its
page; a page of identical keys makes it exact; brute-force page ranking.
"""
from __future__ import annotations

import math

import numpy as np


def quest_meta(K: np.ndarray, page_size: int):
    """``K [T_b, d]`` of one KV head -> ``kmin, kmax [n_pages, d]`` (Q1)."""
    T_b, d = K.shape
    n = (T_b + page_size - 1) // page_size
    kmin = np.empty((n, d), dtype=np.float64)
    kmax = np.empty((n, d), dtype=np.float64)
    for p in range(n):
        blk = np.asarray(K[p * page_size:min(T_b, (p + 1) * page_size)], dtype=np.float64)
        kmin[p] = blk.min(axis=0)
        kmax[p] = blk.max(axis=0)
    return kmin, kmax


def quest_page_scores(qgroup: np.ndarray, kmin: np.ndarray, kmax: np.ndarray) -> np.ndarray:
    """``qgroup [G, d]`` -> page upper bounds ``[n_pages]`` (Q2)."""
    q = np.asarray(qgroup, dtype=np.float64)[:, None, :]          # [G, 1, d]
    ub = np.maximum(q * kmin[None], q * kmax[None]).sum(axis=-1)   # [G, n_pages]
    return ub.max(axis=0) / math.sqrt(kmin.shape[-1])


def quest_select_row(page_scores: np.ndarray, T_b: int, C: int, page_size: int):
    """Q3 for one KV head -> (ascending token indices, count)."""
    s = np.asarray(page_scores, dtype=np.float64)
    n_pages = s.shape[0]
    keep = min(n_pages, (C + page_size - 1) // page_size)
    order = np.lexsort((np.arange(n_pages), -s))
    pages = np.sort(order[:keep])
    toks = (pages[:, None] * page_size + np.arange(page_size)[None, :]).reshape(-1)
    toks = toks[toks < T_b].astype(np.int32)
    return toks, int(toks.shape[0])


def quest_select(q: np.ndarray, keys, C: int, page_size: int):
    """Whole batch: ``q [B, Hq, d]``, ``keys[b] [Hkv, T_b, d]`` -> ``idx [B, Hkv, C']``, ``count``.

    ``C' = ceil(C / P) * P`` so that whole pages fit.
    """
    B, Hq, d = q.shape
    Hkv = keys[0].shape[0]
    G = Hq // Hkv
    cap = ((C + page_size - 1) // page_size) * page_size
    idx = np.full((B, Hkv, cap), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv), dtype=np.int32)
    for b in range(B):
        T_b = keys[b].shape[1]
        for h in range(Hkv):
            kmin, kmax = quest_meta(keys[b][h], page_size)
            ps = quest_page_scores(q[b, h * G:(h + 1) * G], kmin, kmax)
            toks, n = quest_select_row(ps, T_b, C, page_size)
            idx[b, h, :n] = toks
            cnt[b, h] = n
    return idx, cnt
