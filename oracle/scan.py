"""Oracle steps 2-3: score every cached key, then pick the top C (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU arms may use this.

Pages: token-level, query-aware KV selection replaces page-level filtering
(abstract; summary, "Problem"); the budget is about two thousand selected
tokens (summary, "Key results"; repro card, "Key finding ...").  The targets
are Qwen3 models, whose attention groups G = Hq / Hkv query heads on one KV
head (summary, "Key results").  Readings:

S1  score = (qhat . k_j) / sqrt(d).
S2  GQA: one score per KV head, the maximum over the G query heads of its group
    (query head hq belongs to KV head hq // G).  One index set per KV head.
T1  scores are compared as IEEE values (-0.0 == +0.0; +-inf allowed; NaN is
    invalid input).
T2  ties at the threshold go to the lowest token index.
T3  the chosen indices are returned in ascending order.
T4  only tokens j < T_b are candidates; if T_b <= C all of them are chosen and
    the rest of the output is -1.
T5  no forced sink or recent tokens: plain top C.

Pins (tests/test_oracle_scan.py): hand-computed scores; a triple-loop brute
force; invariance under permuting the heads of a group; the G=1 case;
selection against the definition "j is chosen iff #{i: s_i > s_j} +
#{i < j: s_i == s_j} < C" evaluated by brute force; all-equal, heavy-tie,
+-0.0 and +-inf rows.  S2 as a reading of the paper is parity unpinned.
"""
from __future__ import annotations

import math

import numpy as np


def gather_sequence(k_pages: np.ndarray, table_row: np.ndarray, T_b: int, page_size: int) -> np.ndarray:
    """Resolve a paged cache ``[n_pages, Hkv, P, d]`` into ``[Hkv, T_b, d]`` for one sequence.

    Token j of the sequence lives in physical page ``table_row[j // P]`` at row ``j % P``.
    """
    Hkv, d = k_pages.shape[1], k_pages.shape[3]
    out = np.empty((Hkv, T_b, d), dtype=k_pages.dtype)
    for j0 in range(0, T_b, page_size):
        n = min(page_size, T_b - j0)
        p = int(table_row[j0 // page_size])
        out[:, j0:j0 + n, :] = k_pages[p, :, :n, :]
    return out


def score_row(qgroup: np.ndarray, K: np.ndarray) -> np.ndarray:
    """Scores of one KV head: ``qgroup [G, d]``, ``K [T, d]`` -> ``[T]`` (S1, S2)."""
    qgroup = np.asarray(qgroup, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    d = K.shape[-1]
    return (qgroup @ K.T).max(axis=0) / math.sqrt(d)


def score_keys(qpred: np.ndarray, keys, t_max: int) -> np.ndarray:
    """All scores: ``qpred [B, Hq, d]``; ``keys[b]`` is ``[Hkv, T_b, d]``.

    Returns ``[B, Hkv, t_max]`` float64 with ``-inf`` at ``j >= T_b``.
    """
    B, Hq, d = qpred.shape
    Hkv = keys[0].shape[0]
    G = Hq // Hkv
    out = np.full((B, Hkv, t_max), -np.inf)
    for b in range(B):
        T_b = keys[b].shape[1]
        for h in range(Hkv):
            out[b, h, :T_b] = score_row(qpred[b, h * G:(h + 1) * G], keys[b][h])
    return out


def select_row(scores: np.ndarray, T_b: int, C: int):
    """Top C of ``scores[:T_b]`` (T1-T5) -> (ascending int32 indices, count)."""
    s = np.asarray(scores[:T_b], dtype=np.float64)
    if np.isnan(s).any():
        raise ValueError("NaN score")
    n = min(C, T_b)
    order = np.lexsort((np.arange(T_b), -s))   # primary: larger score; then lower index
    chosen = np.sort(order[:n]).astype(np.int32)
    return chosen, n


def select_topk(scores: np.ndarray, seq_lens, C: int):
    """Per (b, KV head) selection: ``scores [B, Hkv, t_max]`` -> ``idx [B, Hkv, C]`` (-1 padded), ``count [B, Hkv]``."""
    B, Hkv, _ = scores.shape
    idx = np.full((B, Hkv, C), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv), dtype=np.int32)
    for b in range(B):
        for h in range(Hkv):
            chosen, n = select_row(scores[b, h], int(seq_lens[b]), C)
            idx[b, h, :n] = chosen
            cnt[b, h] = n
    return idx, cnt
