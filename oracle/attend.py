"""Oracle step 4: single-token attention over the selected K/V only (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU arms may use this.

Pages: the prediction only decides *which* tokens are attended; the decode
step itself attends over the selected tokens, the same set a page-level
method would attend at the same budget (repro card, "Key finding ..."), and
the query-aware sparsity no longer waits inside the decoding loop (abstract).
Readings:

A1  the attention uses the true current query q_t, not the prediction.
A2  tokens appended after the selection snapshot, [tail_begin, T_b), are
    always attended in addition to the selected set (a consequence of the
    selection running one step ahead; the pages do not discuss it).
A3  logits q . k_j / sqrt(d), softmax over the attended set, output
    sum_j p_j v_j; lse = log sum_j exp(logit_j) (natural log).  An empty set
    (an empty sum) gives output 0 and lse = -inf.

Pins (tests/test_oracle_attend.py): with every token selected the result is
dense attention, checked against torch's scaled_dot_product_attention run in
float64 on the CPU; a two-token case in closed form; invariance to the order
and duplication of indices; the output is a convex combination of the
attended V rows.
"""
from __future__ import annotations

import math

import numpy as np


def attend_set(q: np.ndarray, K: np.ndarray, V: np.ndarray, S: np.ndarray):
    """``q [G, d]``, ``K, V [T, d]``, attended token set ``S`` -> (``o [G, d]``, ``lse [G]``)."""
    q = np.asarray(q, dtype=np.float64)
    S = np.unique(np.asarray(S, dtype=np.int64))
    if S.size == 0:
        return np.zeros_like(q), np.full(q.shape[0], -np.inf)
    Ks = np.asarray(K[S], dtype=np.float64)
    Vs = np.asarray(V[S], dtype=np.float64)
    logits = q @ Ks.T / math.sqrt(q.shape[-1])          # [G, |S|]
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    z = e.sum(axis=1, keepdims=True)
    o = (e / z) @ Vs
    lse = (m + np.log(z))[:, 0]
    return o, lse


def attended_set(idx_row, count: int, tail_begin, T_b: int) -> np.ndarray:
    """The tokens one KV head attends: the selected ones plus the tail (A2)."""
    sel = np.asarray(idx_row[:count], dtype=np.int64)
    tail = np.arange(T_b if tail_begin is None else int(tail_begin), T_b, dtype=np.int64)
    return np.union1d(sel, tail)


def sparse_attend(q: np.ndarray, keys, values, idx: np.ndarray, count: np.ndarray, tail_begin=None):
    """``q [B, Hq, d]``; ``keys[b], values[b]`` are ``[Hkv, T_b, d]``; ``idx [B, Hkv, C]``.

    Returns ``out [B, Hq, d]`` and ``lse [B, Hq]`` (float64).
    """
    B, Hq, d = q.shape
    Hkv = keys[0].shape[0]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        T_b = keys[b].shape[1]
        tb = None if tail_begin is None else tail_begin[b]
        for h in range(Hkv):
            S = attended_set(idx[b, h], int(count[b, h]), tb, T_b)
            o, l = attend_set(q[b, h * G:(h + 1) * G], keys[b][h], values[b][h], S)
            out[b, h * G:(h + 1) * G] = o
            lse[b, h * G:(h + 1) * G] = l
    return out, lse
