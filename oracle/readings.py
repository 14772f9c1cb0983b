"""Oracle of the readings the pages leave open, beside the chosen ones (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU arms may use this.

The pages name the method's parts without printing them (no equation, no
code), so several steps have more than one plain reading.  The chosen readings
live in predict.py (R1-R5) and scan.py (S1-S2); this module states the
recorded alternatives, so that what each reading does to the selection can be
measured, and the mechanism measurement the pages report beside the
prediction:

S2-mean       one score per KV head from the mean of its group's queries:
              s_j = (mean_g q_g) . k_j / sqrt(d).
S2-mass       the sum over the group of each head's attention probabilities:
              s_j = sum_g softmax_j(q_g . k_j / sqrt(d)), the softmax over the
              head's candidate tokens j < T_b.
S2-per-head   every query head keeps its own top C (the union is gathered).
R5-pooled     "multi-window average pooling" read as pooling first: each
              window w in Omega gives the feature f_w(s) = mean(q_{s-w+1} .. q_s);
              one ridge regression per head fits q_t on the features at s = t-1,
              beta = (F F^T + lam I)^-1 F q_t (F: |Omega| x d), the coefficients
              are softmax-normalised (R3) and the prediction applies them to the
              features one step later: qhat = sum_w beta_w f_w(t).
Overlap       temporal locality of the selection (the reproduction card's
              claim C5, "recent-16-window overlap", the paper's Fig. 4): for the
              sets S_{t-W} .. S_t chosen with the true queries of W+1 successive
              steps, the mean over the W earlier steps s of |S_t & S_s| / |S_t|
              (reading "mean"), or |S_t & (S_{t-W} u .. u S_{t-1})| / |S_t|
              (reading "union").

Pins (tests/test_oracle_readings.py): hand-computed scores; G = 1, where the
mean and the per-head readings reduce to the pinned plain score; the
probabilities of each head summing to one over its tokens; the two-token
closed form of the mass; the pooled regression's exact recovery of planted
coefficients (which pins the features' one-step shift), a window of one (the
current query) and a constant history; hand-made overlaps and the union
bounding the mean.  As readings of the paper they are parity unpinned, like
S2 and R5 themselves.
"""
from __future__ import annotations

import math

import numpy as np

from .predict import normalise_coefficients, ridge_coefficients
from .scan import select_row


def score_row_mean(qgroup: np.ndarray, K: np.ndarray) -> np.ndarray:
    """S2-mean: ``qgroup [G, d]``, ``K [T, d]`` -> ``[T]``."""
    qgroup = np.asarray(qgroup, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    return K @ qgroup.mean(axis=0) / math.sqrt(K.shape[-1])


def score_row_mass(qgroup: np.ndarray, K: np.ndarray) -> np.ndarray:
    """S2-mass: ``qgroup [G, d]``, ``K [T, d]`` (the head's candidate tokens) -> ``[T]``."""
    qgroup = np.asarray(qgroup, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    logits = qgroup @ K.T / math.sqrt(K.shape[-1])       # [G, T]
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    return (e / e.sum(axis=1, keepdims=True)).sum(axis=0)


def select_per_head(qgroup: np.ndarray, K: np.ndarray, T_b: int, C: int):
    """S2-per-head: each query head's own top C of ``K[:T_b]`` -> list of G ascending index arrays."""
    qgroup = np.asarray(qgroup, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    out = []
    for g in range(qgroup.shape[0]):
        s = K[:T_b] @ qgroup[g] / math.sqrt(K.shape[-1])
        out.append(select_row(s, T_b, C)[0])
    return out


def pooled_features(hist: np.ndarray, windows, s: int) -> np.ndarray:
    """``[len(windows), d]``: row i is the mean of the ``windows[i]`` vectors ending at
    index ``s`` of ``hist [W+1, d]`` (oldest first)."""
    hist = np.asarray(hist, dtype=np.float64)
    return np.stack([hist[s - w + 1:s + 1].mean(axis=0) for w in windows])


def pooled_prediction(hist: np.ndarray, windows, lam: float, coef: str = "softmax") -> np.ndarray:
    """R5-pooled for one head: ``hist [W+1, d]`` oldest first -> ``qhat [d]``."""
    hist = np.asarray(hist, dtype=np.float64)
    W = hist.shape[0] - 1
    windows = [int(w) for w in windows]
    if not all(1 <= w <= W for w in windows):
        raise ValueError(f"windows {windows} outside [1, {W}]")
    F = pooled_features(hist, windows, W - 1)      # the features one step back
    beta = normalise_coefficients(ridge_coefficients(F, hist[W], lam), coef)
    return beta @ pooled_features(hist, windows, W)


def predict_query_pooled(qhist: np.ndarray, windows, lam: float, coef: str = "softmax") -> np.ndarray:
    """R5-pooled for every head: ``qhist [..., W+1, d]`` -> ``[..., d]`` float64."""
    qhist = np.asarray(qhist, dtype=np.float64)
    lead = qhist.shape[:-2]
    flat = qhist.reshape((-1,) + qhist.shape[-2:])
    out = np.stack([pooled_prediction(h, windows, lam, coef) for h in flat])
    return out.reshape(lead + (qhist.shape[-1],))


def set_overlap(a, b) -> float:
    """``|a & b| / |b|`` of two index sets (1.0 for an empty ``b``)."""
    a = np.unique(np.asarray(a, dtype=np.int64))
    b = np.unique(np.asarray(b, dtype=np.int64))
    return 1.0 if b.size == 0 else np.intersect1d(a, b).size / b.size


def recent_window_overlap(sets, reading: str = "mean") -> float:
    """Overlap of the last of ``sets`` (S_{t-W} .. S_t, oldest first) with the earlier ones."""
    *earlier, last = [np.asarray(s, dtype=np.int64) for s in sets]
    if not earlier:
        raise ValueError("need at least two sets")
    if reading == "mean":
        return float(np.mean([set_overlap(s, last) for s in earlier]))
    if reading == "union":
        return set_overlap(np.concatenate(earlier), last)
    raise ValueError(reading)
