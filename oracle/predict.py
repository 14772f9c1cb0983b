"""Oracle step 1: the temporal-regressive next-query predictor (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU arms may use this.

What the pages say: a light-weight temporal-regressive module predicts the
next query state from the few most recent queries (abstract, component (1));
the fit is a ridge regression whose coefficients are normalised by a softmax,
pooled by averaging over several window lengths (summary, "Approach"); the
reproduction fits it one step ahead on a window of the last 16 queries (repro
card, claim C5).  No equation is printed, so the steps below are this reading:

R1  one regression per query head; the samples are the d channels and the
    features are the w lagged query vectors of that head.
R2  the history holds W+1 vectors q_{t-W} .. q_t (oldest first).  For a
    window w the lag matrix X_w has rows q_{t-w} .. q_{t-1} (row i, i=1..w, is
    q_{t-w+i-1}) and the target is y = q_t.  Ridge:
        a_w = argmin_a ||X_w^T a - y||^2 + lam ||a||^2
            = (X_w X_w^T + lam I)^{-1} X_w y          (a w x w SPD system).
    The one-step-ahead prediction applies coefficient i to the vector one step
    later:  qhat^(w) = sum_i alpha_{w,i} q_{t-w+i}.
R3  softmax normalisation: alpha_w = softmax(a_w) over the w coefficients
    (temperature 1).  The raw coefficients (alpha = a) are kept as a switch.
R4  lam is added to the diagonal unscaled.
R5  multi-window average pooling: qhat = mean over the windows in Omega of
    qhat^(w).

Pins (tests/test_oracle_predict.py): the ridge solve against an augmented
least-squares problem solved by SVD; exact-fit recovery of planted
coefficients as lam -> 0 (pins which lag gets which coefficient); the w=1 case
(qhat = q_t); identical lags (uniform weights over the shifted window, which
pins the one-step shift); locality (older vectors do not matter); pooling
linearity.  R3 and R5 as readings of the paper are parity unpinned: the pages
print no number that fixes them.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import cho_factor, cho_solve


def ridge_coefficients(X: np.ndarray, y: np.ndarray, lam: float) -> np.ndarray:
    """Ridge coefficients ``a`` for lag matrix ``X [w, d]`` and target ``y [d]`` (R2, R4).

    Normal equations ``(X X^T + lam I) a = X y`` solved by Cholesky.
    """
    X = np.asarray(X, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    w = X.shape[0]
    A = X @ X.T + lam * np.eye(w)
    return cho_solve(cho_factor(A, lower=True), X @ y)


def normalise_coefficients(a: np.ndarray, coef: str = "softmax") -> np.ndarray:
    """R3: softmax over the window's coefficients (``coef="raw"`` keeps them)."""
    a = np.asarray(a, dtype=np.float64)
    if coef == "raw":
        return a
    if coef != "softmax":
        raise ValueError(coef)
    e = np.exp(a - a.max())
    return e / e.sum()


def window_prediction(hist: np.ndarray, w: int, lam: float, coef: str = "softmax") -> np.ndarray:
    """qhat^(w) for one head: ``hist [W+1, d]`` oldest first (R2, R3)."""
    hist = np.asarray(hist, dtype=np.float64)
    W = hist.shape[0] - 1
    if not 1 <= w <= W:
        raise ValueError(f"window {w} outside [1, {W}]")
    X = hist[W - w:W]          # q_{t-w} .. q_{t-1}
    y = hist[W]                # q_t
    alpha = normalise_coefficients(ridge_coefficients(X, y, lam), coef)
    shifted = hist[W - w + 1:W + 1]   # q_{t-w+1} .. q_t
    return alpha @ shifted


def predict_query(qhist: np.ndarray, windows, lam: float, coef: str = "softmax") -> np.ndarray:
    """Predicted next query for every head.

    ``qhist [..., W+1, d]`` (oldest first) -> ``qpred [..., d]`` float64:
    the mean over ``windows`` of the per-window predictions (R5).
    """
    qhist = np.asarray(qhist, dtype=np.float64)
    lead = qhist.shape[:-2]
    flat = qhist.reshape((-1,) + qhist.shape[-2:])
    out = np.zeros((flat.shape[0], flat.shape[-1]))
    for n in range(flat.shape[0]):
        acc = np.zeros(flat.shape[-1])
        for w in windows:
            acc += window_prediction(flat[n], int(w), lam, coef)
        out[n] = acc / len(windows)
    return out.reshape(lead + (flat.shape[-1],))
