"""Pins for the oracle's next-query predictor (CPU only).

Each check below fixes the oracle against something other than its own code:
an SVD least-squares solve, planted exact-fit coefficients, closed forms of
special cases and invariants.  The mutant tests plant plausible mistakes in a
copy of the oracle's window prediction and show that a pin catches each one.
"""
import numpy as np
import pytest
from scipy.special import softmax as sp_softmax

from oracle import predict as P

RNG = np.random.default_rng(1234)


def _hist(W=16, d=128, rng=RNG):
    return rng.standard_normal((W + 1, d))


@pytest.mark.parametrize("w", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("lam", [1e-2, 1.0, 37.0])
def test_ridge_equals_augmented_least_squares(w, lam):
    # ridge == ordinary least squares on [X^T; sqrt(lam) I] a = [y; 0], solved by SVD (lstsq)
    X = RNG.standard_normal((w, 128))
    y = RNG.standard_normal(128)
    A = np.vstack([X.T, np.sqrt(lam) * np.eye(w)])
    rhs = np.concatenate([y, np.zeros(w)])
    ref = np.linalg.lstsq(A, rhs, rcond=None)[0]
    got = P.ridge_coefficients(X, y, lam)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-12)


def pin_exact_fit(window_fn, w=6, d=64, coef="raw", seed=7):
    """Plant coefficients a*: q_t = sum_i a*_i q_{t-w+i-1}; as lam -> 0 the fit recovers a*,
    and the prediction must apply a*_i (or its softmax) to q_{t-w+i}.  Returns the max error."""
    rng = np.random.default_rng(seed)
    W = w + 3
    hist = rng.standard_normal((W + 1, d))
    a_star = rng.uniform(-1.0, 1.5, size=w)
    lags = [hist[W - w + i - 1] for i in range(1, w + 1)]          # q_{t-w} .. q_{t-1}
    hist[W] = sum(a_star[i] * lags[i] for i in range(w))            # exact target
    weights = a_star if coef == "raw" else sp_softmax(a_star)
    nxt = [hist[W - w + i] for i in range(1, w + 1)]                # q_{t-w+1} .. q_t
    expect = sum(weights[i] * nxt[i] for i in range(w))
    got = window_fn(hist, w, 1e-13, coef)
    return float(np.max(np.abs(got - expect)) / np.max(np.abs(expect)))


@pytest.mark.parametrize("coef", ["raw", "softmax"])
@pytest.mark.parametrize("w", [2, 4, 6, 8])
def test_exact_fit_recovers_planted_coefficients(coef, w):
    assert pin_exact_fit(P.window_prediction, w=w, coef=coef) < 1e-7


def test_window_one_predicts_current_query():
    hist = _hist(W=8)
    got = P.window_prediction(hist, 1, 1e-2, "softmax")
    assert np.array_equal(got, hist[-1])        # softmax of one coefficient is exactly 1


def pin_identical_lags(window_fn, w=8, d=32):
    """All lags equal x, q_t = y: by symmetry a = c * 1, softmax is uniform, and the
    shifted window holds (w-1) copies of x plus y."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal(d)
    y = rng.standard_normal(d)
    hist = np.vstack([np.tile(x, (w + 2, 1)), y[None]])
    expect = ((w - 1) * x + y) / w
    got = window_fn(hist, w, 1e-2, "softmax")
    return float(np.max(np.abs(got - expect)))


@pytest.mark.parametrize("w", [2, 4, 8])
def test_identical_lags_give_shifted_window_mean(w):
    assert pin_identical_lags(P.window_prediction, w=w) < 1e-12


@pytest.mark.parametrize("w", [2, 4, 8])
def test_window_only_reads_its_last_w_plus_one_vectors(w):
    W = 16
    hist = _hist(W=W, d=64)
    base = P.window_prediction(hist, w, 1e-2)
    h2 = hist.copy()
    h2[: W - w] += 5.0                         # older than the window: no effect
    assert np.array_equal(P.window_prediction(h2, w, 1e-2), base)
    h3 = hist.copy()
    h3[W - w] += 0.5                           # the oldest lag of the window: must matter
    assert not np.allclose(P.window_prediction(h3, w, 1e-2), base)


def test_multi_window_pooling_is_the_mean_of_single_windows():
    hist = RNG.standard_normal((2, 3, 17, 64))
    both = P.predict_query(hist, (4, 8, 16), 1e-2)
    singles = [P.predict_query(hist, (w,), 1e-2) for w in (4, 8, 16)]
    assert np.allclose(both, sum(singles) / 3, rtol=1e-13, atol=1e-13)


def test_softmax_prediction_is_a_convex_combination():
    hist = RNG.standard_normal((17, 8))
    for w in (4, 8, 16):
        got = P.window_prediction(hist, w, 1e-2)
        win = hist[17 - w:]
        assert np.all(got <= win.max(axis=0) + 1e-12)
        assert np.all(got >= win.min(axis=0) - 1e-12)


def test_bad_window_rejected():
    with pytest.raises(ValueError):
        P.window_prediction(_hist(W=4), 5, 1e-2)


# ---- planted mistakes: each mutant must fail at least one pin ---------------------------

def _mutant_no_shift(hist, w, lam, coef="softmax"):
    W = hist.shape[0] - 1
    X, y = hist[W - w:W], hist[W]
    alpha = P.normalise_coefficients(P.ridge_coefficients(X, y, lam), coef)
    return alpha @ hist[W - w:W]                       # forgot the one-step shift


def _mutant_reversed(hist, w, lam, coef="softmax"):
    W = hist.shape[0] - 1
    X, y = hist[W - w:W], hist[W]
    alpha = P.normalise_coefficients(P.ridge_coefficients(X, y, lam), coef)
    return alpha[::-1] @ hist[W - w + 1:W + 1]         # coefficients applied newest-first


def _mutant_sum_normalised(hist, w, lam, coef="softmax"):
    W = hist.shape[0] - 1
    X, y = hist[W - w:W], hist[W]
    a = P.ridge_coefficients(X, y, lam)
    alpha = a if coef == "raw" else a / a.sum()         # sum-to-one instead of softmax
    return alpha @ hist[W - w + 1:W + 1]


@pytest.mark.parametrize("mutant", [_mutant_no_shift, _mutant_reversed, _mutant_sum_normalised])
def test_pins_catch_planted_mistakes(mutant):
    errs = [pin_exact_fit(mutant, coef="raw"), pin_exact_fit(mutant, coef="softmax"),
            pin_identical_lags(mutant)]
    assert max(errs) > 1e-3


def test_ridge_pin_catches_dropped_lambda():
    X = RNG.standard_normal((8, 128))
    y = RNG.standard_normal(128)
    lam = 5.0
    A = np.vstack([X.T, np.sqrt(lam) * np.eye(8)])
    ref = np.linalg.lstsq(A, np.concatenate([y, np.zeros(8)]), rcond=None)[0]
    bad = np.linalg.lstsq(X.T, y, rcond=None)[0]
    assert not np.allclose(bad, ref, rtol=1e-6)
