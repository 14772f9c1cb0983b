"""Pins of the oracle's alternative readings (oracle/readings.py), against facts
that do not come from the functions themselves: hand-computed values, cases that
reduce to the pinned plain readings, probabilities summing to one, exact recovery
of planted regression coefficients, hand-made set overlaps."""
import math

import numpy as np
import pytest

import oracle


def test_mean_score_hand_values_and_single_head():
    q = np.array([[1.0, 0.0, 2.0, 0.0], [3.0, 2.0, 0.0, 0.0]])       # mean (2, 1, 1, 0)
    K = np.array([[1.0, 1.0, 1.0, 1.0], [0.0, -1.0, 0.0, 4.0]])
    assert np.allclose(oracle.score_row_mean(q, K), [4.0 / 2.0, -1.0 / 2.0])
    rng = np.random.default_rng(0)
    q1, K1 = rng.standard_normal((1, 16)), rng.standard_normal((40, 16))
    assert np.allclose(oracle.score_row_mean(q1, K1), oracle.score_row(q1, K1))   # G = 1: the plain score


def test_mass_sums_to_the_group_size_and_two_token_closed_form():
    rng = np.random.default_rng(1)
    q, K = rng.standard_normal((4, 32)), rng.standard_normal((100, 32))
    m = oracle.score_row_mass(q, K)
    assert m.min() > 0 and abs(m.sum() - 4.0) < 1e-12      # each head's probabilities sum to one
    # one head, two tokens with logits a and b: e^a / (e^a + e^b) and e^b / (e^a + e^b)
    q2 = np.array([[2.0, 0.0, 0.0, 0.0]])
    K2 = np.array([[1.0, 0.0, 0.0, 0.0], [-1.0, 0.0, 0.0, 0.0]])
    a, b = 2.0 / 2.0, -2.0 / 2.0                           # / sqrt(4)
    assert np.allclose(oracle.score_row_mass(q2, K2), [math.exp(a) / (math.exp(a) + math.exp(b)),
                                                       math.exp(b) / (math.exp(a) + math.exp(b))])
    # one head: the mass ranks tokens as the plain score does, so the top-C sets agree
    q1 = q[:1]
    s_plain, s_mass = oracle.score_row(q1, K), oracle.score_row_mass(q1, K)
    assert np.array_equal(oracle.select_row(s_plain, 100, 17)[0], oracle.select_row(s_mass, 100, 17)[0])


def test_per_head_selection_reduces_to_the_plain_selection():
    rng = np.random.default_rng(2)
    q, K = rng.standard_normal((3, 8)), rng.standard_normal((50, 8))
    sets = oracle.select_per_head(q, K, 45, 10)
    assert len(sets) == 3
    for g in range(3):
        want = oracle.select_row(oracle.score_row(q[g:g + 1], K[:45]), 45, 10)[0]
        assert np.array_equal(sets[g], want)
        assert sets[g].max() < 45 and sets[g].size == 10


def test_pooled_features_hand_values():
    hist = np.array([[1.0, 0.0], [3.0, 2.0], [5.0, 4.0], [7.0, 6.0]])   # q_{t-3} .. q_t
    f = oracle.pooled_features(hist, [1, 2, 3], 3)
    assert np.allclose(f, [[7.0, 6.0], [6.0, 5.0], [5.0, 4.0]])
    f_prev = oracle.pooled_features(hist, [1, 2, 3], 2)                 # one step back
    assert np.allclose(f_prev, [[5.0, 4.0], [4.0, 3.0], [3.0, 2.0]])


def test_pooled_regression_recovers_planted_coefficients():
    """With q_t built exactly as sum_w beta_w f_w(t-1) and lambda -> 0, the raw
    coefficients are beta and the prediction applies them to the features one step
    later: a dropped or misplaced shift fails this."""
    rng = np.random.default_rng(3)
    W, d, windows = 16, 64, [4, 8, 16]
    hist = rng.standard_normal((W + 1, d))
    beta = np.array([0.7, -0.2, 0.4])
    hist[W] = beta @ oracle.pooled_features(hist, windows, W - 1)
    got = oracle.pooled_prediction(hist, windows, 1e-12, coef="raw")
    assert np.allclose(got, beta @ oracle.pooled_features(hist, windows, W), atol=1e-8)
    # softmax weights are a convex combination of the one-step-later features
    w = np.exp(beta - beta.max())
    soft = oracle.pooled_prediction(hist, windows, 1e-12)
    assert np.allclose(soft, (w / w.sum()) @ oracle.pooled_features(hist, windows, W), atol=1e-8)


def test_pooled_prediction_special_cases():
    rng = np.random.default_rng(4)
    hist = rng.standard_normal((9, 32))
    assert np.allclose(oracle.pooled_prediction(hist, [1], 1e-2), hist[8])    # one window of one: q_t
    const = np.tile(rng.standard_normal(32), (9, 1))
    assert np.allclose(oracle.pooled_prediction(const, [2, 4, 8], 1e-2), const[0])
    batched = oracle.predict_query_pooled(np.stack([hist, const]), [2, 4, 8], 1e-2)
    assert np.allclose(batched[1], const[0]) and batched.shape == (2, 32)
    with pytest.raises(ValueError):
        oracle.pooled_prediction(hist, [9], 1e-2)


def test_recent_window_overlap_hand_values():
    sets = [[1, 2, 3, 4], [3, 4, 5, 6], [1, 5, 7, 8]]      # S_{t-2}, S_{t-1}, S_t
    # mean over the two earlier sets of |S_t & S_s| / |S_t|: (1/4 + 1/4) / 2
    assert oracle.recent_window_overlap(sets, "mean") == 0.25
    # union of the earlier sets holds 1 and 5
    assert oracle.recent_window_overlap(sets, "union") == 0.5
    assert oracle.recent_window_overlap([[1, 2], [1, 2]]) == 1.0
    assert oracle.recent_window_overlap([[1, 2], [3, 4]]) == 0.0
    rng = np.random.default_rng(5)
    rnd = [rng.choice(100, 20, replace=False) for _ in range(17)]
    assert oracle.recent_window_overlap(rnd, "union") >= oracle.recent_window_overlap(rnd, "mean")
