"""Pins for the oracle's key scoring and top-C selection (CPU only)."""
import math

import numpy as np
import pytest

from oracle import scan as S
from synth import score_rows

RNG = np.random.default_rng(99)


def test_scores_hand_computed():
    # d = 4 (scale 1/2), G = 2: q0 = e0, q1 = 2 e1
    q = np.array([[1.0, 0, 0, 0], [0, 2.0, 0, 0]])
    K = np.array([[1.0, 1, 0, 0],       # dots (1, 2)   -> max 2  -> 1.0
                  [-1.0, -1, 0, 0],     # dots (-1, -2) -> max -1 -> -0.5
                  [3.0, -1, 1, 1]])     # dots (3, -2)  -> max 3  -> 1.5
    assert np.array_equal(S.score_row(q, K), np.array([1.0, -0.5, 1.5]))


def _brute_scores(qpred, keys, t_max):
    B, Hq, d = qpred.shape
    Hkv = keys[0].shape[0]
    G = Hq // Hkv
    out = np.full((B, Hkv, t_max), -np.inf)
    for b in range(B):
        for h in range(Hkv):
            for j in range(keys[b].shape[1]):
                best = -np.inf
                for g in range(G):
                    acc = 0.0
                    for c in range(d):
                        acc += float(qpred[b, h * G + g, c]) * float(keys[b][h, j, c])
                    best = max(best, acc)
                out[b, h, j] = best / math.sqrt(d)
    return out


def test_scores_match_loop_brute_force_ragged():
    B, Hq, Hkv, d, t_max = 2, 6, 2, 8, 13
    q = RNG.standard_normal((B, Hq, d))
    keys = [RNG.standard_normal((Hkv, 13, d)), RNG.standard_normal((Hkv, 7, d))]
    got = S.score_keys(q, keys, t_max)
    ref = _brute_scores(q, keys, t_max)
    assert np.array_equal(np.isinf(got), np.isinf(ref))
    fin = np.isfinite(ref)
    assert np.allclose(got[fin], ref[fin], rtol=1e-12, atol=1e-12)
    assert np.all(got[1, :, 7:] == -np.inf)


def test_scores_invariant_to_head_order_within_group():
    q = RNG.standard_normal((4, 16))
    K = RNG.standard_normal((40, 16))
    assert np.allclose(S.score_row(q, K), S.score_row(q[::-1], K), rtol=0, atol=1e-14)


def test_group_of_one_is_plain_scaled_dot():
    q = RNG.standard_normal((1, 64))
    K = RNG.standard_normal((50, 64))
    assert np.allclose(S.score_row(q, K), np.array([np.dot(q[0], k) for k in K]) / 8.0, atol=1e-13)


def test_gather_sequence_walks_the_page_table():
    P, Hkv, d = 4, 2, 3
    pages = RNG.standard_normal((5, Hkv, P, d))
    table = np.array([3, 0, 4, -1])
    seq = S.gather_sequence(pages, table, 10, P)
    for j in range(10):
        assert np.array_equal(seq[:, j], pages[table[j // P], :, j % P])


def _definition_select(s, T_b, C):
    """j is chosen iff #{i: s_i > s_j} + #{i < j: s_i == s_j} < C (pure Python)."""
    vals = [float(x) for x in s[:T_b]]
    chosen = []
    for j in range(T_b):
        rank = sum(1 for i in range(T_b) if vals[i] > vals[j]) + sum(1 for i in range(j) if vals[i] == vals[j])
        if rank < C:
            chosen.append(j)
    return chosen


@pytest.mark.parametrize("kind", ["normal", "ties", "special", "equal"])
@pytest.mark.parametrize("T_b,C", [(1, 1), (5, 8), (37, 5), (64, 64), (64, 17), (90, 31)])
def test_selection_matches_definition(kind, T_b, C):
    rows = score_rows(3, 96, seed=T_b * 100 + C, kind=kind).numpy()
    for r in range(rows.shape[0]):
        got, n = S.select_row(rows[r], T_b, C)
        ref = _definition_select(rows[r], T_b, C)
        assert n == min(C, T_b) == len(ref)
        assert got.tolist() == ref


def test_selection_tie_break_and_signed_zero():
    s = np.array([0.0, -0.0, 1.0, -0.0, 0.0], dtype=np.float32)
    got, _ = S.select_row(s, 5, 3)
    assert got.tolist() == [0, 1, 2]          # -0.0 ties +0.0; lowest indices win


def test_selection_pads_and_ignores_tokens_past_length():
    s = np.array([[[5.0, 4.0, 3.0, 9.0, 9.0, 9.0]]], dtype=np.float32)
    idx, cnt = S.select_topk(s, [3], 4)
    assert cnt.tolist() == [[3]]
    assert idx.tolist() == [[[0, 1, 2, -1]]]


def test_selection_rejects_nan():
    with pytest.raises(ValueError):
        S.select_row(np.array([1.0, np.nan], dtype=np.float32), 2, 1)


def test_selection_pin_catches_highest_index_tie_break():
    s = np.array([1.0, 2.0, 2.0, 2.0, 0.5], dtype=np.float32)
    order = np.lexsort((-np.arange(5), -s.astype(np.float64)))   # planted: highest index first
    mutant = sorted(order[:2].tolist())
    assert mutant != _definition_select(s, 5, 2)
    assert S.select_row(s, 5, 2)[0].tolist() == _definition_select(s, 5, 2)
