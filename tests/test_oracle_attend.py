"""Pins for the oracle's sparse attention (CPU only)."""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import attend as A

RNG = np.random.default_rng(5)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_all_selected_equals_dense_attention(G):
    # library routine: torch's SDPA in float64 on the CPU, one query per head
    B, Hkv, T, d = 2, 2, 37, 16
    Hq = Hkv * G
    q = RNG.standard_normal((B, Hq, d))
    keys = [RNG.standard_normal((Hkv, T, d)) for _ in range(B)]
    vals = [RNG.standard_normal((Hkv, T, d)) for _ in range(B)]
    idx = np.tile(np.arange(T, dtype=np.int32), (B, Hkv, 1))
    cnt = np.full((B, Hkv), T, dtype=np.int32)
    out, lse = A.sparse_attend(q, keys, vals, idx, cnt)
    Kt = torch.from_numpy(np.stack(keys)).repeat_interleave(G, dim=1)      # [B, Hq, T, d]
    Vt = torch.from_numpy(np.stack(vals)).repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q)[:, :, None, :], Kt, Vt)[:, :, 0, :]
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    logits = np.einsum("bhd,bhtd->bht", q, Kt.numpy()) / math.sqrt(d)
    assert np.allclose(lse, logsumexp(logits, axis=-1), rtol=1e-12, atol=1e-12)


def test_two_tokens_closed_form():
    q = np.array([[2.0, 0.0, 0.0, 0.0]])          # d = 4, scale 1/2
    K = np.array([[1.0, 0, 0, 0], [0.0, 0, 0, 0]])  # logits 1 and 0
    V = np.array([[1.0, 2, 3, 4], [-1.0, 0, 0, 1]])
    o, lse = A.attend_set(q, K, V, np.array([0, 1]))
    p0 = 1.0 / (1.0 + math.exp(-1.0))
    assert np.allclose(o[0], p0 * V[0] + (1 - p0) * V[1], rtol=1e-14, atol=1e-14)
    assert math.isclose(lse[0], math.log(math.e + 1.0), rel_tol=1e-14)


def test_single_token_returns_its_value():
    q = RNG.standard_normal((3, 8))
    K = RNG.standard_normal((10, 8))
    V = RNG.standard_normal((10, 8))
    o, _ = A.attend_set(q, K, V, np.array([7]))
    assert np.allclose(o, np.tile(V[7], (3, 1)), rtol=0, atol=0)


def test_order_and_duplicates_do_not_matter():
    q = RNG.standard_normal((2, 8))
    K = RNG.standard_normal((30, 8))
    V = RNG.standard_normal((30, 8))
    a, la = A.attend_set(q, K, V, np.array([3, 9, 21, 4]))
    b, lb = A.attend_set(q, K, V, np.array([21, 4, 4, 3, 9, 9]))
    assert np.allclose(a, b, atol=1e-15) and np.allclose(la, lb, atol=1e-15)


def test_output_is_convex_combination_of_attended_values():
    q = RNG.standard_normal((4, 16)) * 3
    K = RNG.standard_normal((64, 16))
    V = RNG.standard_normal((64, 16))
    S = np.array([1, 5, 8, 40, 63])
    o, _ = A.attend_set(q, K, V, S)
    assert np.all(o <= V[S].max(axis=0) + 1e-12) and np.all(o >= V[S].min(axis=0) - 1e-12)


def test_tail_tokens_are_added_to_the_selection():
    B, Hkv, G, T, d = 1, 1, 2, 20, 8
    q = RNG.standard_normal((B, Hkv * G, d))
    keys = [RNG.standard_normal((Hkv, T, d))]
    vals = [RNG.standard_normal((Hkv, T, d))]
    idx = np.array([[[2, 5, 17, -1]]], dtype=np.int32)
    cnt = np.array([[3]], dtype=np.int32)
    out, _ = A.sparse_attend(q, keys, vals, idx, cnt, tail_begin=[16])
    ref, _ = A.attend_set(q[0], keys[0][0], vals[0][0], np.array([2, 5, 16, 17, 18, 19]))
    assert np.allclose(out[0], ref, rtol=1e-14, atol=1e-14)


def test_empty_set_is_an_empty_sum():
    q = RNG.standard_normal((2, 8))
    o, lse = A.attend_set(q, RNG.standard_normal((5, 8)), RNG.standard_normal((5, 8)), np.array([], dtype=np.int64))
    assert np.array_equal(o, np.zeros((2, 8))) and np.all(lse == -np.inf)
