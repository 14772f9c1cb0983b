"""Pins for the oracle's page-level comparison path and the decode-FLOPs model (CPU only)."""
import math
import os

import numpy as np
import pytest

from oracle import quest as Q
from oracle import flops as F
from oracle import pipeline, scan, attend, predict

RNG = np.random.default_rng(21)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "flops_claims.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        out[key] = [float(v) for v in vals]
    return out


def test_page_bound_dominates_every_logit_of_its_page():
    T, d, P, G = 101, 32, 16, 4
    K = RNG.standard_normal((T, d))
    q = RNG.standard_normal((G, d))
    kmin, kmax = Q.quest_meta(K, P)
    ub = Q.quest_page_scores(q, kmin, kmax)
    exact = (q @ K.T).max(axis=0) / math.sqrt(d)
    for p in range(len(ub)):
        assert ub[p] >= exact[p * P:(p + 1) * P].max() - 1e-12


def test_page_of_identical_keys_is_exact():
    d, P = 16, 16
    k = RNG.standard_normal(d)
    K = np.tile(k, (P, 1))
    q = RNG.standard_normal((3, d))
    kmin, kmax = Q.quest_meta(K, P)
    assert np.allclose(Q.quest_page_scores(q, kmin, kmax), [(q @ k).max() / 4.0], atol=1e-13)


def test_page_selection_ties_and_ragged_tail():
    s = np.array([1.0, 3.0, 3.0, 0.0, 3.0])
    toks, n = Q.quest_select_row(s, T_b=70, C=32, page_size=16)      # keep 2 pages: 1 and 2
    assert toks.tolist() == list(range(16, 48)) and n == 32
    toks, n = Q.quest_select_row(s, T_b=70, C=33, page_size=16)      # keep 3 pages: 1, 2, 4 (ragged)
    assert toks.tolist() == list(range(16, 48)) + list(range(64, 70)) and n == 38


def test_flops_model_reproduces_printed_claims():
    g = _golden()
    r = F.decode_flops(**F.QWEN3_8B, T=32768, C=2048, page=int(g["page_size"][0]))
    dec = int(g["reduction_printed_decimals"][0])
    assert round(100 * r["reduction"], dec) == g["reduction_qwen3_8b_T32768_C2048_percent"][0]
    lo, hi = g["page_gap_C2048_min_percent"][0], g["page_gap_C2048_max_percent"][0]
    gaps = [F.decode_flops(**F.QWEN3_8B, T=int(T), C=2048)["page_gap"] for T in g["page_gap_contexts"]]
    assert all(lo <= round(100 * x) <= hi for x in gaps)
    assert round(100 * gaps[0]) == lo and round(100 * gaps[-1]) == hi     # the range's two ends


def test_flops_pin_catches_dropped_mlp_term():
    cfg = dict(F.QWEN3_8B)
    cfg["inter"] = 0                      # a model without the MLP term gives a different reduction
    r = F.decode_flops(**cfg, T=32768, C=2048)
    assert round(100 * r["reduction"], 1) != 54.5


def test_pipeline_step_composes_the_four_steps():
    B, Hq, Hkv, d, T, W, C = 1, 4, 2, 16, 40, 4, 8
    keys = [RNG.standard_normal((Hkv, T, d))]
    vals = [RNG.standard_normal((Hkv, T, d))]
    qhist = RNG.standard_normal((B, Hq, W + 1, d))
    q_t = RNG.standard_normal((B, Hq, d))
    idx, cnt = scan.select_topk(RNG.standard_normal((B, Hkv, T)), [T], C)
    r = pipeline.decode_step(q_t, qhist, keys, vals, idx, cnt, C, (2, 4), 1e-2, T)
    hist = np.concatenate([qhist[:, :, 1:], q_t[:, :, None]], axis=2)
    assert np.array_equal(r["qhist"][:, :, -1], q_t)
    qp = predict.predict_query(hist, (2, 4), 1e-2)
    assert np.allclose(r["qpred"], qp)
    sc = scan.score_keys(qp, keys, T).astype(np.float32)
    assert np.array_equal(r["scores"], sc)
    o, _ = attend.sparse_attend(q_t, keys, vals, idx, cnt)
    assert np.allclose(r["out"], o)
