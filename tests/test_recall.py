"""Selection recall (the synthetic analogue of the pages' selection-quality evidence)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from query_predicted_token_b200.recall import overlap


def test_overlap_counts_shared_indices_over_the_reference_set():
    a = np.array([[[1, 3, 5, 7], [0, 2, -1, -1]]])
    ca = np.array([[4, 2]])
    b = np.array([[[3, 4, 5, 9], [2, 5, 8, -1]]])
    cb = np.array([[4, 3]])
    got = overlap(a, ca, b, cb)
    assert got.shape == (1, 2)
    assert got[0, 0] == 2 / 4          # {3, 5}
    assert got[0, 1] == 1 / 3          # {2}; a's padding is not counted
    assert overlap(a, ca, a, ca).tolist() == [[1.0, 1.0]]
    assert overlap(a, ca, b, np.array([[0, 0]])).tolist() == [[1.0, 1.0]]   # empty reference set


@pytest.mark.gpu
def test_recall_report_matches_the_oracle_sets():
    import query_predicted_token_b200 as asp
    from query_predicted_token_b200.recall import recall_report
    wl = synth.workload("tiny_f32_t512")
    kvd = synth.kv_cache(wl, "cuda")
    kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"])
    qhist, q_next = synth.query_history(wl, steps=2)
    q_t, q_true = q_next[0].cuda(), q_next[1].cuda()
    got = recall_report(kv, wl.C, q_true, {"current_query": q_t, "itself": q_true})
    assert got["itself"] == 1.0
    # the oracle's sets from its own float64 scores
    keys = [kvd["k"][b].double().cpu().numpy() for b in range(wl.batch)]
    lens = [wl.t_max] * wl.batch
    s_cur = oracle.score_keys(q_t.double().cpu().numpy(), keys, wl.t_max)
    s_true = oracle.score_keys(q_true.double().cpu().numpy(), keys, wl.t_max)
    i_cur, c_cur = oracle.select_topk(s_cur, lens, wl.C)
    i_true, c_true = oracle.select_topk(s_true, lens, wl.C)
    ref = overlap(i_cur, c_cur, i_true, c_true).mean()
    # fp32 against float64 scores: a near-tie at either threshold may swap one token
    assert abs(got["current_query"] - ref) <= 2 / wl.C
