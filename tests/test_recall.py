"""Selection recall and temporal locality (the synthetic analogue of the pages'
selection-quality evidence): the host-side set arithmetic on CPU, and the sets the
library forms under each reading against the oracle's on the tiny workload (GPU)."""
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


def _tiny():
    import query_predicted_token_b200 as asp
    wl = synth.workload("tiny_f32_t512")
    kvd = synth.kv_cache(wl, "cuda")
    kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"])
    keys = [kvd["k"][b].double().cpu().numpy() for b in range(wl.batch)]
    return wl, kv, keys


@pytest.mark.gpu
def test_recall_report_matches_the_oracle_sets():
    from query_predicted_token_b200.recall import recall_report
    wl, kv, keys = _tiny()
    qhist, q_next = synth.query_history(wl, steps=2)
    q_t, q_true = q_next[0].cuda(), q_next[1].cuda()
    got = recall_report(kv, wl.C, q_true, {"current_query": q_t, "itself": q_true})
    assert got["itself"] == 1.0
    # the oracle's sets from its own float64 scores
    lens = [wl.t_max] * wl.batch
    s_cur = oracle.score_keys(q_t.double().cpu().numpy(), keys, wl.t_max)
    s_true = oracle.score_keys(q_true.double().cpu().numpy(), keys, wl.t_max)
    i_cur, c_cur = oracle.select_topk(s_cur, lens, wl.C)
    i_true, c_true = oracle.select_topk(s_true, lens, wl.C)
    ref = overlap(i_cur, c_cur, i_true, c_true).mean()
    # fp32 against float64 scores: a near-tie at either threshold may swap one token
    assert abs(got["current_query"] - ref) <= 2 / wl.C


def _oracle_sets(q, keys, wl, reading):
    """The oracle's top-C sets under an S2 reading: list over (b, h) (per_head: over (b, h, g))."""
    G = wl.n_q_heads // wl.n_kv_heads
    out = []
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            qg, K = q[b, h * G:(h + 1) * G], keys[b][h]
            if reading == "mean":
                out.append(oracle.select_row(oracle.score_row_mean(qg, K), K.shape[0], wl.C)[0])
            elif reading == "mass":
                out.append(oracle.select_row(oracle.score_row_mass(qg, K), K.shape[0], wl.C)[0])
            else:
                out.extend(oracle.select_per_head(qg, K, K.shape[0], wl.C))
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("reading", ["mean", "mass", "per_head"])
def test_sets_under_each_gqa_reading_match_the_oracle(reading):
    from query_predicted_token_b200.recall import topk_sets_reading
    wl, kv, keys = _tiny()
    q = synth.query_history(wl, steps=1)[1][0]
    idx, cnt = topk_sets_reading(q.cuda(), kv, wl.C, reading)
    ref = _oracle_sets(q.double().numpy(), keys, wl, reading)
    got = [idx[u][: int(cnt[u])] for u in np.ndindex(cnt.shape)]
    assert len(got) == len(ref)
    for g, r in zip(got, ref):
        # fp32 scores against float64: at most a swap at the threshold
        assert g.size == r.size and np.intersect1d(g, r).size >= r.size - 1


@pytest.mark.gpu
def test_window_overlap_matches_the_oracle():
    from query_predicted_token_b200.recall import window_overlap
    wl, kv, keys = _tiny()
    qhist, _ = synth.query_history(wl, steps=1)
    queries = [qhist[:, :, s] for s in range(qhist.shape[2])]
    got = window_overlap(kv, wl.C, [q.cuda() for q in queries])
    lens = [wl.t_max] * wl.batch
    sets = [oracle.select_topk(oracle.score_keys(q.double().numpy(), keys, wl.t_max), lens, wl.C) for q in queries]
    ref_mean, ref_union = [], []
    for b in range(wl.batch):
        for h in range(wl.n_kv_heads):
            per = [i[b, h, :c[b, h]] for i, c in sets]
            ref_mean.append(oracle.recent_window_overlap(per, "mean"))
            ref_union.append(oracle.recent_window_overlap(per, "union"))
    assert got["window"] == wl.W
    assert abs(got["mean"] - np.mean(ref_mean)) <= 2 / wl.C
    assert abs(got["union"] - np.mean(ref_union)) <= 2 / wl.C
