"""Oracle of one asynchronous decode step (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU arms may use this.

The abstract (component (2)) decouples KV selection from the decoding loop:
while step t attends over the tokens chosen for it, the selection for step
t+1 is made from a *predicted* query.  One step of that schedule, as a plain
sequence:

    out_t        = attend(q_t, idx_t)                    (attend.py, A1-A3)
    history      <- drop oldest, append q_t              (W+1 vectors kept)
    qhat_{t+1}   = predict(history)                      (predict.py, R1-R5)
    scores       = score(qhat_{t+1}, K)                  (scan.py, S1-S2)
    idx_{t+1}    = top-C(scores)                         (scan.py, T1-T5)

Scores are rounded to float32 before selection, the precision in which the
CUDA path takes the same decision.
"""
from __future__ import annotations

import numpy as np

from .attend import sparse_attend
from .predict import predict_query
from .scan import score_keys, select_topk


def decode_step(q_t, qhist, keys, values, idx_cur, cnt_cur, C, windows, lam, t_max,
                coef="softmax", tail_begin=None, q_hist_value=None):
    """One step.  ``q_t [B, Hq, d]``; ``qhist [B, Hq, W+1, d]`` oldest first.

    ``q_hist_value`` is the value pushed into the history (defaults to q_t).
    Returns dict(out, lse, qhist, qpred, scores, idx, count).
    """
    q_t = np.asarray(q_t, dtype=np.float64)
    out, lse = sparse_attend(q_t, keys, values, idx_cur, cnt_cur, tail_begin)
    push = q_t if q_hist_value is None else np.asarray(q_hist_value, dtype=np.float64)
    hist = np.concatenate([np.asarray(qhist, dtype=np.float64)[:, :, 1:], push[:, :, None]], axis=2)
    qpred = predict_query(hist, windows, lam, coef)
    scores = score_keys(qpred, keys, t_max).astype(np.float32)
    seq_lens = [k.shape[1] for k in keys]
    idx, cnt = select_topk(scores, seq_lens, C)
    return dict(out=out, lse=lse, qhist=hist, qpred=qpred, scores=scores, idx=idx, count=cnt)
