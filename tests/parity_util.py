"""Shared helpers of the GPU parity tests: tolerance rules and host copies.

Tolerances (stated once, used everywhere):
  * predicted query:  ||qhat_gpu - qhat_ref|| <= 1e-4 ||qhat_ref|| per head (fp32 I/O);
  * scores:           |s - s_ref| <= 1e-3 |s_ref| + 1e-6 max_g||q_g|| ||k_j|| / sqrt(d)
                      (the absolute floor covers scores near zero, where a purely
                      relative bound is ill-posed);
  * selection:        bit-exact indices and counts on the same score vector;
  * attention output: 2e-2 absolute for bf16, 1e-5 absolute for fp32;
    lse:              1e-4 absolute + 1e-5 relative.
"""
import math

import numpy as np
import torch

import oracle

PRED_RTOL = 1e-4
SCORE_RTOL, SCORE_FLOOR = 1e-3, 1e-6
OUT_ATOL = {torch.bfloat16: 2e-2, torch.float32: 1e-5}


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def host_sequences(kvd: dict, batches=None):
    """Per-sequence ``[Hkv, T_b, d]`` float64 copies of K and V (the oracle's paging walk)."""
    k, v = kvd["k"], kvd["v"]
    lens = kvd["seq_lens"].cpu().tolist()
    batches = range(len(lens)) if batches is None else batches
    keys, vals = {}, {}
    if kvd.get("page_table") is None:
        for b in batches:
            keys[b] = np64(k[b, :, :lens[b]])
            vals[b] = np64(v[b, :, :lens[b]])
    else:
        table = kvd["page_table"].cpu().numpy()
        P = kvd["page_size"]
        for b in batches:
            n = (lens[b] + P - 1) // P
            pages = table[b, :n]
            kp = np64(k[torch.as_tensor(pages, device=k.device).long()])     # [n, Hkv, P, d]
            vp = np64(v[torch.as_tensor(pages, device=v.device).long()])
            remap = np.arange(n)
            keys[b] = oracle.gather_sequence(kp, remap, lens[b], P)
            vals[b] = oracle.gather_sequence(vp, remap, lens[b], P)
    return keys, vals


def assert_scores_close(got: np.ndarray, ref: np.ndarray, qgroup: np.ndarray, K: np.ndarray, what=""):
    d = K.shape[-1]
    qn = np.linalg.norm(qgroup, axis=-1).max()
    kn = np.linalg.norm(K, axis=-1)
    bound = SCORE_RTOL * np.abs(ref) + SCORE_FLOOR * qn * kn / math.sqrt(d)
    err = np.abs(got.astype(np.float64) - ref)
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, f"{what}: {bad.size} scores out of tolerance, first j={bad[:5]}, err={err[bad[:5]]}, bound={bound[bad[:5]]}"


def assert_pred_close(got: np.ndarray, ref: np.ndarray, what=""):
    num = np.linalg.norm(got.astype(np.float64) - ref, axis=-1)
    den = np.linalg.norm(ref, axis=-1)
    rel = num / np.maximum(den, 1e-30)
    assert rel.max() <= PRED_RTOL, f"{what}: max relative error {rel.max():.3e}"


def assert_out_close(got: torch.Tensor, ref: np.ndarray, dtype, what=""):
    err = np.abs(np64(got) - ref)
    tol = OUT_ATOL[dtype]
    assert err.max() <= tol, f"{what}: max abs error {err.max():.3e} > {tol}"


def assert_lse_close(got: torch.Tensor, ref: np.ndarray, what=""):
    g = np64(got)
    both_inf = np.isneginf(g) & np.isneginf(ref)
    fin = ~both_inf
    assert np.array_equal(np.isneginf(g), np.isneginf(ref)), f"{what}: -inf pattern differs"
    err = np.abs(g[fin] - ref[fin])
    assert (err <= 1e-4 + 1e-5 * np.abs(ref[fin])).all(), f"{what}: lse error {err.max():.3e}"


def assert_valid_topk(scores_row: np.ndarray, T_b: int, C: int, idx_row: np.ndarray, count: int, what=""):
    """The chosen set is the top C of ``scores_row[:T_b]`` with lowest-index ties (checked as a property)."""
    n = min(C, T_b)
    assert count == n, f"{what}: count {count} != {n}"
    chosen = idx_row[:n]
    assert np.all(idx_row[n:] == -1), f"{what}: padding"
    assert np.all(np.diff(chosen) > 0), f"{what}: not ascending"
    assert chosen.min(initial=0) >= 0 and (n == 0 or chosen.max() < T_b)
    s = scores_row[:T_b].astype(np.float64)
    mask = np.zeros(T_b, bool)
    mask[chosen] = True
    if n and n < T_b:
        lo = s[mask].min()
        hi = s[~mask].max()
        assert lo >= hi, f"{what}: an unselected score exceeds a selected one"
        if lo == hi:   # ties at the threshold: selected ties must precede unselected ties
            assert np.nonzero(mask & (s == lo))[0].max() < np.nonzero(~mask & (s == hi))[0].min()
