"""The decode path at the workloads' full sizes, in the bench's launch configuration (GPU).

One ``asp_decode_step`` per test: attention of step t over a seeded selection
on the main stream, prediction / scoring / selection for step t+1 on the side
stream.  The oracle recomputes sampled outputs one (sequence, KV head) unit at
a time; the whole selection is checked as a property of the GPU's own scores
and against the oracle's selection where the oracle's scores leave no near-tie.
"""
import numpy as np
import pytest
import torch

import oracle
import query_predicted_token_b200 as asp
import synth
from parity_util import (assert_lse_close, assert_out_close, assert_pred_close, assert_scores_close,
                         assert_valid_topk, host_sequences, np64)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from query_predicted_token_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert asp.device_status() == 0


def run_step(wl, kvd, tail=0, sample_units=((0, 0),), steps=1):
    """One decode step of a workload; checks it against the oracle on sampled units."""
    B, Hq, Hkv, d = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    G = Hq // Hkv
    lens = kvd["seq_lens"].cpu()
    kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], kvd["page_table"], t_max=wl.t_max)
    qhist, q_next = synth.query_history(wl, steps=1)
    q_t = q_next[0].to(wl.torch_dtype())
    tail_begin = (lens - tail).clamp(min=0) if tail else None
    snap = tail_begin.tolist() if tail else lens.tolist()
    idx0, cnt0 = synth.random_selection(B, Hkv, wl.C, snap, seed=wl.seed + 99)
    st = asp.DecodeState(kv, Hq, asp.PredCfg(wl.W, wl.windows, wl.lam), wl.C, qhist.to(DEV).contiguous(),
                         max_tail=tail, tail_begin=tail_begin.to(torch.int32).to(DEV) if tail else None)
    st.set_selection(idx0.to(DEV), cnt0.to(DEV))
    out = torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=DEV)
    lse = torch.empty(B, Hq, device=DEV)
    st.step(q_t.to(DEV), out, lse)
    assert asp.wait_selection(st.ev_sel_done, 60_000_000) == 0
    torch.cuda.synchronize()
    assert asp.device_status() == 0

    # step 1: predicted query of every head
    hist1 = torch.cat([qhist[:, :, 1:], q_t.float()[:, :, None]], dim=2)
    ref_pred = oracle.predict_query(hist1.double().numpy(), wl.windows, wl.lam)
    assert_pred_close(st.qpred.cpu().numpy(), ref_pred, wl.name)

    scores = st.scores.cpu().numpy()
    idx1, cnt1 = (t.cpu().numpy() for t in st.selection)
    # step 3 on every row: the chosen set is the top C of the GPU's own scores
    for b in range(B):
        for h in range(Hkv):
            assert_valid_topk(scores[b, h], int(lens[b]), wl.C, idx1[b, h], int(cnt1[b, h]), f"{wl.name} b{b}h{h}")

    bs = sorted({b for b, _ in sample_units})
    keys, vals = host_sequences(kvd, bs)
    qn = np64(q_t)
    gpu_pred = st.qpred.cpu().double().numpy()
    for b, h in sample_units:
        Tb = int(lens[b])
        K, V = keys[b][h], vals[b][h]
        qg = gpu_pred[b, h * G:(h + 1) * G]
        # step 2: scores of this unit for every token (same predicted query on both sides)
        ref_s = oracle.score_row(qg, K)
        assert_scores_close(scores[b, h, :Tb], ref_s, qg, K, f"{wl.name} b{b}h{h}")
        # step 3 against the oracle's own selection from its float64 scores: identical
        # except where the oracle's scores are closer than the score tolerance
        ref_sel, _ = oracle.select_row(ref_s.astype(np.float32), Tb, wl.C)
        got_sel = idx1[b, h, :int(cnt1[b, h])]
        diff = np.setxor1d(ref_sel, got_sel)
        if diff.size:
            thr = np.sort(ref_s)[::-1][min(wl.C, Tb) - 1]
            assert np.all(np.abs(ref_s[diff] - thr) <= 1e-3 * abs(thr) + 1e-5), f"{wl.name}: selection differs"
        # step 4: attention of step t over the seeded selection (+ tail)
        S = oracle.attend.attended_set(idx0[b, h].numpy(), int(cnt0[b, h]), snap[b] if tail else None, Tb)
        ref_o, ref_l = oracle.attend_set(qn[b, h * G:(h + 1) * G], K, V, S)
        assert_out_close(out[b, h * G:(h + 1) * G], ref_o, wl.torch_dtype(), f"{wl.name} out b{b}h{h}")
        assert_lse_close(lse[b, h * G:(h + 1) * G], ref_l)
    return st


def test_tiny_f32_t512_two_steps_against_the_oracle_pipeline():
    wl = synth.workload("tiny_f32_t512")
    kvd = synth.kv_cache(wl, DEV)
    units = [(0, 0), (0, 1)]
    st = run_step(wl, kvd, sample_units=units)
    # the whole two-step schedule against the oracle's own pipeline
    qhist, q_next = synth.query_history(wl, steps=2)
    keys, vals = host_sequences(kvd)
    idx0, cnt0 = synth.random_selection(1, 2, wl.C, [wl.t_max], seed=wl.seed + 99)
    r1 = oracle.decode_step(q_next[0].numpy(), qhist.numpy(), [keys[0]], [vals[0]], idx0.numpy(), cnt0.numpy(),
                            wl.C, wl.windows, wl.lam, wl.t_max)
    idx1, cnt1 = (t.cpu().numpy() for t in st.selection)
    assert np.array_equal(idx1, r1["idx"]) and np.array_equal(cnt1, r1["count"])
    out2 = torch.empty(1, 4, 64, device=DEV)
    st.step(q_next[1].to(DEV), out2)
    torch.cuda.synchronize()
    r2 = oracle.decode_step(q_next[1].numpy(), r1["qhist"], [keys[0]], [vals[0]], r1["idx"], r1["count"], wl.C,
                            wl.windows, wl.lam, wl.t_max)
    assert_out_close(out2, r2["out"], torch.float32, "step 2")
    idx2, cnt2 = (t.cpu().numpy() for t in st.selection)
    assert np.array_equal(idx2, r2["idx"]) and np.array_equal(cnt2, r2["count"])


def test_qwen3_8b_shaped_32k():
    wl = synth.workload("qwen3_8b_shaped_32k")
    kvd = synth.kv_cache(wl, DEV)
    run_step(wl, kvd, sample_units=[(0, 0), (5, 7), (7, 3)])


def test_qwen3_32b_shaped_32k():
    wl = synth.workload("qwen3_32b_shaped_32k")
    kvd = synth.kv_cache(wl, DEV)
    run_step(wl, kvd, sample_units=[(0, 0), (15, 7)])


def test_longcot_ragged_paged_b64():
    wl = synth.workload("longcot_ragged_paged_b64")
    kvd = synth.kv_cache(wl, DEV)
    lens = kvd["seq_lens"].cpu()
    b_long, b_short = int(lens.argmax()), int(lens.argmin())
    run_step(wl, kvd, tail=1, sample_units=[(b_long, 0), (b_short, 5)])
    del kvd
    torch.cuda.empty_cache()


def test_quest_page_scan_8b_32k():
    wl = synth.workload("quest_page_scan_8b_32k")
    kvd = synth.kv_cache(wl, DEV, layout="contiguous")
    B, Hq, Hkv, d, P = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, 16
    G = Hq // Hkv
    kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"])
    npm = wl.t_max // P
    meta = torch.empty(B, Hkv, npm, 2, d, dtype=torch.bfloat16, device=DEV)
    asp.quest_build_meta(kv, P, meta)
    _, q_next = synth.query_history(wl, steps=1)
    q = q_next[0].to(torch.bfloat16).to(DEV)
    ps = torch.empty(B, Hkv, npm, device=DEV)
    idx = torch.empty(B, Hkv, wl.C, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, Hkv, dtype=torch.int32, device=DEV)
    asp.quest_select(q, kv, meta, P, wl.C, ps, idx, cnt)
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(asp.attend_workspace_bytes(B, Hq, Hkv, d, wl.C), dtype=torch.uint8, device=DEV)
    asp.sparse_attend(q, kv, idx, cnt, wl.C, out, workspace=ws)
    torch.cuda.synchronize()
    assert (cnt == wl.C).all()
    keys, vals = host_sequences(kvd, [2])
    for h in (0, 6):
        kmin, kmax = oracle.quest_meta(keys[2][h], P)
        assert np.array_equal(np64(meta[2, h, :, 0]), kmin) and np.array_equal(np64(meta[2, h, :, 1]), kmax)
        qg = np64(q[2, h * G:(h + 1) * G])
        sel = idx[2, h].cpu().numpy()
        pages = np.unique(sel // P)
        assert pages.size == wl.C // P
        assert_valid_topk(ps[2, h].cpu().numpy(), npm, wl.C // P, pages, pages.size, "pages")
        ref_o, _ = oracle.attend_set(qg, keys[2][h], vals[2][h], sel)
        assert_out_close(out[2, h * G:(h + 1) * G], ref_o, torch.bfloat16, "quest attention")


def _decode_once(k, v, lens, Hq, C, W=8, windows=(4, 8), seed=5):
    """One decode step over a given cache; returns (scores, idx, count) of the new selection."""
    B, Hkv, T, d = k.shape
    g = torch.Generator().manual_seed(seed)
    kv = asp.KV(k, v, lens.to(DEV), t_max=T)
    qhist = torch.randn(B, Hq, W + 1, d, generator=g).to(DEV)
    q_t = torch.randn(B, Hq, d, generator=g).to(k.dtype).to(DEV)
    idx0, cnt0 = synth.random_selection(B, Hkv, C, lens.tolist(), seed=seed)
    st = asp.DecodeState(kv, Hq, asp.PredCfg(W, windows, 1e-2), C, qhist.contiguous())
    st.set_selection(idx0.to(DEV), cnt0.to(DEV))
    out = torch.empty(B, Hq, d, dtype=k.dtype, device=DEV)
    st.step(q_t, out)
    assert asp.wait_selection(st.ev_sel_done, 60_000_000) == 0
    torch.cuda.synchronize()
    assert asp.device_status() == 0
    idx1, cnt1 = (t.cpu().numpy() for t in st.selection)
    return st.scores.cpu().numpy(), idx1, cnt1


def test_decode_selection_of_tied_scores_keeps_the_first_tokens():
    """Zero keys make every score equal: each row keeps its first C tokens.  The rows
    span every path of the selection: shorter than C, fitting its shared memory, and
    longer than that (where the packed lists of all-tied rows overflow)."""
    B, Hkv, G, d, T, C = 4, 2, 2, 128, 65536, 2048
    lens = torch.tensor([1000, 30000, 50000, 65536], dtype=torch.int32)
    k = torch.zeros(B, Hkv, T, d, dtype=torch.bfloat16, device=DEV)
    v = torch.zeros(B, Hkv, T, d, dtype=torch.bfloat16, device=DEV)
    scores, idx, cnt = _decode_once(k, v, lens, Hkv * G, C)
    for b in range(B):
        n = min(C, int(lens[b]))
        for h in range(Hkv):
            assert np.all(scores[b, h, :lens[b]] == 0.0)
            assert int(cnt[b, h]) == n
            assert idx[b, h, :n].tolist() == list(range(n)), f"b{b}h{h}"
            assert np.all(idx[b, h, n:] == -1)


def test_decode_selection_ties_across_the_halves_of_a_row():
    """Two-valued scores: a set of tokens, most of them in the second half of the
    row, scores one value and every other token the other (0.0).  The quota of tied
    tokens (lowest index first) runs past the middle of the row, across the warps'
    ranges and the warp-offset scan; the result must equal the oracle's selection
    over the same scores, index for index."""
    B, Hkv, G, d, T, C = 2, 2, 2, 128, 16384, 12000
    lens = torch.tensor([16384, 13001], dtype=torch.int32)
    g = torch.Generator().manual_seed(11)
    u = torch.randn(d, generator=g)
    k = torch.zeros(B, Hkv, T, d)
    marked = torch.zeros(T, dtype=torch.bool)
    marked[9000::7] = True           # second half, strided
    marked[15000:15500] = True       # a block near the end
    marked[100:140] = True           # a few in the first half
    k[:, :, marked] = u
    k = k.to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    scores, idx, cnt = _decode_once(k, v, lens, Hkv * G, C)
    ref_idx, ref_cnt = oracle.select_topk(scores, lens.tolist(), C)
    assert np.array_equal(cnt, ref_cnt)
    assert np.array_equal(idx, ref_idx)


@pytest.mark.parametrize("precompute", [True, False], ids=["factor_from_previous_step", "full_factorisation"])
def test_predictor_over_several_steps_against_the_oracle(precompute):
    """Four decode steps at the Qwen3-8B head shapes (W = 16, windows 4, 8, 16).  With
    the precomputation every step after the first predicts with the lag factor the
    step before it stored (the next step's lag Gram holds q_t and the 15 queries
    before it): the stored factor equals the Cholesky factor of that Gram computed
    on the host, and every step's prediction matches the oracle's on the ring's
    history, as it does with the full factorisation in every step."""
    B, Hkv, G, d, T, C, W, windows, lam = 8, 8, 4, 128, 4096, 256, 16, (4, 8, 16), 1e-2
    Hq = Hkv * G
    g = torch.Generator().manual_seed(31)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    kv = asp.KV(k, v, torch.full((B,), T, dtype=torch.int32, device=DEV), t_max=T)
    seq = [torch.randn(B, Hq, d, generator=g)]
    for _ in range(W + 4):
        seq.append(0.9 * seq[-1] + 0.1 * torch.randn(B, Hq, d, generator=g))
    seq = [x.to(torch.bfloat16).float() for x in seq]   # the queries arrive as bf16
    hist = torch.stack(seq[:W + 1], dim=2)              # oldest first, ring_start 0
    st = asp.DecodeState(kv, Hq, asp.PredCfg(W, windows, lam), C, hist.to(DEV).contiguous(),
                         precompute_factor=precompute)
    assert (st.pred_factor is not None) == precompute
    idx0, cnt0 = synth.random_selection(B, Hkv, C, [T] * B, seed=3)
    st.set_selection(idx0.to(DEV), cnt0.to(DEV))
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=DEV)
    for step in range(4):
        t = W + 1 + step                                 # seq[t] is this step's query
        nxt = 1 - st.cur
        st.step(seq[t].to(torch.bfloat16).to(DEV), out)
        assert asp.wait_selection(st.ev_sel_done, 60_000_000) == 0
        torch.cuda.synchronize()
        window = torch.stack(seq[t - W:t + 1], dim=2)    # q_{t-W} .. q_t
        ref = oracle.predict_query(window.double().numpy(), windows, lam)
        assert_pred_close(st.qpred.cpu().numpy(), ref, f"step {step}")
        if precompute:
            # the factor stored for the next step: its lags are q_t, q_{t-1}, ... (newest first)
            lags = torch.stack([seq[t - r] for r in range(W)], dim=2).double()      # [B, Hq, W, d]
            gram = lags @ lags.transpose(-1, -2) + lam * torch.eye(W, dtype=torch.float64)
            L = torch.linalg.cholesky(gram)
            inv = 1.0 / torch.diagonal(L, dim1=-2, dim2=-1)
            scaled = torch.tril(L * inv[..., :, None], diagonal=-1)
            fac = st.pred_factor[nxt].cpu().view(B * Hq, W * W + W)
            got_rows = torch.tril(fac[:, :W * W].view(B * Hq, W, W), diagonal=-1)
            assert torch.allclose(got_rows, scaled.view(B * Hq, W, W), rtol=1e-4, atol=1e-5), f"step {step} factor"
            assert torch.allclose(fac[:, W * W:], inv.view(B * Hq, W), rtol=1e-4), f"step {step} 1/diag"
    assert asp.device_status() == 0


def test_decode_selection_up_to_32k_tokens_matches_the_oracle_on_ragged_rows():
    """Rows of at most 32K tokens keep the whole row in registers (one 16-byte vector
    per lane and chunk): ragged lengths that end inside a vector, inside a warp's
    span and exactly at C, and a row shorter than C, against the oracle's selection
    over the same scores, index for index."""
    B, Hkv, G, d, T, C = 5, 2, 2, 128, 32768, 2048
    lens = torch.tensor([1000, 2048, 3001, 17003, 32768], dtype=torch.int32)
    g = torch.Generator().manual_seed(21)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    scores, idx, cnt = _decode_once(k, v, lens, Hkv * G, C)
    ref_idx, ref_cnt = oracle.select_topk(scores, lens.tolist(), C)
    assert np.array_equal(cnt, ref_cnt)
    assert np.array_equal(idx, ref_idx)


def test_decode_selection_up_to_32k_tokens_of_tied_scores():
    """Every score equal on rows of at most 32K tokens: the first C tokens of each row
    (the first digit's bin holds the whole row, and the third digit still leaves
    exact ties, taken lowest index first)."""
    B, Hkv, G, d, T, C = 4, 2, 2, 128, 32768, 2048
    lens = torch.tensor([1000, 2048, 20001, 32768], dtype=torch.int32)
    k = torch.zeros(B, Hkv, T, d, dtype=torch.bfloat16, device=DEV)
    v = torch.zeros(B, Hkv, T, d, dtype=torch.bfloat16, device=DEV)
    scores, idx, cnt = _decode_once(k, v, lens, Hkv * G, C)
    for b in range(B):
        n = min(C, int(lens[b]))
        for h in range(Hkv):
            assert int(cnt[b, h]) == n
            assert idx[b, h, :n].tolist() == list(range(n)), f"b{b}h{h}"
            assert np.all(idx[b, h, n:] == -1)


def test_decode_selection_up_to_32k_tokens_with_few_distinct_scores():
    """Keys drawn from eight vectors give eight score values per row, so the C-th
    largest sits inside a group of exactly equal scores that the three digits cannot
    split: the group's first tokens by index fill the quota, as in the oracle."""
    B, Hkv, G, d, T, C = 2, 2, 2, 128, 30000, 5000
    lens = torch.tensor([30000, 24001], dtype=torch.int32)
    g = torch.Generator().manual_seed(23)
    basis = torch.randn(8, d, generator=g)
    pick = torch.randint(0, 8, (B, Hkv, T), generator=g)
    k = basis[pick].to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    scores, idx, cnt = _decode_once(k, v, lens, Hkv * G, C)
    for b in range(B):
        for h in range(Hkv):
            assert np.unique(scores[b, h, :lens[b]]).size <= 8
    ref_idx, ref_cnt = oracle.select_topk(scores, lens.tolist(), C)
    assert np.array_equal(cnt, ref_cnt)
    assert np.array_equal(idx, ref_idx)


def test_decode_selection_when_most_tokens_survive_the_first_digit():
    """C close to T_b on rows longer than the selection's shared memory: the survivors
    of the first digit overflow the packed lists and the row is re-read from L2."""
    B, Hkv, G, d, T, C = 2, 2, 2, 128, 60000, 50000
    lens = torch.tensor([60000, 52000], dtype=torch.int32)
    g = torch.Generator().manual_seed(7)
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).to(DEV)
    scores, idx, cnt = _decode_once(k, v, lens, Hkv * G, C)
    for b in range(B):
        for h in range(Hkv):
            assert_valid_topk(scores[b, h], int(lens[b]), C, idx[b, h], int(cnt[b, h]), f"b{b}h{h}")


@pytest.mark.parametrize("page_size", [0, 16])
def test_decode_steps_that_append_the_new_token(page_size):
    """Three decode steps, each appending the new token first: the lengths advance,
    the attention covers the previous selection plus the new token (its tail), the
    next selection is the top C of the step's own scores over every token so far,
    and the kept page bounds equal bounds rebuilt from the grown cache."""
    from test_gpu_kernels import make_cache
    B, Hkv, G, d, C, W, P, cap = 2, 8, 4, 128, 128, 8, 16, 1024
    lens0 = [1000, 700]
    if page_size == 0:
        kvd, _ = make_cache(B, Hkv, d, cap, torch.bfloat16, lens0, 0, seed=41)
    else:   # every sequence owns all its pages; the lengths start shorter
        kvd, _ = make_cache(B, Hkv, d, cap, torch.bfloat16, [cap] * B, P, seed=41)
        kvd["seq_lens"] = torch.tensor(lens0, dtype=torch.int32, device=DEV)
    kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], kvd["page_table"], t_max=cap)
    meta = torch.zeros(B, Hkv, cap // P, 2, d, dtype=torch.bfloat16, device=DEV)
    asp.quest_build_meta(kv, P, meta)
    g = torch.Generator().manual_seed(42)
    qhist = torch.randn(B, Hkv * G, W + 1, d, generator=g).to(DEV).contiguous()
    tail = torch.tensor(lens0, dtype=torch.int32, device=DEV)
    st = asp.DecodeState(kv, Hkv * G, asp.PredCfg(W, (4, 8), 1e-2), C, qhist, max_tail=1, tail_begin=tail)
    idx0, cnt0 = synth.random_selection(B, Hkv, C, lens0, seed=43)
    st.set_selection(idx0.to(DEV), cnt0.to(DEV))
    for step in range(3):
        q = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16).to(DEV)
        k_new = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16).to(DEV)
        v_new = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16).to(DEV)
        old = kvd["seq_lens"].cpu().tolist()
        idx_cur, cnt_cur = st.idx[st.cur].cpu().numpy(), st.count[st.cur].cpu().numpy()
        out = torch.empty(B, Hkv * G, d, dtype=torch.bfloat16, device=DEV)
        lse = torch.empty(B, Hkv * G, device=DEV)
        st.step(q, out, lse, k_new, v_new, meta, P)
        assert asp.wait_selection(st.ev_sel_done, 60_000_000) == 0
        torch.cuda.synchronize()
        assert asp.device_status() == 0
        new = kvd["seq_lens"].cpu().tolist()
        assert new == [t + 1 for t in old] and tail.cpu().tolist() == old
        keys, vals = host_sequences(kvd)
        scores = st.scores.cpu().numpy()
        idx1, cnt1 = (t.cpu().numpy() for t in st.selection)
        for b in range(B):
            assert np.array_equal(keys[b][:, old[b]], np64(k_new[b]))      # the token is in the cache
            for h in range(Hkv):
                S = oracle.attend.attended_set(idx_cur[b, h], int(cnt_cur[b, h]), old[b], new[b])
                assert old[b] in S.tolist()
                ref_o, ref_l = oracle.attend_set(np64(q[b, h * G:(h + 1) * G]), keys[b][h], vals[b][h], S)
                assert_out_close(out[b, h * G:(h + 1) * G], ref_o, torch.bfloat16, f"step {step} b{b}h{h}")
                assert_lse_close(lse[b, h * G:(h + 1) * G], ref_l)
                assert_valid_topk(scores[b, h], new[b], C, idx1[b, h], int(cnt1[b, h]), f"step {step} b{b}h{h}")
    ref = torch.zeros_like(meta)
    asp.quest_build_meta(kv, P, ref)
    torch.cuda.synchronize()
    for b in range(B):
        n = -(-int(kvd["seq_lens"][b]) // P)
        assert torch.equal(meta[b, :, :n], ref[b, :, :n])


def test_graph_replay_reproduces_eager_steps_bit_for_bit():
    """Steps replayed from captured CUDA graphs (one per parity x ring state, with
    the append of the new token) give exactly the eager steps' outputs, selections,
    lengths and tails."""
    from test_gpu_kernels import make_cache
    B, Hkv, G, d, C, W, cap = 2, 8, 4, 128, 128, 4, 2048
    lens0 = [1500, 900]
    states = []
    for _ in range(2):
        kvd, _ = make_cache(B, Hkv, d, cap, torch.bfloat16, lens0, 0, seed=51)
        kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], t_max=cap)
        qhist = torch.randn(B, Hkv * G, W + 1, d, generator=torch.Generator().manual_seed(52)).to(DEV).contiguous()
        tail = torch.tensor(lens0, dtype=torch.int32, device=DEV)
        st = asp.DecodeState(kv, Hkv * G, asp.PredCfg(W, (2, 4), 1e-2), C, qhist, max_tail=1, tail_begin=tail)
        idx0, cnt0 = synth.random_selection(B, Hkv, C, lens0, seed=53)
        st.set_selection(idx0.to(DEV), cnt0.to(DEV))
        bufs = dict(q=torch.empty(B, Hkv * G, d, dtype=torch.bfloat16, device=DEV),
                    k=torch.empty(B, Hkv, d, dtype=torch.bfloat16, device=DEV),
                    v=torch.empty(B, Hkv, d, dtype=torch.bfloat16, device=DEV),
                    out=torch.empty(B, Hkv * G, d, dtype=torch.bfloat16, device=DEV),
                    lse=torch.empty(B, Hkv * G, device=DEV))
        states.append((kvd, st, tail, bufs))
    g = torch.Generator().manual_seed(54)
    inputs = [(torch.randn(B, Hkv * G, d, generator=g), torch.randn(B, Hkv, d, generator=g),
               torch.randn(B, Hkv, d, generator=g)) for _ in range(14)]
    graphed = False
    for step, (q, k, v) in enumerate(inputs):
        for i, (kvd, st, tail, bf) in enumerate(states):
            bf["q"].copy_(q.to(torch.bfloat16))
            bf["k"].copy_(k.to(torch.bfloat16))
            bf["v"].copy_(v.to(torch.bfloat16))
            if i == 1 and step >= 1:
                if not graphed:   # after one eager step: one graph per state of the cycle
                    assert st.capture(bf["q"], bf["out"], bf["lse"], bf["k"], bf["v"]) == 10   # lcm(2, W + 1)
                    graphed = True
                st.replay()
            else:
                st.step(bf["q"], bf["out"], bf["lse"], bf["k"], bf["v"])
            torch.cuda.current_stream().wait_event(st.ev_sel_done)
        torch.cuda.synchronize()
        (ka, sa, ta, ba), (kb, sb, tb, bb) = states
        assert torch.equal(ba["out"], bb["out"]) and torch.equal(ba["lse"], bb["lse"]), f"step {step}"
        for x, y in zip(sa.selection, sb.selection):
            assert torch.equal(x, y), f"step {step}"
        assert torch.equal(ka["seq_lens"], kb["seq_lens"]) and torch.equal(ta, tb)
    assert states[1][1].ring_start == states[0][1].ring_start and states[1][1].cur == states[0][1].cur
    states[1][1].release_graphs()
    assert asp.device_status() == 0


def test_dense_attention_bf16_at_the_8b_shape():
    """Full attention (the pages' other baseline) as the bench times it: bf16, every
    one of the 32768 cached tokens through the tail path (count 0, tail_begin 0),
    sampled units against the oracle's dense softmax attention."""
    wl = synth.workload("qwen3_8b_shaped_32k")
    kvd = synth.kv_cache(wl, DEV)
    B, Hq, Hkv, d, T = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.t_max
    G = Hq // Hkv
    kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], t_max=T)
    q = synth.query_history(wl, steps=1)[1][0].to(torch.bfloat16).to(DEV)
    out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, Hq, device=DEV)
    zero = torch.zeros(B, dtype=torch.int32, device=DEV)
    ws = torch.empty(max(16, asp.attend_workspace_bytes(B, Hq, Hkv, d, 0, T)), dtype=torch.uint8, device=DEV)
    asp.sparse_attend(q, kv, None, None, 0, out, lse, zero, T, ws)
    torch.cuda.synchronize()
    assert asp.device_status() == 0
    units = [(0, 0), (3, 5), (7, 7)]
    keys, vals = host_sequences(kvd, sorted({b for b, _ in units}))
    qn = np64(q)
    for b, h in units:
        ref_o, ref_l = oracle.attend_set(qn[b, h * G:(h + 1) * G], keys[b][h], vals[b][h], np.arange(T))
        assert_out_close(out[b, h * G:(h + 1) * G], ref_o, torch.bfloat16, f"dense b{b}h{h}")
        assert_lse_close(lse[b, h * G:(h + 1) * G], ref_l)


def test_layer_stack_gives_each_layer_its_single_step_results():
    """Three layers decoded as the bench's stack does (every layer's attention on the
    main stream in layer order, every layer's selection chain on one shared side
    stream): each layer's output and next selection equal those of the same layer
    stepped alone, bit for bit, and one layer matches the oracle."""
    B, Hkv, G, d, T, C, W, windows = 2, 8, 4, 128, 4096, 256, 8, (4, 8)
    Hq = Hkv * G
    from test_gpu_kernels import make_cache

    def layer(l):
        kvd, kv = make_cache(B, Hkv, d, T, torch.bfloat16, [T, 3000], 0, seed=60 + l)
        g = torch.Generator().manual_seed(70 + l)
        qhist = torch.randn(B, Hq, W + 1, d, generator=g)
        q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
        idx0, cnt0 = synth.random_selection(B, Hkv, C, [T, 3000], seed=80 + l)
        return kvd, kv, qhist, q, idx0, cnt0

    layers = [layer(l) for l in range(3)]
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream(priority=-100)
    stacked, alone = [], []
    for shared in (True, False):
        for l, (kvd, kv, qhist, q, idx0, cnt0) in enumerate(layers):
            st = asp.DecodeState(kv, Hq, asp.PredCfg(W, windows, 1e-2), C, qhist.to(DEV).contiguous(),
                                 s_main=main, s_side=side if shared else None)
            st.set_selection(idx0.to(DEV), cnt0.to(DEV))
            out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=DEV)
            (stacked if shared else alone).append((st, out))
        states = stacked if shared else alone
        for l, (st, out) in enumerate(states):   # one token through the stack (or each layer on its own)
            st.step(layers[l][3].to(DEV), out)
            if not shared:
                main.wait_event(st.ev_sel_done)
        for st, _ in states:
            main.wait_event(st.ev_sel_done)
        torch.cuda.synchronize()
    assert asp.device_status() == 0
    for (sa, oa), (sb, ob) in zip(stacked, alone):
        assert torch.equal(oa, ob)
        for x, y in zip(sa.selection, sb.selection):
            assert torch.equal(x, y)
    # layer 1 against the oracle's step
    kvd, kv, qhist, q, idx0, cnt0 = layers[1]
    keys, vals = host_sequences(kvd)
    r = oracle.decode_step(q.double().numpy(), qhist.numpy(), [keys[0], keys[1]], [vals[0], vals[1]], idx0.numpy(),
                           cnt0.numpy(), C, windows, 1e-2, T)
    st, out = stacked[1]
    assert_out_close(out, r["out"], torch.bfloat16, "stack layer 1")
    assert_pred_close(st.qpred.cpu().numpy(), r["qpred"], "stack layer 1")
    scores = st.scores.cpu().numpy()
    idx1, cnt1 = (t.cpu().numpy() for t in st.selection)
    for b, Tb in enumerate([T, 3000]):
        for h in range(Hkv):
            assert_valid_topk(scores[b, h], Tb, C, idx1[b, h], int(cnt1[b, h]), f"stack b{b}h{h}")
