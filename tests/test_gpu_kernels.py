"""Parity of each CUDA step with the oracle on small seeded inputs (GPU).

Sizes span several 16-row blocks / tiles, ragged tails, empty sequences and
every supported (dtype, head_dim, group) combination.  All inputs come from
the seeded generators; all calls go through the C ABI.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import query_predicted_token_b200 as asp
from parity_util import (OUT_ATOL, assert_lse_close, assert_out_close, assert_pred_close, assert_scores_close,
                         assert_valid_topk, host_sequences, np64)
from synth import random_selection, score_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from query_predicted_token_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    asp.lib()
    yield
    assert asp.device_status() == 0


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def make_cache(B, Hkv, d, T, dtype, lens, page_size=0, seed=0):
    """Small KV cache on the GPU (contiguous or paged with a shuffled table)."""
    g = _gen(seed)
    if page_size == 0:
        k = torch.randn(B, Hkv, T, d, generator=g).to(dtype)
        v = torch.randn(B, Hkv, T, d, generator=g).to(dtype)
        kvd = dict(k=k.to(DEV), v=v.to(DEV), seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV),
                   page_table=None, page_size=0)
        return kvd, asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"])
    P = page_size
    maxp = (T + P - 1) // P
    per = [(t + P - 1) // P for t in lens]
    n = max(1, sum(per))
    perm = torch.randperm(n, generator=g).to(torch.int32)
    table = torch.full((B, maxp), -1, dtype=torch.int32)
    off = 0
    for b, c in enumerate(per):
        table[b, :c] = perm[off:off + c]
        off += c
    k = torch.randn(n, Hkv, P, d, generator=g).to(dtype)
    v = torch.randn(n, Hkv, P, d, generator=g).to(dtype)
    kvd = dict(k=k.to(DEV), v=v.to(DEV), seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV),
               page_table=table.to(DEV), page_size=P)
    return kvd, asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], kvd["page_table"], t_max=T)


CASES = [(dt, d, G) for dt in (torch.bfloat16, torch.float32) for d in (64, 128) for G in (1, 2, 4, 8)]


@pytest.mark.parametrize("dtype,d,G", CASES)
@pytest.mark.parametrize("page_size", [0, 16, 32])
def test_score_keys(dtype, d, G, page_size):
    B, Hkv, T = 3, 2, 1000
    lens = [1000, 517, 1] if page_size == 0 else [1000, 530, 17]
    kvd, kv = make_cache(B, Hkv, d, T, dtype, lens, page_size, seed=G * 10 + d)
    qpred = torch.randn(B, Hkv * G, d, generator=_gen(5)).to(DEV)
    scores = torch.full((B, Hkv, T), float("nan"), device=DEV)
    asp.score_keys(qpred, kv, scores)
    # the CUDA-core scan (the tensor-core scan's comparison for bf16 keys) gives the same scores
    scores_cc = torch.full((B, Hkv, T), float("nan"), device=DEV)
    asp.score_keys_cuda_cores(qpred, kv, scores_cc)
    torch.cuda.synchronize()
    keys, _ = host_sequences(kvd)
    ref = oracle.score_keys(np64(qpred), [keys[b] for b in range(B)], T)
    for got in (scores.cpu().numpy(), scores_cc.cpu().numpy()):
        for b in range(B):
            for h in range(Hkv):
                Tb = lens[b]
                assert_scores_close(got[b, h, :Tb], ref[b, h, :Tb], np64(qpred[b, h * G:(h + 1) * G]),
                                    keys[b][h], what=f"b{b} h{h}")
                assert np.isnan(got[b, h, Tb:]).all()      # entries past T_b are not written


_MANY_SHORT = [int(x) for x in np.random.default_rng(3).integers(1, 41, 200)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("lens", [[1000, 530, 17], _MANY_SHORT], ids=["three", "many_short"])
def test_score_keys_whole_pages(d, G, lens):
    """8 KV heads in 16-token pages: one tile per page of every head.  200 short
    sequences make every CTA switch sequences within a few tiles."""
    B, Hkv = len(lens), 8
    T = max(lens)
    kvd, kv = make_cache(B, Hkv, d, T, torch.bfloat16, lens, 16, seed=G + d)
    qpred = torch.randn(B, Hkv * G, d, generator=_gen(6)).to(DEV)
    scores = torch.full((B, Hkv, T), float("nan"), device=DEV)
    asp.score_keys(qpred, kv, scores)
    torch.cuda.synchronize()
    keys, _ = host_sequences(kvd)
    ref = oracle.score_keys(np64(qpred), [keys[b] for b in range(B)], T)
    got = scores.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            Tb = lens[b]
            assert_scores_close(got[b, h, :Tb], ref[b, h, :Tb], np64(qpred[b, h * G:(h + 1) * G]), keys[b][h],
                                what=f"b{b} h{h}")
            assert np.isnan(got[b, h, Tb:]).all()


def test_decode_step_on_whole_pages_selects_the_top_scores():
    """The decode step on a paged cache of 8 KV heads (GQA group 8, d = 64): the
    selection, made from the histogram the page scan counts, is the top C of the
    step's own scores, and the scores match the oracle."""
    lens = [3000, 5000, 700, 4100]
    B, Hkv, G, d, C, W = len(lens), 8, 8, 64, 256, 8
    kvd, kv = make_cache(B, Hkv, d, max(lens), torch.bfloat16, lens, 16, seed=12)
    g = _gen(13)
    qhist = torch.randn(B, Hkv * G, W + 1, d, generator=g).to(DEV).contiguous()
    q_t = torch.randn(B, Hkv * G, d, generator=g).to(torch.bfloat16).to(DEV)
    idx0, cnt0 = random_selection(B, Hkv, C, lens, seed=14)
    st = asp.DecodeState(kv, Hkv * G, asp.PredCfg(W, (4, 8), 1e-2), C, qhist)
    st.set_selection(idx0.to(DEV), cnt0.to(DEV))
    out = torch.empty(B, Hkv * G, d, dtype=torch.bfloat16, device=DEV)
    st.step(q_t, out)
    assert asp.wait_selection(st.ev_sel_done, 60_000_000) == 0
    torch.cuda.synchronize()
    scores = st.scores.cpu().numpy()
    idx1, cnt1 = (t.cpu().numpy() for t in st.selection)
    keys, _ = host_sequences(kvd)
    pred = st.qpred.cpu().double().numpy()
    for b in range(B):
        for h in range(Hkv):
            assert_valid_topk(scores[b, h], lens[b], C, idx1[b, h], int(cnt1[b, h]), f"b{b}h{h}")
            ref = oracle.score_row(pred[b, h * G:(h + 1) * G], keys[b][h])
            assert_scores_close(scores[b, h, :lens[b]], ref, pred[b, h * G:(h + 1) * G], keys[b][h], f"b{b}h{h}")


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 128)])
@pytest.mark.parametrize("page_size", [0, 16])
def test_append_kv_writes_the_token_and_keeps_the_page_bounds(dtype, d, page_size):
    B, Hkv, P = 3, 2, 16
    if page_size == 0:
        lens = [40, 95, 17]
        kvd, kv = make_cache(B, Hkv, d, 96, dtype, lens, 0, seed=d)
    else:   # every sequence owns 4 pages (64 tokens) and uses fewer: the append has room
        lens = [40, 63, 17]
        kvd, _ = make_cache(B, Hkv, d, 64, dtype, [64] * B, 16, seed=d + 1)
        kvd["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device=DEV)
        kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], kvd["page_table"], t_max=64)
    npm = (kv.t_max + P - 1) // P
    meta = torch.zeros(B, Hkv, npm, 2, d, dtype=dtype, device=DEV)
    asp.quest_build_meta(kv, P, meta)
    k0, v0 = kvd["k"].clone(), kvd["v"].clone()
    g = _gen(21)
    k_new = torch.randn(B, Hkv, d, generator=g).to(dtype).to(DEV)
    v_new = torch.randn(B, Hkv, d, generator=g).to(dtype).to(DEV)
    tail = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    asp.append_kv(kv, k_new, v_new, tail, meta, P)
    torch.cuda.synchronize()
    assert kvd["seq_lens"].cpu().tolist() == [t + 1 for t in lens]
    assert tail.cpu().tolist() == lens
    for b in range(B):
        T_b = lens[b]
        for h in range(Hkv):
            if page_size == 0:
                at = (b, h, T_b)
            else:
                at = (int(kvd["page_table"][b, T_b // P]), h, T_b % P)
            assert torch.equal(kvd["k"][at], k_new[b, h]) and torch.equal(kvd["v"][at], v_new[b, h])
            kvd["k"][at], kvd["v"][at] = k0[at], v0[at]   # everything else is untouched
    assert torch.equal(kvd["k"], k0) and torch.equal(kvd["v"], v0)
    # the kept bounds equal bounds rebuilt from the cache with the token in it
    kvd["k"].copy_(k0)
    for b in range(B):
        for h in range(Hkv):
            at = (b, h, lens[b]) if page_size == 0 else (int(kvd["page_table"][b, lens[b] // P]), h, lens[b] % P)
            kvd["k"][at] = k_new[b, h]
    ref = torch.zeros_like(meta)
    asp.quest_build_meta(kv, P, ref)
    torch.cuda.synchronize()
    for b in range(B):
        n = (lens[b] + 1 + P - 1) // P
        assert torch.equal(meta[b, :, :n], ref[b, :, :n])


def test_append_kv_at_capacity_changes_nothing_and_reports_it():
    kvd, kv = make_cache(2, 2, 64, 32, torch.bfloat16, [32, 5])
    k_new = torch.ones(2, 2, 64, dtype=torch.bfloat16, device=DEV)
    before = kvd["k"].clone()
    asp.append_kv(kv, k_new, k_new)
    torch.cuda.synchronize()
    assert kvd["seq_lens"].cpu().tolist() == [32, 6]          # the full sequence keeps its length
    assert torch.equal(kvd["k"][0], before[0])
    assert asp.device_status() & asp.ASP_DEV_BAD_PAGE          # reported (and cleared)


def test_score_empty_sequence_writes_nothing():
    kvd, kv = make_cache(2, 2, 128, 64, torch.bfloat16, [0, 40])
    qpred = torch.randn(2, 8, 128, generator=_gen(1)).to(DEV)
    scores = torch.full((2, 2, 64), float("nan"), device=DEV)
    asp.score_keys(qpred, kv, scores)
    torch.cuda.synchronize()
    assert torch.isnan(scores[0]).all() and not torch.isnan(scores[1, :, :40]).any()


@pytest.mark.parametrize("T,C", [(1, 1), (100, 7), (2048, 2048), (5000, 2048), (5000, 4999), (32768, 2048),
                                 (65536, 2048), (100003, 1000), (70000, 65536)])
@pytest.mark.parametrize("kind", ["normal", "ties", "special", "equal"])
def test_select_topk_bit_exact(T, C, kind):
    rows = 4
    s = score_rows(rows, T, seed=T + C, kind=kind)
    lens = torch.tensor([T, max(1, T // 3), max(1, T - 5), min(T, C)], dtype=torch.int32)
    sc = s.to(DEV).view(rows, 1, T).repeat(1, 2, 1).contiguous()        # 2 KV heads, same row
    idx = torch.full((rows, 2, C), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((rows, 2), -7, dtype=torch.int32, device=DEV)
    asp.select_topk(sc, lens.to(DEV), C, idx, cnt)
    torch.cuda.synchronize()
    ref_idx, ref_cnt = oracle.select_topk(np.repeat(s.numpy()[:, None, :], 2, axis=1), lens.tolist(), C)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)


def test_select_without_seq_lens_uses_t_max():
    s = score_rows(3, 3000, seed=1).to(DEV).view(3, 1, 3000)
    idx = torch.empty(3, 1, 100, dtype=torch.int32, device=DEV)
    cnt = torch.empty(3, 1, dtype=torch.int32, device=DEV)
    asp.select_topk(s, None, 100, idx, cnt)
    ref_idx, ref_cnt = oracle.select_topk(s.cpu().numpy(), [3000] * 3, 100)
    assert np.array_equal(idx.cpu().numpy(), ref_idx) and np.array_equal(cnt.cpu().numpy(), ref_cnt)


def test_select_empty_rows():
    s = score_rows(2, 50, seed=3).to(DEV).view(2, 1, 50)
    idx = torch.full((2, 1, 8), 5, dtype=torch.int32, device=DEV)
    cnt = torch.full((2, 1), 5, dtype=torch.int32, device=DEV)
    asp.select_topk(s, torch.tensor([0, 3], dtype=torch.int32, device=DEV), 8, idx, cnt)
    assert cnt.cpu().tolist() == [[0], [3]]
    assert idx[0].cpu().tolist() == [[-1] * 8] and idx[1].cpu().tolist() == [[0, 1, 2] + [-1] * 5]


@pytest.mark.parametrize("dtype,d,G", CASES)
@pytest.mark.parametrize("page_size", [0, 16])
@pytest.mark.parametrize("C", [1, 37, 300])
def test_sparse_attend(dtype, d, G, page_size, C):
    B, Hkv, T = 3, 2, 700
    lens = [700, 333, 5]
    kvd, kv = make_cache(B, Hkv, d, T, dtype, lens, page_size, seed=C + d)
    q = torch.randn(B, Hkv * G, d, generator=_gen(C)).to(dtype).to(DEV)
    idx, cnt = random_selection(B, Hkv, C, lens, seed=C * 7 + G)
    out = torch.empty(B, Hkv * G, d, dtype=dtype, device=DEV)
    lse = torch.empty(B, Hkv * G, device=DEV)
    ws = torch.empty(max(16, asp.attend_workspace_bytes(B, Hkv * G, Hkv, d, C)), dtype=torch.uint8, device=DEV)
    asp.sparse_attend(q, kv, idx.to(DEV), cnt.to(DEV), C, out, lse, workspace=ws)
    torch.cuda.synchronize()
    keys, vals = host_sequences(kvd)
    ref, ref_lse = oracle.sparse_attend(np64(q), [keys[b] for b in range(B)], [vals[b] for b in range(B)],
                                        idx.numpy(), cnt.numpy())
    assert_out_close(out, ref, dtype, f"{dtype} d{d} G{G} P{page_size} C{C}")
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_sparse_attend_many_splits_and_tail(dtype):
    B, Hkv, G, d, T = 2, 2, 4, 128, 6000
    lens = [6000, 4100]
    kvd, kv = make_cache(B, Hkv, d, T, dtype, lens, 16, seed=11)
    C, max_tail = 2048, 64
    # the selection was made on a snapshot; tokens from tail_begin on are attended in full
    tail_begin = torch.tensor([5990, 4100 - 64], dtype=torch.int32)
    idx, cnt = random_selection(B, Hkv, C, tail_begin.tolist(), seed=3)
    q = torch.randn(B, Hkv * G, d, generator=_gen(9)).to(dtype).to(DEV)
    out = torch.empty(B, Hkv * G, d, dtype=dtype, device=DEV)
    lse = torch.empty(B, Hkv * G, device=DEV)
    ws = torch.empty(asp.attend_workspace_bytes(B, Hkv * G, Hkv, d, C, max_tail), dtype=torch.uint8, device=DEV)
    asp.sparse_attend(q, kv, idx.to(DEV), cnt.to(DEV), C, out, lse, tail_begin.to(DEV), max_tail, ws)
    torch.cuda.synchronize()
    keys, vals = host_sequences(kvd)
    ref, ref_lse = oracle.sparse_attend(np64(q), [keys[0], keys[1]], [vals[0], vals[1]], idx.numpy(), cnt.numpy(),
                                        tail_begin.tolist())
    assert_out_close(out, ref, dtype)
    assert_lse_close(lse, ref_lse)


def _lens(n, lo, hi, seed):
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, n)]


# B, Hkv, G, d, C, lens, page_size, tail: each at least 200 16-row tiles per SM (the
# gather kernel's range): ragged counts below C with a tail; a paged ragged batch with
# groups of 8; d = 64 with one query head per KV head
_GATHER_CASES = [
    (64, 8, 4, 128, 1024, _lens(64, 600, 1500, 1), 0, 3),
    (32, 8, 8, 128, 2048, _lens(32, 1000, 3000, 2), 16, 5),
    (16, 16, 1, 64, 1900, [2000] * 16, 0, 0),
]


@pytest.mark.parametrize("case", _GATHER_CASES, ids=["ragged_tail_G4", "paged_G8", "d64_G1"])
def test_sparse_attend_gather_kernel(case):
    """bf16 attention on batches large enough for the persistent gather kernel:
    units split over CTA boundaries (partials merged by the log-sum-exp kernel) and
    CTAs holding several units, against the oracle."""
    B, Hkv, G, d, C, lens, page_size, tail = case
    assert B * Hkv * -(-(C + tail) // 16) >= 200 * 148
    T = max(lens)
    kvd, kv = make_cache(B, Hkv, d, T, torch.bfloat16, lens, page_size, seed=B + C)
    tb = [max(0, t - tail) for t in lens]
    idx, cnt = random_selection(B, Hkv, C, tb, seed=C + G)
    q = torch.randn(B, Hkv * G, d, generator=_gen(B * 7 + d)).to(torch.bfloat16).to(DEV)
    out = torch.full((B, Hkv * G, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, Hkv * G), float("nan"), device=DEV)
    ws = torch.empty(max(16, asp.attend_workspace_bytes(B, Hkv * G, Hkv, d, C, tail)), dtype=torch.uint8, device=DEV)
    tail_begin = torch.tensor(tb, dtype=torch.int32, device=DEV) if tail else None
    asp.sparse_attend(q, kv, idx.to(DEV), cnt.to(DEV), C, out, lse, tail_begin, tail, ws)
    torch.cuda.synchronize()
    keys, vals = host_sequences(kvd)
    ref, ref_lse = oracle.sparse_attend(np64(q), [keys[b] for b in range(B)], [vals[b] for b in range(B)],
                                        idx.numpy(), cnt.numpy(), tb if tail else None)
    assert_out_close(out, ref, torch.bfloat16, f"gather {case[:5]}")
    assert_lse_close(lse, ref_lse)


def _standalone_splits(units, rows):
    """Splits per unit of the per-item kernels' stand-alone plan (three 4-warp CTAs per
    SM on 148 SMs, splits of a multiple of 64 rows)."""
    splits = max(1, 444 // units)
    per = -(-(-(-rows // splits)) // 64) * 64
    return -(-rows // per)


_CLUSTER_CASES = [
    (8, 8, 4, 128, 2048, _lens(8, 2100, 3000, 4), 0, 0),
    (55, 1, 8, 128, 2048, _lens(55, 2049, 2600, 5), 16, 0),
    (37, 3, 2, 64, 1000, _lens(37, 900, 1400, 6), 0, 0),
    (16, 4, 4, 128, 1024, _lens(16, 1100, 1500, 7), 0, 16),
]


@pytest.mark.parametrize("case", _CLUSTER_CASES, ids=["splits6_G4", "splits8_G8_paged", "splits4_d64_G2", "splits6_tail"])
def test_sparse_attend_cluster_merge(case):
    """bf16 attention whose stand-alone plan has 4 to 8 splits per unit: the splits of
    a unit form one thread-block cluster and merge their partials in the first CTA's
    shared memory.  Ragged rows (some units shorter than C), a paged cache, head
    dimension 64 and a tail, against the oracle."""
    B, Hkv, G, d, C, lens, page_size, tail = case
    assert 4 <= _standalone_splits(B * Hkv, C + tail) <= 8
    T = max(lens)
    kvd, kv = make_cache(B, Hkv, d, T, torch.bfloat16, lens, page_size, seed=B + C + d)
    tb = [max(0, t - tail) for t in lens]
    idx, cnt = random_selection(B, Hkv, C, tb, seed=C + G + 1)
    q = torch.randn(B, Hkv * G, d, generator=_gen(B * 5 + d)).to(torch.bfloat16).to(DEV)
    out = torch.full((B, Hkv * G, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, Hkv * G), float("nan"), device=DEV)
    ws = torch.empty(max(16, asp.attend_workspace_bytes(B, Hkv * G, Hkv, d, C, tail)), dtype=torch.uint8, device=DEV)
    tail_begin = torch.tensor(tb, dtype=torch.int32, device=DEV) if tail else None
    asp.sparse_attend(q, kv, idx.to(DEV), cnt.to(DEV), C, out, lse, tail_begin, tail, ws)
    torch.cuda.synchronize()
    keys, vals = host_sequences(kvd)
    ref, ref_lse = oracle.sparse_attend(np64(q), [keys[b] for b in range(B)], [vals[b] for b in range(B)],
                                        idx.numpy(), cnt.numpy(), tb if tail else None)
    assert_out_close(out, ref, torch.bfloat16, f"cluster {case[:5]}")
    assert_lse_close(lse, ref_lse)


def test_gather_kernel_flags_out_of_range_indices_and_skips_them():
    B, Hkv, G, d, C, T = 64, 8, 2, 128, 1024, 1100
    kvd, kv = make_cache(B, Hkv, d, T, torch.bfloat16, [T] * B, seed=5)
    idx, cnt = random_selection(B, Hkv, C, [T] * B, seed=6)
    bad = idx.clone()
    bad[3, 2, 10] = T + 5          # past the sequence
    bad[40, 7, 1000] = -3          # negative
    q = torch.randn(B, Hkv * G, d, generator=_gen(7)).to(torch.bfloat16).to(DEV)
    out = torch.empty(B, Hkv * G, d, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(max(16, asp.attend_workspace_bytes(B, Hkv * G, Hkv, d, C)), dtype=torch.uint8, device=DEV)
    assert asp.device_status() == 0
    asp.sparse_attend(q, kv, bad.to(DEV), cnt.to(DEV), C, out, workspace=ws)
    assert asp.device_status() & asp.ASP_DEV_BAD_INDEX
    keys, vals = host_sequences(kvd)
    keep = bad.numpy().copy()
    cnt_ref = cnt.numpy().copy()
    for (b, h, j) in ((3, 2, 10), (40, 7, 1000)):   # the oracle attends the rest of the set
        row = [x for x in keep[b, h, :cnt_ref[b, h]] if 0 <= x < T]
        keep[b, h, :len(row)] = row
        cnt_ref[b, h] = len(row)
    ref, _ = oracle.sparse_attend(np64(q), [keys[b] for b in range(B)], [vals[b] for b in range(B)], keep, cnt_ref)
    assert_out_close(out, ref, torch.bfloat16)


def test_dense_attention_through_the_tail():
    """count = 0 and tail_begin = 0 attends every token: full attention."""
    B, Hkv, G, d, T = 2, 2, 2, 64, 3000
    kvd, kv = make_cache(B, Hkv, d, T, torch.float32, [3000, 1234], seed=4)
    q = torch.randn(B, Hkv * G, d, generator=_gen(2)).to(DEV)
    zero = torch.zeros(B, dtype=torch.int32, device=DEV)
    out = torch.empty(B, Hkv * G, d, device=DEV)
    ws = torch.empty(max(16, asp.attend_workspace_bytes(B, Hkv * G, Hkv, d, 0, T)), dtype=torch.uint8, device=DEV)
    asp.sparse_attend(q, kv, None, None, 0, out, None, zero, T, ws)
    torch.cuda.synchronize()
    keys, vals = host_sequences(kvd)
    Kt = [torch.from_numpy(keys[b]) for b in range(B)]
    Vt = [torch.from_numpy(vals[b]) for b in range(B)]
    for b in range(B):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(np64(q[b]))[:, None, :], Kt[b].repeat_interleave(G, 0), Vt[b].repeat_interleave(G, 0))
        assert (np64(out[b]) - ref[:, 0].numpy()).__abs__().max() <= OUT_ATOL[torch.float32]


def test_attend_flags_out_of_range_indices_and_skips_them():
    B, Hkv, G, d, T = 1, 1, 2, 128, 200
    kvd, kv = make_cache(B, Hkv, d, T, torch.bfloat16, [200], seed=8)
    idx = torch.tensor([[[3, 10, 250, 60, -4]]], dtype=torch.int32)
    cnt = torch.tensor([[5]], dtype=torch.int32)
    q = torch.randn(B, Hkv * G, d, generator=_gen(3)).to(torch.bfloat16).to(DEV)
    out = torch.empty(B, Hkv * G, d, dtype=torch.bfloat16, device=DEV)
    assert asp.device_status() == 0
    asp.sparse_attend(q, kv, idx.to(DEV), cnt.to(DEV), 5, out)
    bits = asp.device_status()
    assert bits & asp.ASP_DEV_BAD_INDEX
    keys, vals = host_sequences(kvd)
    ref, _ = oracle.sparse_attend(np64(q), [keys[0]], [vals[0]], np.array([[[3, 10, 60]]]), np.array([[3]]))
    assert_out_close(out, ref, torch.bfloat16)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("W,windows", [(1, (1,)), (8, (4, 8)), (16, (4, 8, 16)), (16, (2, 5, 11)), (32, (1, 7, 32))])
@pytest.mark.parametrize("coef", ["softmax", "raw"])
@pytest.mark.parametrize("pool", ["predictions", "features"])
def test_predict_query(d, W, windows, coef, pool):
    B, Hq = 2, 6
    g = _gen(W * 100 + d)
    q = [torch.randn(B, Hq, d, generator=g)]
    for _ in range(W):
        q.append(0.9 * q[-1] + 0.1 * torch.randn(B, Hq, d, generator=g))
    hist = torch.stack(q, dim=2)                          # [B, Hq, W+1, d] oldest first
    for ring in (0, W // 2 + (W > 0), W):
        ring = ring % (W + 1)
        slots = torch.roll(hist, shifts=ring, dims=2)      # slot (ring + s) % (W+1) holds s-th oldest
        qhist = slots.contiguous().to(DEV)
        qpred = torch.empty(B, Hq, d, device=DEV)
        cfg = asp.PredCfg(W, windows, 1e-2, coef, pool)
        asp.predict_query(qhist, ring, cfg, qpred)
        torch.cuda.synchronize()
        fn = oracle.predict_query if pool == "predictions" else oracle.predict_query_pooled
        ref = fn(hist.double().numpy(), windows, 1e-2, coef)
        assert_pred_close(qpred.cpu().numpy(), ref, f"W{W} {windows} ring{ring} {coef}")
        assert torch.equal(qhist.cpu(), slots)             # read-only without q_new


@pytest.mark.parametrize("qdtype", [torch.float32, torch.bfloat16])
def test_predict_query_pushes_the_new_query(qdtype):
    B, Hq, d, W, windows = 2, 4, 128, 16, (4, 8, 16)
    g = _gen(77)
    seq = [torch.randn(B, Hq, d, generator=g)]
    for _ in range(W + 1):
        seq.append(0.9 * seq[-1] + 0.1 * torch.randn(B, Hq, d, generator=g))
    hist0 = torch.stack(seq[:W + 1], dim=2)
    q_new = seq[W + 1].to(qdtype)
    ring = 5
    qhist = torch.roll(hist0, shifts=ring, dims=2).contiguous().to(DEV)
    qpred = torch.empty(B, Hq, d, device=DEV)
    asp.predict_query(qhist, ring, asp.PredCfg(W, windows, 1e-2), qpred, q_new=q_new.to(DEV))
    torch.cuda.synchronize()
    hist1 = torch.cat([hist0[:, :, 1:], q_new.float()[:, :, None]], dim=2)
    ref = oracle.predict_query(hist1.double().numpy(), windows, 1e-2)
    assert_pred_close(qpred.cpu().numpy(), ref)
    assert torch.equal(qhist.cpu()[:, :, ring], q_new.float())          # oldest slot overwritten
    assert torch.equal(torch.roll(qhist.cpu(), shifts=-(ring + 1), dims=2), hist1)


@pytest.mark.parametrize("dtype,d,G", [(torch.bfloat16, 128, 4), (torch.bfloat16, 128, 8), (torch.float32, 64, 2)])
@pytest.mark.parametrize("page_size", [0, 16])
def test_quest_path(dtype, d, G, page_size):
    B, Hkv, T, P, C = 2, 2, 1500, 16, 256
    lens = [1500, 777]
    kvd, kv = make_cache(B, Hkv, d, T, dtype, lens, page_size, seed=31)
    npm = (T + P - 1) // P
    meta = torch.zeros(B, Hkv, npm, 2, d, dtype=dtype, device=DEV)
    asp.quest_build_meta(kv, P, meta)
    q = torch.randn(B, Hkv * G, d, generator=_gen(4)).to(dtype).to(DEV)
    ps = torch.full((B, Hkv, npm), float("nan"), device=DEV)
    cap = ((C + P - 1) // P) * P
    idx = torch.empty(B, Hkv, cap, dtype=torch.int32, device=DEV)
    cnt = torch.empty(B, Hkv, dtype=torch.int32, device=DEV)
    asp.quest_select(q, kv, meta, P, C, ps, idx, cnt)
    ps_alone = torch.full_like(ps, float("nan"))
    asp.quest_page_scores(q, kv, meta, P, ps_alone)
    torch.cuda.synchronize()
    for b in range(B):   # the page scores alone are the selection's own, bit for bit
        n = (lens[b] + P - 1) // P
        assert torch.equal(ps_alone[b, :, :n], ps[b, :, :n])
    keys, _ = host_sequences(kvd)
    for b in range(B):
        for h in range(Hkv):
            kmin, kmax = oracle.quest_meta(keys[b][h], P)
            n = kmin.shape[0]
            assert np.array_equal(np64(meta[b, h, :n, 0]), kmin) and np.array_equal(np64(meta[b, h, :n, 1]), kmax)
            qg = np64(q[b, h * G:(h + 1) * G])
            ref_ps = oracle.quest_page_scores(qg, kmin, kmax)
            got_ps = ps[b, h, :n].cpu().numpy()
            # the bound is a sum of |q| |k| terms: same tolerance rule as the key scores, on page rows
            rows = np.concatenate([kmin, kmax], axis=1)
            assert_scores_close(got_ps, ref_ps, np.concatenate([qg, qg], axis=1), rows / math.sqrt(2), f"pages b{b}h{h}")
            m = cnt[b, h].item()
            chosen = idx[b, h, :m].cpu().numpy()
            pages = np.unique(chosen // P)
            # the kept pages are the best ceil(C/P) of the GPU's own page scores, lowest index on ties
            page_idx = np.full(npm, -1, dtype=np.int64)
            page_idx[:pages.size] = pages
            assert_valid_topk(got_ps, n, (C + P - 1) // P, page_idx[:(C + P - 1) // P], pages.size, f"b{b}h{h}")
            expect = (pages[:, None] * P + np.arange(P)[None, :]).reshape(-1)
            expect = expect[expect < lens[b]]
            assert chosen.tolist() == expect.tolist() and m == expect.size
            assert (idx[b, h, m:] == -1).all()


def test_wait_selection_times_out_then_completes():
    s = torch.cuda.Stream()
    ev = asp.make_event()
    with torch.cuda.stream(s):
        torch.cuda._sleep(200_000_000)           # ~0.1 s of GPU spinning, bounded
        ev.record(s)
    assert asp.wait_selection(ev, 10) == asp._lib.ASP_ERR_TIMEOUT
    assert asp.wait_selection(ev, 30_000_000) == asp._lib.ASP_OK


@pytest.mark.parametrize("T", [5000, 100003])
def test_select_flags_nan_scores(T):
    """NaN scores are invalid input: the selection reports them (ASP_DEV_NAN_SCORE)
    and still writes a valid, bounded selection."""
    C = 300
    s = score_rows(2, T, seed=T)
    s[1, 17] = float("nan")
    s[1, T - 3] = float("nan")
    sc = s.to(DEV).view(2, 1, T).contiguous()
    idx = torch.full((2, 1, C), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((2, 1), -7, dtype=torch.int32, device=DEV)
    assert asp.device_status() == 0
    asp.select_topk(sc, None, C, idx, cnt)
    bits = asp.device_status()
    assert bits & asp.ASP_DEV_NAN_SCORE
    got = idx.cpu().numpy()
    assert cnt.cpu().tolist() == [[C], [C]]
    for r in range(2):
        assert np.all(np.diff(got[r, 0]) > 0) and got[r, 0].min() >= 0 and got[r, 0].max() < T
    # the row without a NaN is still the exact top C
    ref_idx, _ = oracle.select_topk(s[:1].numpy()[:, None, :], [T], C)
    assert np.array_equal(got[0], ref_idx[0])


def test_bounded_wait_gives_up_and_reports_it():
    """The bounded barrier wait of every kernel, cut to a few attempts on a barrier
    that nothing arrives on: the kernel gives up, records ASP_DEV_WAIT_LIMIT and
    returns (no fault, no hang)."""
    ret = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert asp.device_status() == 0
    asp.check_wait_limit(64, ret)
    torch.cuda.synchronize()
    assert ret.item() == 1
    assert asp.device_status() == asp.ASP_DEV_WAIT_LIMIT
