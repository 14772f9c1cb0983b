"""The C ABI boundary without a GPU: exports, struct layout, host-side validation.

Every call below is rejected by host validation before anything reaches CUDA,
so these tests never launch a kernel (fake pointers are never dereferenced).
"""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from query_predicted_token_b200 import _lib as L
from query_predicted_token_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "asp.h")
FAKE = 0x10000   # 16-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^ASP_API\s+[\w\s\*]+?\b(asp_\w+)\(", text, flags=re.M)))


def test_header_declares_the_step_entry_points():
    names = header_functions()
    for n in ["asp_predict_query", "asp_score_keys", "asp_select_topk", "asp_sparse_attend", "asp_decode_step"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(L.SIGNATURES) == names       # the binding covers exactly the header


def test_exported_symbols_are_only_the_abi(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(set(re.findall(r" T (asp_\w+)", out)))
    assert exported == header_functions()


def test_struct_layout_matches_the_c_compiler():
    src = r'''
#include <stdio.h>
#include <stddef.h>
#include "asp.h"
int main(void) {
  printf("asp_kv %zu %zu %zu %zu %zu\n", sizeof(asp_kv), offsetof(asp_kv, k), offsetof(asp_kv, page_size),
         offsetof(asp_kv, page_table), offsetof(asp_kv, seq_lens));
  printf("asp_pred_cfg %zu %zu %zu %zu\n", sizeof(asp_pred_cfg), offsetof(asp_pred_cfg, windows), offsetof(asp_pred_cfg, lambda),
         offsetof(asp_pred_cfg, pool));
  printf("asp_decode_args %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(asp_decode_args), offsetof(asp_decode_args, kv),
         offsetof(asp_decode_args, workspace_bytes), offsetof(asp_decode_args, s_main), offsetof(asp_decode_args, timing),
         offsetof(asp_decode_args, k_new), offsetof(asp_decode_args, quest_page), offsetof(asp_decode_args, pred_factor_cur),
         offsetof(asp_decode_args, pred_factor_valid), offsetof(asp_decode_args, pred_factor_next),
         offsetof(asp_decode_args, ev_attend_done));
  return 0;
}
'''
    scratch = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "_build")
    os.makedirs(scratch, exist_ok=True)
    with tempfile.TemporaryDirectory(dir=scratch) as d:
        c = os.path.join(d, "l.c")
        open(c, "w").write(src)
        exe = os.path.join(d, "l")
        subprocess.check_call(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe])
        lines = dict((ln.split()[0], [int(x) for x in ln.split()[1:]]) for ln in subprocess.check_output([exe], text=True).splitlines())
    K, P, D = L.AspKv, L.AspPredCfg, L.AspDecodeArgs
    assert lines["asp_kv"] == [ctypes.sizeof(K), K.k.offset, K.page_size.offset, K.page_table.offset, K.seq_lens.offset]
    assert lines["asp_pred_cfg"] == [ctypes.sizeof(P), P.windows.offset, P.lam.offset, P.pool.offset]
    assert lines["asp_decode_args"] == [ctypes.sizeof(D), D.kv.offset, D.workspace_bytes.offset, D.s_main.offset,
                                        D.timing.offset, D.k_new.offset, D.quest_page.offset, D.pred_factor_cur.offset,
                                        D.pred_factor_valid.offset, D.pred_factor_next.offset, D.ev_attend_done.offset]


def test_version_and_status_strings(lib):
    assert lib.asp_abi_version() == 5
    assert L.status_string(L.ASP_OK) == "ok"
    assert "workspace" in L.status_string(L.ASP_ERR_WORKSPACE)
    assert L.status_string(99) == "unknown status"


def _kv(**kw):
    base = dict(batch=2, n_kv_heads=2, head_dim=128, t_max=1024, kv_dtype=L.ASP_BF16, k=FAKE, v=FAKE, page_size=0,
                page_table=None, max_pages=0, n_pages=0, seq_lens=None)
    base.update(kw)
    return L.AspKv(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(head_dim=96), L.ASP_ERR_UNSUPPORTED),
    (dict(batch=0), L.ASP_ERR_INVALID_ARG),
    (dict(k=None), L.ASP_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), L.ASP_ERR_INVALID_ARG),                 # not 16-byte aligned
    (dict(kv_dtype=7), L.ASP_ERR_INVALID_ARG),
    (dict(page_size=8), L.ASP_ERR_UNSUPPORTED),
    (dict(page_size=16), L.ASP_ERR_INVALID_ARG),               # paged without a page table
    (dict(page_size=16, page_table=FAKE, seq_lens=FAKE, max_pages=10, n_pages=20), L.ASP_ERR_INVALID_ARG),  # 160 < t_max
    (dict(batch=70000), L.ASP_ERR_UNSUPPORTED),
])
def test_score_rejects_bad_caches(lib, kw, expect):
    kv = _kv(**kw)
    assert lib.asp_score_keys(FAKE, 8, ctypes.byref(kv), FAKE, None) == expect


def test_score_rejects_bad_groups(lib):
    kv = _kv()
    assert lib.asp_score_keys(FAKE, 6, ctypes.byref(kv), FAKE, None) == L.ASP_ERR_UNSUPPORTED   # G = 3
    assert lib.asp_score_keys(FAKE, 5, ctypes.byref(kv), FAKE, None) == L.ASP_ERR_INVALID_ARG   # 5 % 2
    assert lib.asp_score_keys(None, 8, ctypes.byref(kv), FAKE, None) == L.ASP_ERR_INVALID_ARG
    assert lib.asp_score_keys(FAKE, 8, None, FAKE, None) == L.ASP_ERR_INVALID_ARG


def test_append_validation(lib):
    """asp_append_kv checks everything on the host; nothing here reaches a kernel."""
    kv = _kv(seq_lens=FAKE)
    call = lambda kv, k=FAKE, v=FAKE, meta=None, page=16: lib.asp_append_kv(ctypes.byref(kv), k, v, None, meta, page, None)
    assert call(_kv()) == L.ASP_ERR_INVALID_ARG                     # lengths must live on the device
    assert call(kv, k=None) == L.ASP_ERR_INVALID_ARG
    assert call(kv, v=None) == L.ASP_ERR_INVALID_ARG
    assert call(_kv(seq_lens=FAKE, v=None)) == L.ASP_ERR_INVALID_ARG  # the cache needs its values
    assert call(kv, k=FAKE + 4) == L.ASP_ERR_INVALID_ARG              # not 16-byte aligned
    assert call(kv, meta=FAKE, page=0) == L.ASP_ERR_INVALID_ARG
    assert call(kv, meta=FAKE, page=24) == L.ASP_ERR_UNSUPPORTED
    paged = _kv(seq_lens=FAKE, page_size=16, page_table=FAKE, max_pages=64, n_pages=200)
    assert call(paged, meta=FAKE, page=32) == L.ASP_ERR_UNSUPPORTED  # bounds pages must be the cache's pages
    assert call(_kv(seq_lens=FAKE, head_dim=96)) == L.ASP_ERR_UNSUPPORTED


def test_select_validation(lib):
    assert lib.asp_select_topk(FAKE, None, 2, 2, 1024, 0, FAKE, FAKE, None) == L.ASP_ERR_INVALID_ARG
    assert lib.asp_select_topk(None, None, 2, 2, 1024, 8, FAKE, FAKE, None) == L.ASP_ERR_INVALID_ARG
    assert lib.asp_select_topk(FAKE, None, 70000, 1, 1024, 8, FAKE, FAKE, None) == L.ASP_ERR_UNSUPPORTED


def _ceil256(n):
    return -(-n // 256) * 256


def _ring_ws(B, Hq, Hkv, d, C, max_tail):
    # the gather kernel (batches of at least 200 16-row tiles per SM): every unit
    # planned for C + max_tail rows in 16-row tiles,
    # spread over at most 148 CTAs (at least 8 tiles each); when a unit is shared
    # by several CTAs, two partial slots per CTA, each G heads of (fp32 output,
    # max, sum)
    units, G = B * Hkv, Hq // Hkv
    tpu = -(-(C + max_tail) // 16)
    tiles = units * tpu
    if tiles < 200 * 148:          # smaller batches keep the per-item kernel
        return 0
    n = min(148, -(-tiles // 8))
    shared = False    # some unit starts in a CTA's range and runs past it
    for c in range(n):
        t0, t1 = c * tiles // n, (c + 1) * tiles // n
        ua = (t1 - 1) // tpu * tpu
        shared |= t0 < t1 and ua >= t0 and ua + tpu > t1
    if not shared:
        return 0
    slots = 2 * n * G
    return _ceil256(slots * d * 4) + _ceil256(slots * 2 * 4)


def _split_ws(B, Hq, Hkv, d, C, max_tail, ctas_per_sm):
    # the per-item kernels: splits of a multiple of 64 rows filling one wave
    units, G = B * Hkv, Hq // Hkv
    target = 148 * (ctas_per_sm or 3)
    splits = max(1, target // units)
    rows = C + max_tail
    per = -(-(-(-rows // splits)) // 64) * 64
    splits = -(-rows // per)
    if splits == 1:
        return 0
    return _ceil256(B * Hq * splits * d * 4) + _ceil256(B * Hq * splits * 2 * 4)


def test_attend_workspace_rules(lib):
    need = lib.asp_attend_workspace_bytes(8, 32, 8, 128, 2048, 0)
    assert need > 0 and need % 256 == 0
    # the larger of the two kernels' needs (the data types decide which one runs)
    for args in [(8, 32, 8, 128, 2048, 0), (1, 4, 2, 64, 64, 0), (16, 64, 8, 128, 2048, 0), (64, 32, 8, 128, 2048, 1),
                 (1, 8, 1, 128, 5000, 0), (3, 6, 2, 64, 37, 4), (64, 256, 8, 128, 1024, 3), (32, 256, 8, 128, 2048, 5)]:
        assert lib.asp_attend_workspace_bytes(*args) == max(_ring_ws(*args), _split_ws(*args, 0)), args
    assert lib.asp_attend_workspace_bytes(1, 2, 1, 128, 5, 0) == 0     # one tile in one CTA: nothing to merge
    # dense attention (a tail longer than 4096 and than C) keeps the per-item kernel only
    assert lib.asp_attend_workspace_bytes(8, 32, 8, 128, 0, 32768) == _split_ws(8, 32, 8, 128, 0, 32768, 0)
    assert lib.asp_attend_workspace_bytes(8, 32, 8, 96, 2048, 0) == 0    # unsupported head_dim
    assert lib.asp_attend_workspace_bytes(8, 32, 8, 128, 0, 0) == 0      # nothing to attend
    kv = _kv(batch=8, n_kv_heads=8, t_max=32768)
    st = lib.asp_sparse_attend(FAKE, L.ASP_BF16, 32, ctypes.byref(kv), FAKE, FAKE, 2048, None, 0, FAKE, None,
                               FAKE, need - 256, None)
    assert st == L.ASP_ERR_WORKSPACE
    st = lib.asp_sparse_attend(FAKE, L.ASP_BF16, 32, ctypes.byref(kv), FAKE, FAKE, 2048, None, 0, FAKE, None,
                               None, 0, None)
    assert st == L.ASP_ERR_WORKSPACE
    st = lib.asp_sparse_attend(FAKE, L.ASP_BF16, 32, ctypes.byref(kv), None, FAKE, 2048, None, 0, FAKE, None,
                               FAKE, need, None)
    assert st == L.ASP_ERR_INVALID_ARG
    st = lib.asp_sparse_attend(FAKE, 5, 32, ctypes.byref(kv), FAKE, FAKE, 2048, None, 0, FAKE, None, FAKE, need, None)
    assert st == L.ASP_ERR_INVALID_ARG


def test_decode_workspace_holds_the_partials_and_the_histogram(lib):
    # the decode step's attention is planned for one CTA per SM (148 SMs): 64 units
    # -> 2 splits of 1024 rows; partials (fp32 out + (max, sum) per head and split),
    # each 256-byte aligned, then the [64, 2048] int32 histogram
    B, Hq, Hkv, d, C = 8, 32, 8, 128, 2048
    parts = _split_ws(B, Hq, Hkv, d, C, 0, 1)
    dec = lib.asp_decode_workspace_bytes(B, Hq, Hkv, d, C, 0)
    assert dec == parts + B * Hkv * 2048 * 4
    # fewer splits than the stand-alone attention's plan (3 CTAs per SM)
    assert dec < lib.asp_attend_workspace_bytes(B, Hq, Hkv, d, C, 0) + B * Hkv * 2048 * 4
    assert lib.asp_decode_workspace_bytes(8, 32, 8, 96, 2048, 0) == 0
    assert lib.asp_decode_workspace_bytes(8, 32, 8, 128, 0, 0) == 0


def test_workspace_grows_with_the_tail(lib):
    a = lib.asp_attend_workspace_bytes(64, 32, 8, 128, 2048, 0)
    b = lib.asp_attend_workspace_bytes(64, 32, 8, 128, 2048, 4096)
    assert b >= a


def _cfg(W=16, windows=(4, 8, 16), lam=1e-2, coef=0, pool=0):
    arr = (ctypes.c_int * len(windows))(*windows)
    cfg = L.AspPredCfg(W, ctypes.cast(arr, ctypes.POINTER(ctypes.c_int)), len(windows), lam, coef, pool)
    return cfg, arr


@pytest.mark.parametrize("kw,ring,expect", [
    (dict(windows=(4, 17)), 0, L.ASP_ERR_INVALID_ARG),
    (dict(windows=(0,)), 0, L.ASP_ERR_INVALID_ARG),
    (dict(lam=0.0), 0, L.ASP_ERR_INVALID_ARG),
    (dict(lam=-1.0), 0, L.ASP_ERR_INVALID_ARG),
    (dict(coef=3), 0, L.ASP_ERR_INVALID_ARG),
    (dict(pool=2), 0, L.ASP_ERR_INVALID_ARG),
    (dict(W=40, windows=(4,)), 0, L.ASP_ERR_UNSUPPORTED),
    (dict(), 17, L.ASP_ERR_INVALID_ARG),
    (dict(), -1, L.ASP_ERR_INVALID_ARG),
])
def test_predict_validation(lib, kw, ring, expect):
    cfg, _keep = _cfg(**kw)
    assert lib.asp_predict_query(FAKE, ring, None, 0, 2, 8, 128, ctypes.byref(cfg), FAKE, None) == expect


def test_predict_rejects_shapes(lib):
    cfg, _keep = _cfg()
    assert lib.asp_predict_query(FAKE, 0, None, 0, 2, 8, 96, ctypes.byref(cfg), FAKE, None) == L.ASP_ERR_UNSUPPORTED
    assert lib.asp_predict_query(None, 0, None, 0, 2, 8, 128, ctypes.byref(cfg), FAKE, None) == L.ASP_ERR_INVALID_ARG
    assert lib.asp_predict_query(FAKE, 0, None, 0, 2, 8, 128, None, FAKE, None) == L.ASP_ERR_INVALID_ARG
    assert lib.asp_predict_query(FAKE, 0, FAKE, 9, 2, 8, 128, ctypes.byref(cfg), FAKE, None) == L.ASP_ERR_INVALID_ARG


def test_predictor_factor_bytes(lib):
    """One fp64 factor per query head: the widest window's scaled rows and inverse diagonal."""
    cfg = L.PredCfg(16, (4, 8, 16), 1e-2)
    assert lib.asp_pred_factor_bytes(8, 32, ctypes.byref(cfg.struct)) == 8 * 32 * (16 * 16 + 16) * 8
    cfg8 = L.PredCfg(16, (4, 8), 1e-2)
    assert lib.asp_pred_factor_bytes(2, 4, ctypes.byref(cfg8.struct)) == 2 * 4 * (8 * 8 + 8) * 8
    assert lib.asp_pred_factor_bytes(0, 32, ctypes.byref(cfg.struct)) == 0
    bad = L.PredCfg(4, (8,), 1e-2)   # a window wider than the history
    assert lib.asp_pred_factor_bytes(8, 32, ctypes.byref(bad.struct)) == 0


def test_decode_step_and_wait_validation(lib):
    assert lib.asp_decode_step(None) == L.ASP_ERR_INVALID_ARG
    a = L.AspDecodeArgs()   # all zero: no query, no cache
    assert lib.asp_decode_step(ctypes.byref(a)) == L.ASP_ERR_INVALID_ARG
    assert lib.asp_wait_selection(None, 10) == L.ASP_ERR_INVALID_ARG


def test_decode_step_rejects_bad_factor_buffers(lib):
    """The predictor-factor buffers are validated on the host before any launch:
    8-byte aligned, and never the same buffer for this step and the next."""
    B, Hkv, Hq, d, C = 2, 2, 4, 128, 64
    kv = _kv(batch=B, n_kv_heads=Hkv, t_max=1024)
    cfg = L.PredCfg(8, (4, 8), 1e-2)
    a = L.AspDecodeArgs()
    a.q_t, a.q_dtype, a.n_q_heads, a.qhist, a.ring_start = FAKE, L.ASP_BF16, Hq, FAKE, 0
    a.pred, a.kv, a.C = ctypes.pointer(cfg.struct), ctypes.pointer(kv), C
    a.idx_cur = a.count_cur = a.qpred = a.scores = a.idx_next = a.count_next = a.out = FAKE
    a.workspace = 1 << 20   # 256-byte aligned, never dereferenced on the host
    a.workspace_bytes = lib.asp_decode_workspace_bytes(B, Hq, Hkv, d, C, 0)
    a.ev_fork = a.ev_sel_done = FAKE
    a.pred_factor_cur, a.pred_factor_next = (1 << 21) + 4, 1 << 22      # misaligned
    assert lib.asp_decode_step(ctypes.byref(a)) == L.ASP_ERR_INVALID_ARG
    a.pred_factor_cur, a.pred_factor_next = 1 << 21, (1 << 22) + 2
    assert lib.asp_decode_step(ctypes.byref(a)) == L.ASP_ERR_INVALID_ARG
    a.pred_factor_cur = a.pred_factor_next = 1 << 21                   # the same buffer twice
    assert lib.asp_decode_step(ctypes.byref(a)) == L.ASP_ERR_INVALID_ARG


def test_wait_limit_check_validation(lib):
    assert lib.asp_check_wait_limit(8, None, None) == L.ASP_ERR_INVALID_ARG
    assert lib.asp_check_wait_limit(0, FAKE, None) == L.ASP_ERR_INVALID_ARG
    assert lib.asp_check_wait_limit((1 << 20) + 1, FAKE, None) == L.ASP_ERR_INVALID_ARG


def test_quest_validation(lib):
    kv = _kv()
    assert lib.asp_quest_build_meta(ctypes.byref(kv), 24, FAKE, None) == L.ASP_ERR_UNSUPPORTED
    assert lib.asp_quest_build_meta(ctypes.byref(kv), 16, None, None) == L.ASP_ERR_INVALID_ARG
    kvp = _kv(page_size=32, page_table=FAKE, seq_lens=FAKE, max_pages=32, n_pages=64)
    assert lib.asp_quest_build_meta(ctypes.byref(kvp), 16, FAKE, None) == L.ASP_ERR_UNSUPPORTED   # page mismatch
    assert lib.asp_quest_select(FAKE, L.ASP_BF16, 8, ctypes.byref(kv), FAKE, 16, 0, FAKE, FAKE, FAKE, None) == \
        L.ASP_ERR_INVALID_ARG
    # the page scores alone: the same checks, less the selection's
    score = lambda kv, q=FAKE, meta=FAKE, page=16, ps=FAKE, hq=8: lib.asp_quest_page_scores(
        q, L.ASP_BF16, hq, ctypes.byref(kv), meta, page, ps, None)
    assert score(kv, q=None) == L.ASP_ERR_INVALID_ARG
    assert score(kv, meta=None) == L.ASP_ERR_INVALID_ARG
    assert score(kv, ps=None) == L.ASP_ERR_INVALID_ARG
    assert score(kv, page=24) == L.ASP_ERR_UNSUPPORTED
    assert score(kv, hq=7) == L.ASP_ERR_INVALID_ARG
    assert score(kvp) == L.ASP_ERR_UNSUPPORTED                      # bounds pages must be the cache's pages


def test_product_path_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        L.lib()
