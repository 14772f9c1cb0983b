"""ctypes binding of libasp (include/asp.h).  Argument marshalling only.

Every function here converts torch tensors to device pointers and sizes,
calls the C ABI, and raises :class:`AspError` on a non-OK status.  No step of
the method runs in Python; there is no fallback: if ``libasp.so`` is missing
the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_int32, c_long, c_size_t, c_void_p
from typing import Optional, Sequence

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libasp.so")

ASP_OK, ASP_ERR_INVALID_ARG, ASP_ERR_UNSUPPORTED, ASP_ERR_WORKSPACE, ASP_ERR_CUDA, ASP_ERR_TIMEOUT, ASP_ERR_DEVICE = range(7)
ASP_F32, ASP_BF16 = 0, 1
ASP_COEF_SOFTMAX, ASP_COEF_RAW = 0, 1
ASP_POOL_PREDICTIONS, ASP_POOL_FEATURES = 0, 1
ASP_DEV_BAD_INDEX, ASP_DEV_BAD_PAGE, ASP_DEV_WAIT_LIMIT, ASP_DEV_TAIL_LIMIT, ASP_DEV_SELECT = 1, 2, 4, 8, 16
ASP_DEV_NAN_SCORE = 32

# every entry point of include/asp.h with its ctypes signature
class AspKv(ctypes.Structure):
    _fields_ = [("batch", c_int), ("n_kv_heads", c_int), ("head_dim", c_int), ("t_max", c_int),
                ("kv_dtype", c_int), ("k", c_void_p), ("v", c_void_p), ("page_size", c_int),
                ("page_table", c_void_p), ("max_pages", c_int), ("n_pages", c_int), ("seq_lens", c_void_p)]


class AspPredCfg(ctypes.Structure):
    _fields_ = [("W", c_int), ("windows", POINTER(c_int)), ("n_windows", c_int), ("lam", c_float), ("coef", c_int),
                ("pool", c_int)]


class AspDecodeArgs(ctypes.Structure):
    _fields_ = [("q_t", c_void_p), ("q_dtype", c_int), ("n_q_heads", c_int), ("qhist", c_void_p),
                ("ring_start", c_int), ("pred", POINTER(AspPredCfg)), ("kv", POINTER(AspKv)), ("C", c_int),
                ("idx_cur", c_void_p), ("count_cur", c_void_p), ("tail_begin", c_void_p), ("max_tail", c_int),
                ("qpred", c_void_p), ("scores", c_void_p), ("idx_next", c_void_p), ("count_next", c_void_p),
                ("out", c_void_p), ("lse", c_void_p), ("workspace", c_void_p), ("workspace_bytes", c_size_t),
                ("s_main", c_void_p), ("s_side", c_void_p), ("ev_fork", c_void_p), ("ev_sel_done", c_void_p),
                ("timing", POINTER(c_void_p)), ("k_new", c_void_p), ("v_new", c_void_p), ("quest_meta", c_void_p),
                ("quest_page", c_int), ("pred_factor_cur", c_void_p), ("pred_factor_valid", c_int),
                ("pred_factor_next", c_void_p), ("ev_attend_done", c_void_p)]


SIGNATURES = {
    "asp_predict_query": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int, POINTER(AspPredCfg),
                                  c_void_p, c_void_p]),
    "asp_score_keys": (c_int, [c_void_p, c_int, POINTER(AspKv), c_void_p, c_void_p]),
    "asp_select_topk": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "asp_sparse_attend": (c_int, [c_void_p, c_int, c_int, POINTER(AspKv), c_void_p, c_void_p, c_int, c_void_p, c_int,
                                  c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "asp_attend_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
    "asp_decode_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
    "asp_pred_factor_bytes": (c_size_t, [c_int, c_int, POINTER(AspPredCfg)]),
    "asp_sparse_attend_noalloc": (c_int, [c_void_p, c_int, c_int, POINTER(AspKv), c_void_p, c_void_p, c_int, c_void_p,
                                          c_int, c_void_p, c_void_p, c_void_p]),
    "asp_decode_step": (c_int, [POINTER(AspDecodeArgs)]),
    "asp_append_kv": (c_int, [POINTER(AspKv), c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p]),
    "asp_graph_instantiate": (c_int, [c_void_p, POINTER(c_void_p)]),
    "asp_graph_launch": (c_int, [c_void_p, c_void_p]),
    "asp_graph_destroy": (c_int, [c_void_p]),
    "asp_wait_selection": (c_int, [c_void_p, c_long]),
    "asp_quest_build_meta": (c_int, [POINTER(AspKv), c_int, c_void_p, c_void_p]),
    "asp_score_keys_cuda_cores": (c_int, [c_void_p, c_int, POINTER(AspKv), c_void_p, c_void_p]),
    "asp_quest_page_scores": (c_int, [c_void_p, c_int, c_int, POINTER(AspKv), c_void_p, c_int, c_void_p, c_void_p]),
    "asp_quest_select": (c_int, [c_void_p, c_int, c_int, POINTER(AspKv), c_void_p, c_int, c_int, c_void_p, c_void_p,
                                 c_void_p, c_void_p]),
    "asp_check_wait_limit": (c_int, [c_int, c_void_p, c_void_p]),
    "asp_device_status": (c_int, [c_void_p, POINTER(c_int32)]),
    "asp_status_string": (ctypes.c_char_p, [c_int]),
    "asp_abi_version": (c_int, []),
}

_lib = None


class AspError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libasp.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m query_predicted_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().asp_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != ASP_OK:
        raise AspError(fn, status)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return ASP_F32
    if t.dtype == torch.bfloat16:
        return ASP_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


class KV:
    """A KV cache described for the C ABI (holds references to its tensors).

    Contiguous: ``k, v [B, Hkv, T, d]``.  Paged: ``k, v [n_pages, Hkv, P, d]`` with
    ``page_table [B, max_pages]`` int32 and ``seq_lens [B]`` int32.
    """

    def __init__(self, k: torch.Tensor, v: Optional[torch.Tensor], seq_lens: Optional[torch.Tensor] = None,
                 page_table: Optional[torch.Tensor] = None, t_max: Optional[int] = None, batch: Optional[int] = None):
        self.k, self.v, self.seq_lens, self.page_table = k, v, seq_lens, page_table
        d = k.shape[-1]
        if page_table is None:
            B, Hkv, T, _ = k.shape
            page_size, max_pages, n_pages = 0, 0, 0
            t_max = T if t_max is None else t_max
        else:
            n_pages, Hkv, page_size, _ = k.shape
            B, max_pages = page_table.shape
            t_max = max_pages * page_size if t_max is None else t_max
        self.struct = AspKv(int(B if batch is None else batch), int(Hkv), int(d), int(t_max), dtype_code(k),
                            _ptr(k), _ptr(v), int(page_size), _ptr(page_table), int(max_pages), int(n_pages),
                            _ptr(seq_lens))
        self.batch, self.n_kv_heads, self.head_dim, self.t_max = int(B), int(Hkv), int(d), int(t_max)
        self.page_size = int(page_size)

    @property
    def ref(self):
        return ctypes.byref(self.struct)


class PredCfg:
    """Predictor configuration.  ``coef``: "softmax" (the method's normalisation) or
    "raw"; ``pool``: "predictions" (average the windows' predictions, the default
    reading) or "features" (regress on the windows' pooled features)."""

    def __init__(self, W: int, windows: Sequence[int], lam: float, coef: str = "softmax",
                 pool: str = "predictions"):
        if coef not in ("softmax", "raw") or pool not in ("predictions", "features"):
            raise ValueError(f"coef {coef!r}, pool {pool!r}")
        self._win = (c_int * len(windows))(*[int(w) for w in windows])
        self.struct = AspPredCfg(int(W), ctypes.cast(self._win, POINTER(c_int)), len(windows), float(lam),
                                 ASP_COEF_RAW if coef == "raw" else ASP_COEF_SOFTMAX,
                                 ASP_POOL_FEATURES if pool == "features" else ASP_POOL_PREDICTIONS)
        self.W = int(W)

    @property
    def ref(self):
        return ctypes.byref(self.struct)


def predict_query(qhist: torch.Tensor, ring_start: int, cfg: PredCfg, qpred: torch.Tensor,
                  q_new: Optional[torch.Tensor] = None, stream=None) -> None:
    B, Hq, _, d = qhist.shape
    qd = dtype_code(q_new) if q_new is not None else ASP_F32
    _check("asp_predict_query", lib().asp_predict_query(_ptr(qhist), int(ring_start), _ptr(q_new), qd, B, Hq, d,
                                                        cfg.ref, _ptr(qpred), _stream(stream)))


def score_keys(qpred: torch.Tensor, kv: KV, scores: torch.Tensor, stream=None) -> None:
    _check("asp_score_keys", lib().asp_score_keys(_ptr(qpred), qpred.shape[1], kv.ref, _ptr(scores), _stream(stream)))


def score_keys_cuda_cores(qpred: torch.Tensor, kv: KV, scores: torch.Tensor, stream=None) -> None:
    """The key scan on the CUDA cores (the tensor-core scan's comparison for bf16 keys)."""
    _check("asp_score_keys_cuda_cores", lib().asp_score_keys_cuda_cores(
        qpred.data_ptr(), qpred.shape[1], kv.ref, scores.data_ptr(), _stream(stream)))


def select_topk(scores: torch.Tensor, seq_lens: Optional[torch.Tensor], C: int, idx: torch.Tensor,
                count: torch.Tensor, stream=None) -> None:
    B, H, T = scores.shape
    _check("asp_select_topk", lib().asp_select_topk(_ptr(scores), _ptr(seq_lens), B, H, T, int(C), _ptr(idx),
                                                    _ptr(count), _stream(stream)))


def attend_workspace_bytes(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int, C: int, max_tail: int = 0) -> int:
    return int(lib().asp_attend_workspace_bytes(batch, n_q_heads, n_kv_heads, head_dim, int(C), int(max_tail)))


def sparse_attend(q: torch.Tensor, kv: KV, idx: Optional[torch.Tensor], count: Optional[torch.Tensor], C: int,
                  out: torch.Tensor, lse: Optional[torch.Tensor] = None, tail_begin: Optional[torch.Tensor] = None,
                  max_tail: int = 0, workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("asp_sparse_attend", lib().asp_sparse_attend(_ptr(q), dtype_code(q), q.shape[1], kv.ref, _ptr(idx),
                                                        _ptr(count), int(C), _ptr(tail_begin), int(max_tail),
                                                        _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
                                                        _stream(stream)))


def sparse_attend_noalloc(q: torch.Tensor, kv: KV, idx: Optional[torch.Tensor], count: Optional[torch.Tensor],
                          C: int, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                          tail_begin: Optional[torch.Tensor] = None, max_tail: int = 0, stream=None) -> None:
    """Step 4 for callers that cannot allocate: the split-K partials go to the
    library's fixed scratch array instead of a workspace tensor."""
    _check("asp_sparse_attend_noalloc", lib().asp_sparse_attend_noalloc(
        _ptr(q), dtype_code(q), q.shape[1], kv.ref, _ptr(idx), _ptr(count), int(C), _ptr(tail_begin),
        int(max_tail), _ptr(out), _ptr(lse), _stream(stream)))


def quest_build_meta(kv: KV, quest_page: int, meta: torch.Tensor, stream=None) -> None:
    _check("asp_quest_build_meta", lib().asp_quest_build_meta(kv.ref, int(quest_page), _ptr(meta), _stream(stream)))


def quest_page_scores(q: torch.Tensor, kv: KV, meta: torch.Tensor, quest_page: int, page_scores: torch.Tensor,
                      stream=None) -> None:
    """Page bounds of every page with the current query (the scan half of quest_select)."""
    _check("asp_quest_page_scores", lib().asp_quest_page_scores(
        q.data_ptr(), dtype_code(q), q.shape[1], kv.ref, meta.data_ptr(), int(quest_page),
        page_scores.data_ptr(), _stream(stream)))


def quest_select(q: torch.Tensor, kv: KV, meta: torch.Tensor, quest_page: int, C: int, page_scores: torch.Tensor,
                 idx: torch.Tensor, count: torch.Tensor, stream=None) -> None:
    _check("asp_quest_select", lib().asp_quest_select(_ptr(q), dtype_code(q), q.shape[1], kv.ref, _ptr(meta),
                                                      int(quest_page), int(C), _ptr(page_scores), _ptr(idx),
                                                      _ptr(count), _stream(stream)))


def append_kv(kv: KV, k_new: torch.Tensor, v_new: torch.Tensor, tail_begin: Optional[torch.Tensor] = None,
              quest_meta: Optional[torch.Tensor] = None, quest_page: int = 16, stream=None) -> None:
    """Appends one token per sequence (``k_new, v_new [B, Hkv, d]``) at position
    ``seq_lens[b]`` and advances ``kv.seq_lens`` on the device; ``tail_begin`` gets the
    old lengths; ``quest_meta`` (page bounds) is kept current."""
    _check("asp_append_kv", lib().asp_append_kv(kv.ref, _ptr(k_new), _ptr(v_new), _ptr(tail_begin),
                                                _ptr(quest_meta), int(quest_page), _stream(stream)))


def check_wait_limit(tries: int, returned: torch.Tensor, stream=None) -> None:
    """Runs the bounded-wait check (see asp.h): ``returned`` int32 [1] gets 1 when the wait gave up."""
    _check("asp_check_wait_limit", lib().asp_check_wait_limit(int(tries), returned.data_ptr(), _stream(stream)))


def device_status(stream=None) -> int:
    """Returns (and clears) the device status bits; 0 when no kernel recorded a fault."""
    bits = c_int32(0)
    st = lib().asp_device_status(_stream(stream), ctypes.byref(bits))
    if st not in (ASP_OK, ASP_ERR_DEVICE):
        raise AspError("asp_device_status", st)
    return int(bits.value)


def wait_selection(event: "torch.cuda.Event", timeout_us: int) -> int:
    """Returns ASP_OK or ASP_ERR_TIMEOUT (raises on other statuses)."""
    st = lib().asp_wait_selection(event_handle(event), int(timeout_us))
    if st not in (ASP_OK, ASP_ERR_TIMEOUT):
        raise AspError("asp_wait_selection", st)
    return st


def make_event(timing: bool = False) -> "torch.cuda.Event":
    """A CUDA event whose handle exists (torch creates it lazily on first record)."""
    ev = torch.cuda.Event(enable_timing=timing)
    ev.record()
    return ev


def event_handle(ev) -> int:
    return int(ev.cuda_event)


class DecodeState:
    """Buffers of the asynchronous decode loop: the query ring, double-buffered
    selections, scratch for the side stream, attention workspace, two streams and
    two events.  :meth:`step` is one ``asp_decode_step`` call.  With
    ``precompute_factor`` each step also factorises the next step's lag Gram beside
    its key scan (two double-buffered factor buffers), so that the next step's
    predictor only substitutes; after changing ``qhist`` or ``ring_start`` outside
    :meth:`step`, call :meth:`invalidate_factor`."""

    def __init__(self, kv: KV, n_q_heads: int, cfg: PredCfg, C: int, qhist: torch.Tensor, max_tail: int = 0,
                 tail_begin: Optional[torch.Tensor] = None, s_main=None, s_side=None, timing: bool = False,
                 precompute_factor: bool = True):
        dev = kv.k.device
        B, Hkv, d = kv.batch, kv.n_kv_heads, kv.head_dim
        self.kv, self.cfg, self.C, self.n_q_heads = kv, cfg, int(C), int(n_q_heads)
        self.qhist = qhist
        self.ring_start = 0
        self.tail_begin, self.max_tail = tail_begin, int(max_tail)
        self.qpred = torch.empty(B, n_q_heads, d, dtype=torch.float32, device=dev)
        self.scores = torch.empty(B, Hkv, kv.t_max, dtype=torch.float32, device=dev)
        self.idx = [torch.full((B, Hkv, C), -1, dtype=torch.int32, device=dev) for _ in range(2)]
        self.count = [torch.zeros(B, Hkv, dtype=torch.int32, device=dev) for _ in range(2)]
        self.cur = 0
        ws = int(lib().asp_decode_workspace_bytes(B, n_q_heads, Hkv, d, C, max_tail if tail_begin is not None else 0))
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
        fb = int(lib().asp_pred_factor_bytes(B, n_q_heads, ctypes.byref(cfg.struct))) if precompute_factor else 0
        self.pred_factor = [torch.empty(fb // 8, dtype=torch.float64, device=dev) for _ in range(2)] if fb else None
        self._factor_valid = False
        self.s_main = s_main or torch.cuda.current_stream()
        # the selection chain is the step's critical path: give it the highest priority
        self.s_side = s_side or torch.cuda.Stream(priority=-100)
        self.ev_fork = make_event()
        self.ev_sel_done = make_event()
        # recorded when the step's output is written (a read-back may start there)
        self.ev_attend_done = make_event()
        self.timing_events = [make_event(True) for _ in range(8)] if timing else None
        self._timing_arr = (c_void_p * 8)(*[event_handle(e) for e in self.timing_events]) if timing else None

        self._args = [self._build_args(0), self._build_args(1)]
        self._fn = lib().asp_decode_step

    def _build_args(self, cur: int) -> AspDecodeArgs:
        """The call's arguments for one parity of the double-buffered selection."""
        nxt = 1 - cur
        a = AspDecodeArgs()
        a.n_q_heads = self.n_q_heads
        a.qhist = _ptr(self.qhist)
        a.pred = ctypes.pointer(self.cfg.struct)
        a.kv = ctypes.pointer(self.kv.struct)
        a.C = self.C
        a.idx_cur = _ptr(self.idx[cur])
        a.count_cur = _ptr(self.count[cur])
        a.tail_begin = _ptr(self.tail_begin)
        a.max_tail = self.max_tail
        a.qpred = _ptr(self.qpred)
        a.scores = _ptr(self.scores)
        a.idx_next = _ptr(self.idx[nxt])
        a.count_next = _ptr(self.count[nxt])
        a.workspace = _ptr(self.workspace)
        a.workspace_bytes = self.workspace.numel()
        a.s_main = _stream(self.s_main)
        a.s_side = _stream(self.s_side)
        a.ev_fork = event_handle(self.ev_fork)
        a.ev_sel_done = event_handle(self.ev_sel_done)
        a.ev_attend_done = event_handle(self.ev_attend_done)
        a.timing = ctypes.cast(self._timing_arr, POINTER(c_void_p)) if self._timing_arr is not None else None
        if self.pred_factor is not None:
            a.pred_factor_cur = _ptr(self.pred_factor[cur])
            a.pred_factor_next = _ptr(self.pred_factor[nxt])
        return a

    def invalidate_factor(self) -> None:
        """The next step factorises in full (the stored factor no longer matches the ring)."""
        self._factor_valid = False

    def set_timing(self, on: bool) -> None:
        """Record the per-kernel timing events in later steps (they sit between the
        side stream's kernels, so they also keep those kernels from overlapping)."""
        if on and self._timing_arr is None:
            raise ValueError("DecodeState was created without timing events")
        ptr = ctypes.cast(self._timing_arr, POINTER(c_void_p)) if on else None
        for a in self._args:
            a.timing = ptr

    def set_selection(self, idx: torch.Tensor, count: torch.Tensor) -> None:
        self.idx[self.cur].copy_(idx)
        self.count[self.cur].copy_(count)

    def step(self, q_t: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
             k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
             quest_meta: Optional[torch.Tensor] = None, quest_page: int = 16) -> None:
        """One decode step; with ``k_new``/``v_new`` the new token is appended first
        (``kv.seq_lens`` and ``tail_begin`` are then updated on the device)."""
        a = self._args[self.cur]
        a.q_t = q_t.data_ptr()
        a.q_dtype = dtype_code(q_t)
        a.out = out.data_ptr()
        a.lse = lse.data_ptr() if lse is not None else None
        a.ring_start = self.ring_start
        a.k_new = _ptr(k_new)
        a.v_new = _ptr(v_new)
        a.quest_meta = _ptr(quest_meta)
        a.quest_page = int(quest_page)
        a.pred_factor_valid = 1 if self._factor_valid else 0
        _check("asp_decode_step", self._fn(ctypes.byref(a)))
        self._factor_valid = self.pred_factor is not None
        self.cur = 1 - self.cur
        self.ring_start = (self.ring_start + 1) % (self.cfg.W + 1)

    # ---- CUDA graphs -------------------------------------------------------
    def capture(self, q_t: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
                quest_meta: Optional[torch.Tensor] = None, quest_page: int = 16) -> int:
        """Captures one CUDA graph per state of the step cycle (selection parity x
        ring position: lcm(2, W + 1) graphs), starting from the current state, each
        one :meth:`step` on these fixed buffers (write each step's query, and K/V when
        appending, into them before :meth:`replay`).  Run one eager :meth:`step` first
        (the library prepares its kernels on first use).  Returns the cycle length."""
        import math
        n = 2 * (self.cfg.W + 1) // math.gcd(2, self.cfg.W + 1)
        cur0, ring0, fv0 = self.cur, self.ring_start, self._factor_valid
        main0 = self.s_main
        timing_on = bool(self._args[0].timing)
        cap = torch.cuda.Stream(device=self.kv.k.device)
        self.graphs = []
        try:
            self.s_main = cap
            self._args = [self._build_args(0), self._build_args(1)]
            for a in self._args:   # no timing events inside a graph
                a.timing = None
            for _ in range(n):
                g = torch.cuda.CUDAGraph(keep_graph=True)
                with torch.cuda.graph(g, stream=cap):
                    self.step(q_t, out, lse, k_new, v_new, quest_meta, quest_page)
                    cap.wait_event(self.ev_sel_done)   # the graph joins the side stream
                ex = c_void_p()
                _check("asp_graph_instantiate", lib().asp_graph_instantiate(c_void_p(g.raw_cuda_graph()),
                                                                            ctypes.byref(ex)))
                self.graphs.append((g, ex))
        finally:
            self.s_main = main0
            self._args = [self._build_args(0), self._build_args(1)]
            self.set_timing(timing_on) if self._timing_arr is not None else None
            self.cur, self.ring_start, self._factor_valid = cur0, ring0, fv0
        # the events were last recorded inside the captures: record them once outside
        self.ev_fork.record(self.s_main)
        self.ev_sel_done.record(self.s_main)
        self.ev_attend_done.record(self.s_main)
        self._graph_at = 0
        return n

    def release_graphs(self) -> None:
        for _, ex in getattr(self, "graphs", []):
            lib().asp_graph_destroy(ex)
        self.graphs = []

    def replay(self) -> None:
        """One step by replaying the captured graph of the current state on the
        current stream (the graphs must have been captured from this state on)."""
        _check("asp_graph_launch", lib().asp_graph_launch(self.graphs[self._graph_at][1],
                                                          _stream(torch.cuda.current_stream())))
        self._graph_at = (self._graph_at + 1) % len(self.graphs)
        self._factor_valid = self.pred_factor is not None
        self.cur = 1 - self.cur
        self.ring_start = (self.ring_start + 1) % (self.cfg.W + 1)

    @property
    def selection(self):
        """The selection written by the latest step (for the next step)."""
        return self.idx[self.cur], self.count[self.cur]
