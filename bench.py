#!/usr/bin/env python
"""Benchmark of one asynchronous predicted-query sparse decode step on B200.

A step is one ``asp_decode_step``: attention of step t over the selected K/V
(main stream) while the query predictor, the scan of every cached key and the
top-C selection for step t+1 run on a side stream.  Default workload: Qwen3-8B
head geometry, batch 8, 32768 cached tokens, C = 2048 (bf16 KV, synthetic).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  ``value`` is the step's algorithmic HBM bytes
over its device time (GB/s, all ranks' bytes over the slowest rank's time);
``ms_per_step`` is the mean step time.  N > 1 runs one replica per GPU (each
rank decodes its own batch; the path has no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse decode step µs and KV-scan HBM GB/s (fraction of B200 peak) at 32k ctx"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 512 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="qwen3_8b_shaped_32k")
    ap.add_argument("--impl", default="asp", choices=["asp", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-compare", action="store_true",
                    help="skip the page-level and full-attention timings and the selection recall")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the records of the other decode workloads (32B shapes, ragged paged batch)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--layers", type=int, default=36,
                    help="also time a stack of this many layers (each with its own cache), steady-state period "
                         "(1: no stack)")
    ap.add_argument("--profile", default=None, choices=["scan", "scan_cuda_cores", "attend", "page_scan", "decode"],
                    help="only build the workload and launch this kernel --steps times (for ncu captures); "
                         "prints no JSON line")
    ap.add_argument("--side-streams", type=int, default=1,
                    help="with --layers: side streams the layers' selection chains alternate over")
    return ap.parse_args()


# ----------------------------------------------------------------------------- accounting
def step_bytes(wl, lens):
    """Algorithmic HBM bytes of one decode step (what the method must move)."""
    e = 2 if wl.kv_dtype == "bf16" else 4
    B, Hq, Hkv, d, C, W = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.C, wl.W
    tok = sum(int(t) for t in lens)                       # cached tokens over the batch
    predict = B * Hq * (W + 1) * d * 4 + B * Hq * d * (4 + e) + B * Hq * d * 4
    score = tok * Hkv * d * e + tok * Hkv * 4 + B * Hq * d * 4
    sel_units = sum(min(C, int(t)) for t in lens) * Hkv
    select = tok * Hkv * 4 + B * Hkv * C * 4
    attend = sel_units * d * e * 2 + B * Hq * d * (e + e + 4) + B * Hkv * C * 4
    return dict(predict=predict, score=score, select=select, attend=attend,
                total=predict + score + select + attend)


QUEST_PAGE = 16


def quest_step_bytes(wl, lens):
    """Algorithmic HBM bytes of one step of the page-level comparison path: the
    per-page key bounds (min and max rows), the page scores written and read back,
    the chosen pages' indices, and the attention over the chosen tokens."""
    e = 2 if wl.kv_dtype == "bf16" else 4
    B, Hq, Hkv, d, C = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.C
    pages = sum(math.ceil(int(t) / QUEST_PAGE) for t in lens) * Hkv
    cp = math.ceil(C / QUEST_PAGE) * QUEST_PAGE
    scan = pages * 2 * d * e + pages * 4 + B * Hq * d * e
    select = pages * 4 + B * Hkv * cp * 4
    sel_units = sum(min(cp, int(t)) for t in lens) * Hkv
    attend = sel_units * d * e * 2 + B * Hq * d * (e + e) + B * Hkv * cp * 4
    return dict(scan=scan, select=select, attend=attend, total=scan + select + attend)


def dense_bytes(wl, lens):
    """Full attention over every cached token: every K and V row once."""
    e = 2 if wl.kv_dtype == "bf16" else 4
    tok = sum(int(t) for t in lens)
    return tok * wl.n_kv_heads * wl.head_dim * e * 2 + wl.batch * wl.n_q_heads * wl.head_dim * (e + e)


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def read_traffic(kernel_file: str, launch_units: float, summary: str = "score_keys_qwen3_8b_shaped_32k.txt"):
    """Per-launch DRAM bytes of a kernel from its committed ncu summary (scaled by
    ``launch_units``), if the summary was taken on the kernel's current source (else None)."""
    import hashlib
    src = os.path.join(ROOT, "query_predicted_token_b200", "csrc", kernel_file)
    summ = os.path.join(ROOT, "profiles", summary)
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        kv = {}
        for line in open(summ):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("source_sha256_16") != h:
            return None
        return float(kv["dram_bytes_per_launch"]) * launch_units
    except Exception:
        return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id, self.proc, self.path = gpu_id, None, None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        except Exception:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU baseline
def cpu_sample(wl, kv_host, qhist, q_t, idx0, cnt0, units):
    """The oracle on a bounded sample: full steps 1-4 for the given (b, h) units."""
    import numpy as np
    import oracle
    G = wl.n_q_heads // wl.n_kv_heads
    for b, h in units:
        K, V, Tb = kv_host(b, h)
        hs = qhist[b, h * G:(h + 1) * G]
        hist = np.concatenate([hs[:, 1:], q_t[b, h * G:(h + 1) * G, None]], axis=1)
        qp = oracle.predict_query(hist, wl.windows, wl.lam)
        s = oracle.score_row(qp, K).astype(np.float32)
        oracle.select_row(s, Tb, wl.C)
        oracle.attend_set(q_t[b, h * G:(h + 1) * G], K, V, idx0[b, h, :cnt0[b, h]])


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(wl, seconds, seed=0):
    """Times the oracle on whole (sequence, KV head) units of the workload until
    ``seconds`` elapse; returns (GB/s of the step's algorithmic bytes, sample text)."""
    import numpy as np
    import torch
    import synth
    rng = np.random.default_rng(seed)
    B, Hkv, d, T = wl.batch, wl.n_kv_heads, wl.head_dim, wl.t_max
    qhist, q_next = synth.query_history(wl, 1)
    qhist = qhist.double().numpy()
    q_t = q_next[0].to(wl.torch_dtype()).double().numpy()
    lens = synth.workloads.sequence_lengths(wl).tolist()
    idx0, cnt0 = synth.random_selection(B, Hkv, wl.C, lens, seed=wl.seed + 99)
    idx0, cnt0 = idx0.numpy(), cnt0.numpy()
    scale = synth.workloads.key_channel_scale(wl)
    # a fixed pool of four units drawn once (CPU generator; same shapes and distribution
    # as the GPU draw, different values), cycled through while the oracle is timed
    pool = {}
    for n in range(4):
        b, h = int(rng.integers(B)), int(rng.integers(Hkv))
        g = torch.Generator().manual_seed(wl.seed * 7919 + b * 31 + h)
        Tb = lens[b]
        K = (torch.randn(Tb, d, generator=g) * scale[h]).to(wl.torch_dtype()).double().numpy()
        V = torch.randn(Tb, d, generator=g).to(wl.torch_dtype()).double().numpy()
        pool[(b, h)] = (K, V, Tb)
    keys = list(pool)

    def kv_host(b, h):
        return pool[(b, h)]

    units_done, t_spent, bytes_done = 0, 0.0, 0.0
    per_unit_frac = 1.0 / (B * Hkv)
    total = step_bytes(wl, lens)["total"]
    while t_spent < seconds:
        b, h = keys[units_done % len(keys)]
        t0 = time.perf_counter()
        cpu_sample(wl, kv_host, qhist, q_t, idx0, cnt0, [(b, h)])
        t_spent += time.perf_counter() - t0
        units_done += 1
        bytes_done += total * per_unit_frac * (lens[b] / (sum(lens) / B))
    gbs = bytes_done / t_spent / 1e9
    sample = (f"{units_done} whole (sequence, KV head) units of {wl.name} (predict {wl.group} heads, score "
              f"all T_b keys, select C={wl.C}, attend), {t_spent:.1f} s of oracle time, float64 NumPy")
    return gbs, sample, units_done, t_spent


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synth.workload(args.workload)
    lens = synth.workloads.sequence_lengths(wl).tolist()
    total = step_bytes(wl, lens)["total"]
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    time_oracle(wl, min(2.0, per_step), seed=1)   # warm-up
    vals = []
    for k in range(args.steps):
        gbs, sample, n, t = time_oracle(wl, per_step, seed=100 + k)
        vals.append(gbs)
    value = statistics.mean(vals)
    step_s = total / (value * 1e9)
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "batch": wl.batch, "n_q_heads": wl.n_q_heads,
                       "n_kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "T": wl.t_max, "C": wl.C},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"each step: {sample}"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- timing helpers
L2_BYTES = 126 << 20


def rotation_count(bytes_per_launch: float) -> int:
    """Copies of a kernel's input to rotate over, so that between two launches that
    read the same copy the other launches stream at least twice the L2 through it:
    no launch can find the rows of an earlier one in L2."""
    return max(2, min(8, math.ceil(2 * L2_BYTES / max(1.0, bytes_per_launch)) + 1))


def time_rotating(fn, copies, stream, reps):
    """Mean µs per launch of ``fn(copy)`` over ``reps`` back-to-back launches that
    cycle through ``copies``, between two CUDA events on ``stream``."""
    import torch
    with torch.cuda.stream(stream):
        for c in copies:                       # every copy once, untimed
            fn(c)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(reps):
            fn(copies[i % len(copies)])
        b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1e3 / reps


def time_cold(fn, stream, flush, reps):
    """Median µs of single launches, each after an L2 flush (outside its events);
    an event pair alone measures ~5-6 µs on this part, so this is an upper bound."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for k in range(reps):
            flush.zero_()
            ev[k][0].record(stream)
            fn()
            ev[k][1].record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) * 1e3 for a, b in ev)


def roofline_entry(kernel, nbytes, us_rot, us_cold, peak, peak_kind, timed, traffic=None, extra=None):
    achieved = nbytes / (us_rot / 1e6) / 1e9
    d = {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
         "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic, "algorithmic_bytes": int(nbytes),
         "us": round(us_rot, 2), "cold_us": round(us_cold, 2),
         "cold_frac": round(nbytes / (us_cold / 1e6) / 1e9 / peak, 4), "timed": timed}
    if extra:
        d.update(extra)
    return d


def clone_kv(asp, kvd, wl, with_v=True):
    """Another cache of the same shapes (values copied), for rotation."""
    k2 = kvd["k"].clone()
    v2 = kvd["v"].clone() if with_v else kvd["v"]
    return asp.KV(k2, v2, kvd["seq_lens"], kvd["page_table"], t_max=wl.t_max), (k2, v2)


# ----------------------------------------------------------------------------- one decode workload
def decode_record(wl, dev, args, flush, peak, peak_kind, *, headline, group=None):
    """Times the decode step of a workload and its two roofline kernels.

    Returns (record, extras): the record for the JSON line; extras holds the objects
    the headline reuses (cache, query, state) and the per-step e2e numbers."""
    import torch
    import query_predicted_token_b200 as asp
    import synth
    B, Hq, Hkv, d, C = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.C
    e = 2 if wl.kv_dtype == "bf16" else 4
    steps = args.steps if headline else max(3, min(args.steps, 10))
    kvd = synth.kv_cache(wl, dev)
    lens = kvd["seq_lens"].cpu().tolist()
    paged = kvd["page_table"] is not None
    tail = 1 if paged else 0
    kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], kvd["page_table"], t_max=wl.t_max)
    qhist, q_next = synth.query_history(wl, steps=1)
    q_host = q_next[0].to(wl.torch_dtype()).pin_memory()
    q_t = q_host.to(dev)
    tail_begin = (kvd["seq_lens"] - tail).clamp(min=0).to(torch.int32) if tail else None
    snap = (torch.tensor(lens) - tail).tolist() if tail else lens
    idx0, cnt0 = synth.random_selection(B, Hkv, C, snap, seed=wl.seed + 99)
    st = asp.DecodeState(kv, Hq, asp.PredCfg(wl.W, wl.windows, wl.lam), C, qhist.to(dev).contiguous(),
                         max_tail=tail, tail_begin=tail_begin, timing=True)
    st.set_selection(idx0.to(dev), cnt0.to(dev))
    out = torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=dev)
    out_host = torch.empty_like(out, device="cpu").pin_memory()
    lse = torch.empty(B, Hq, device=dev)
    s_main = st.s_main
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    acct = step_bytes(wl, lens)

    copy_stream = torch.cuda.Stream(device=dev)

    def one_step(state, k=None, e2e=False):
        with torch.cuda.stream(s_main):
            flush.zero_()                                   # L2 flush, outside the timed events
            if k is not None:
                ev[k][0].record(s_main)
            if e2e:
                q_t.copy_(q_host, non_blocking=True)
            state.step(q_t, out, lse)
            if e2e:   # the output is ready when the attention ends: read it back while the selection runs
                copy_stream.wait_event(state.ev_attend_done)
                with torch.cuda.stream(copy_stream):
                    out_host.copy_(out, non_blocking=True)
                s_main.wait_stream(copy_stream)
            s_main.wait_event(state.ev_sel_done)
            if k is not None:
                ev[k][1].record(s_main)

    for _ in range(max(3, args.warmup)):
        one_step(st)
    torch.cuda.synchronize()
    if group is not None:
        group.barrier()
    # timed steps: no events between the kernels, so each kernel of the side
    # stream may launch while the previous one drains
    st.set_timing(False)
    torch.cuda.synchronize()
    for k in range(steps):
        one_step(st, k)
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    # the same steps again with events around every kernel, for the per-kernel times
    kern_ms = {n: [] for n in ("predict", "score", "select", "attend")}
    st.set_timing(True)
    for k in range(steps):
        one_step(st)
        torch.cuda.synchronize()
        te = st.timing_events
        for i, n in enumerate(("predict", "score", "select", "attend")):
            kern_ms[n].append(te[2 * i].elapsed_time(te[2 * i + 1]))
    st.set_timing(False)
    assert asp.device_status() == 0
    e2e_ms = None
    if headline:
        for k in range(steps):
            one_step(st, k, e2e=True)
        torch.cuda.synchronize()
        e2e_ms = [a.elapsed_time(b) for a, b in ev]
    serial_us = None
    if paged:
        # the same kernels on one stream: what the side stream buys on one GPU
        st1 = asp.DecodeState(kv, Hq, asp.PredCfg(wl.W, wl.windows, wl.lam), C, qhist.to(dev).contiguous(),
                              max_tail=tail, tail_begin=tail_begin, s_main=s_main, s_side=s_main)
        st1.set_selection(idx0.to(dev), cnt0.to(dev))
        for _ in range(max(3, args.warmup)):
            one_step(st1)
        for k in range(steps):
            one_step(st1, k)
        torch.cuda.synchronize()
        serial_us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3
        del st1
    # ---- the key scan alone: the same kernel and grid through asp_score_keys,
    # alternating between two copies of the keys
    kv2, keep2 = clone_kv(asp, kvd, wl, with_v=False)

    def scan(kvx):
        asp.score_keys(st.qpred, kvx, st.scores, stream=s_main)
    scan_rot = time_rotating(scan, [kv, kv2], s_main, max(10, steps))
    scan_cold = time_cold(lambda: scan(kv), s_main, flush, max(10, steps))
    del kv2, keep2
    assert asp.device_status() == 0
    # ---- the sparse attention alone (its stand-alone plan), rotating over copies of the cache
    sel_idx, sel_cnt = st.selection
    att_bytes = int(sel_cnt.sum().item()) * 2 * d * e + (B * Hkv * tail * 2 * d * e)
    att_ws = torch.empty(max(16, int(asp.lib().asp_attend_workspace_bytes(B, Hq, Hkv, d, C, tail))),
                         dtype=torch.uint8, device=dev)
    R = rotation_count(att_bytes)
    copies, keep = [kv], []
    for _ in range(R - 1):
        kvx, kk = clone_kv(asp, kvd, wl)
        copies.append(kvx)
        keep.append(kk)

    def attend(kvx):
        asp.sparse_attend(q_t, kvx, sel_idx, sel_cnt, C, out, None, tail_begin, tail, att_ws, stream=s_main)
    att_rot = time_rotating(attend, copies, s_main, max(10, steps))
    att_cold = time_cold(lambda: attend(kv), s_main, flush, max(10, steps))
    del copies, keep
    torch.cuda.empty_cache()
    assert asp.device_status() == 0

    # the stand-alone plan runs the persistent gather kernel from 200 16-row tiles per SM up
    # (148 SMs, C + tail rows a unit, a tail of at most max(C, 4096)), the per-item kernel otherwise:
    # three 4-warp CTAs per SM, splits of a multiple of 64 rows, merged inside a thread-block
    # cluster when there are 4 to 8 of them, else by the merge kernel
    att_tiles = B * Hkv * ((C + tail + 15) // 16)
    att_splits = -(-(C + tail) // (-(-(-(-(C + tail) // max(1, 444 // (B * Hkv)))) // 64) * 64))
    att_kernel = ("attend_gather_kernel (+ merge)" if att_tiles >= 200 * 148 and tail <= max(C, 4096)
                  else "attend_mma_kernel (cluster merge)" if 4 <= att_splits <= 8
                  else "attend_mma_kernel (+ merge)")
    step_us = statistics.mean(step_ms) * 1e3
    gbs = acct["total"] / (step_us / 1e6) / 1e9
    traffic = read_traffic("asp_score_tc.cu", 1.0) if wl.name == "qwen3_8b_shaped_32k" else None
    rot_note = "back-to-back launches cycling through {n} copies of the {what} (no launch finds an earlier launch's data in L2)"
    rec = {
        "workload": wl.name,
        "config": {"batch": B, "n_q_heads": Hq, "n_kv_heads": Hkv, "head_dim": d, "T": wl.t_max,
                   "t_min": wl.t_min, "ragged": wl.ragged, "paged": paged, "C": C, "W": wl.W,
                   "windows": list(wl.windows), "lambda": wl.lam, "tail": tail},
        "steps": steps,
        "step_us": round(step_us, 2),
        "step_us_p90": round(sorted(step_ms)[int(0.9 * (len(step_ms) - 1))] * 1e3, 2),
        "gbs": round(gbs, 1),
        "step_bytes": acct["total"],
        "step_frac_of_peak": round(gbs / peak, 4),
        "ideal_step_us": round(acct["total"] / (peak * 1e9) * 1e6, 2),
        "kernel_us": {n: round(statistics.mean(v) * 1e3, 2) for n, v in kern_ms.items()},
        "roofline": roofline_entry("score_tc_kernel (key scan)", acct["score"], scan_rot, scan_cold, peak, peak_kind,
                                   rot_note.format(n=2, what="keys") + "; cold: one launch after an L2 flush",
                                   traffic=traffic,
                                   extra={"in_step_frac": round(acct["score"] / (statistics.mean(kern_ms["score"]) / 1e3) / 1e9 / peak, 4)}),
        "roofline_attend": roofline_entry(att_kernel + " (sparse attention, stand-alone plan)",
                                          att_bytes, att_rot, att_cold, peak, peak_kind,
                                          rot_note.format(n=R, what="K/V cache") + "; cold: one launch after an L2 flush"),
    }
    if serial_us is not None:
        rec["serial_step_us"] = round(serial_us, 2)
        rec["overlap_gain_us"] = round(serial_us - step_us, 2)
    extras = dict(kvd=kvd, kv=kv, q_t=q_t, q_host=q_host, out=out, st=st, s_main=s_main, e2e_ms=e2e_ms,
                  step_ms=step_ms, acct=acct, lens=lens,
                  h2d=q_host.numel() * q_host.element_size(), d2h=out.numel() * out.element_size())
    return rec, extras


# ----------------------------------------------------------------------------- comparison paths
def page_level_record(wl, kvd, kv, q_dev, stream, flush, steps, peak, peak_kind):
    """The page-level comparison path on the given cache and query: page bounds
    scanned with the current query, the best ceil(C/16) pages kept, attention over
    their tokens.  The bounds are built once beforehand (a serving system keeps them
    current as tokens arrive).  Step time, and the page-bound scan's roofline."""
    import torch
    import query_predicted_token_b200 as asp
    B, Hq, Hkv, d, C = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.C
    e = 2 if wl.kv_dtype == "bf16" else 4
    dev = kvd["k"].device
    lens = kvd["seq_lens"].cpu().tolist()
    npm = math.ceil(wl.t_max / QUEST_PAGE)
    cp = math.ceil(C / QUEST_PAGE) * QUEST_PAGE
    meta = torch.empty(B, Hkv, npm, 2, d, dtype=wl.torch_dtype(), device=dev)
    ps = torch.empty(B, Hkv, npm, device=dev)
    qidx = torch.empty(B, Hkv, cp, dtype=torch.int32, device=dev)
    qcnt = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=dev)
    ws_q = torch.empty(max(16, asp.attend_workspace_bytes(B, Hq, Hkv, d, cp)), dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        asp.quest_build_meta(kv, QUEST_PAGE, meta, stream=stream)

    def quest_step():
        asp.quest_select(q_dev, kv, meta, QUEST_PAGE, C, ps, qidx, qcnt, stream=stream)
        asp.sparse_attend(q_dev, kv, qidx, qcnt, cp, out, workspace=ws_q, stream=stream)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for k in range(-3, steps):
            flush.zero_()
            if k >= 0:
                ev[k][0].record(stream)
            quest_step()
            if k >= 0:
                ev[k][1].record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    nbytes = quest_step_bytes(wl, lens)
    # the page-bound scan alone, rotating over copies of the bounds
    scan_bytes = nbytes["scan"]
    R = rotation_count(scan_bytes)
    metas = [meta] + [meta.clone() for _ in range(R - 1)]

    def bound_scan(m):
        asp.quest_page_scores(q_dev, kv, m, QUEST_PAGE, ps, stream=stream)
    scan_rot = time_rotating(bound_scan, metas, stream, max(10, steps))
    scan_cold = time_cold(lambda: bound_scan(meta), stream, flush, max(10, steps))
    del metas
    assert asp.device_status() == 0
    return {
        "workload": "quest_page_scan_8b_32k",
        "config": {"batch": B, "n_q_heads": Hq, "n_kv_heads": Hkv, "head_dim": d, "T": wl.t_max, "C": C,
                   "page": QUEST_PAGE, "pages_kept": cp // QUEST_PAGE},
        "step_us": round(ms * 1e3, 2), "gbs": round(nbytes["total"] / (ms / 1e3) / 1e9, 1),
        "step_bytes": nbytes["total"], "step_frac_of_peak": round(nbytes["total"] / (ms / 1e3) / 1e9 / peak, 4),
        "roofline": roofline_entry("score_tc_kernel<2d> (page-bound scan)", scan_bytes, scan_rot, scan_cold, peak,
                                   peak_kind, f"back-to-back launches cycling through {R} copies of the page "
                                   "bounds; cold: one launch after an L2 flush",
                                   traffic=read_traffic("asp_score_tc.cu", 1.0, "score_page_bounds_qwen3_8b_shaped_32k.txt")),
        "note": "same cache, query and L2 flush as the token-level step of this shape; the bounds are built once, "
                "untimed; the attention over the chosen pages is the same kernel as the token-level path's",
    }


def full_attention_record(wl, kvd, kv, q_dev, stream, flush, steps, peak):
    """Full attention over every cached token (the pages' other baseline), through
    the tail path of asp_sparse_attend."""
    import torch
    import query_predicted_token_b200 as asp
    B, Hq, Hkv, d = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    dev = kvd["k"].device
    lens = kvd["seq_lens"].cpu().tolist()
    out = torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=dev)
    zero = torch.zeros(B, dtype=torch.int32, device=dev)
    ws_d = torch.empty(max(16, asp.attend_workspace_bytes(B, Hq, Hkv, d, 0, wl.t_max)), dtype=torch.uint8,
                       device=dev)
    us = time_cold(lambda: asp.sparse_attend(q_dev, kv, None, None, 0, out, None, zero, wl.t_max, ws_d,
                                             stream=stream), stream, flush, steps)
    nbytes = dense_bytes(wl, lens)
    return {"step_us": round(us, 2), "gbs": round(nbytes / (us / 1e6) / 1e9, 1), "bytes": nbytes,
            "frac_of_peak": round(nbytes / (us / 1e6) / 1e9 / peak, 4),
            "note": "every cached token through the tail path of asp_sparse_attend; one launch after an L2 flush"}
# ----------------------------------------------------------------------------- selection recall
def recall_analysis(wl, kv, dev):
    """Selection quality on the synthetic queries (untimed).

    recall: share of the true next query's top-C set that a selection keeps -- the
    step's own selection (softmax-normalised coefficients, windows' predictions
    averaged), the same step with raw coefficients, the same step with the pooled-
    features reading of the averaging, and the current query reused one step late.
    by_reading: the same recall when the KV head's set is formed from its group
    under the other readings of the GQA aggregation (mean query, summed softmax
    mass, one set per query head), for the predicted and the current query.
    window_overlap: overlap of the top-C set of the last of 17 successive true
    queries with the 16 before it (mean over them, and with their union)."""
    import torch
    import query_predicted_token_b200 as asp
    import synth
    from query_predicted_token_b200.recall import reading_recall, recall_report, window_overlap
    qhist, q_next = synth.query_history(wl, steps=2)
    q_t = q_next[0].to(wl.torch_dtype()).to(dev)
    q_true = q_next[1].to(wl.torch_dtype()).to(dev)     # the model's next query, as attention sees it
    B, Hq, d, C = wl.batch, wl.n_q_heads, wl.head_dim, wl.C
    chosen, qpred = {}, None
    for name, coef, pool in (("predicted", "softmax", "predictions"),
                             ("predicted_raw_coefficients", "raw", "predictions"),
                             ("predicted_pooled_features", "softmax", "features")):
        st = asp.DecodeState(kv, Hq, asp.PredCfg(wl.W, wl.windows, wl.lam, coef, pool), C,
                             qhist.to(dev).contiguous())
        out = torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=dev)
        st.step(q_t, out)
        torch.cuda.synchronize()
        chosen[name] = tuple(t.clone() for t in st.selection)
        if name == "predicted":
            qpred = st.qpred.clone()
    res = recall_report(kv, C, q_true, {"current_query": q_t}, chosen)
    res = {k: round(v, 4) for k, v in res.items()}
    res["by_reading"] = {r: {k: round(v, 4) for k, v in m.items()}
                         for r, m in reading_recall(kv, C, q_true, {"predicted": qpred, "current_query": q_t}).items()}
    hist = [qhist[:, :, s].to(wl.torch_dtype()).to(dev) for s in range(qhist.shape[2])]
    res["window_overlap"] = {k: (round(v, 4) if isinstance(v, float) else v)
                             for k, v in window_overlap(kv, C, hist).items()}
    res["note"] = ("mean over (sequence, KV head) of |S & S_true| / |S_true|, S_true = top C with the true "
                   "next query; synthetic AR(1) queries (rho %.2f), so an analogue, not the pages' numbers" % wl.rho)
    return res


# ----------------------------------------------------------------------------- multi-layer stack
def multi_layer_period(wl, layers, tokens, dev, side_streams=1):
    """Steady-state decode period of a stack of `layers` layers, each with its own
    cache and query history: per token, layer l's attention runs on the main stream
    in layer order, and layer l's prediction, scan and selection run on side stream
    l mod `side_streams` (the cache side of the pages' two ranks; with two streams,
    one layer's latency-bound prediction and selection can overlap the next
    layer's scan).  The period is the time of `tokens` tokens over `tokens`, after
    2 warm-up tokens; a layer is only allocated while the device keeps 20% more
    memory free than it needs."""
    import torch
    import query_predicted_token_b200 as asp
    import synth
    B, Hq, Hkv, d, C = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.C
    e = 2 if wl.kv_dtype == "bf16" else 4
    per_layer = 2 * B * Hkv * wl.t_max * d * e
    main_s = torch.cuda.current_stream()
    side = [torch.cuda.Stream(priority=-100) for _ in range(max(1, side_streams))]
    states, outs, qs = [], [], []
    for l in range(layers):
        free, _ = torch.cuda.mem_get_info(dev)
        if free < 1.2 * per_layer + (2 << 30):
            break
        wl_l = wl.replace(seed=wl.seed + 1009 * (l + 1))
        kvd = synth.kv_cache(wl_l, dev)
        kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], kvd["page_table"], t_max=wl.t_max)
        qhist, q_next = synth.query_history(wl_l, steps=1)
        st = asp.DecodeState(kv, Hq, asp.PredCfg(wl.W, wl.windows, wl.lam), C, qhist.to(dev).contiguous(),
                             s_main=main_s, s_side=side[l % len(side)])
        lens = kvd["seq_lens"].cpu().tolist()
        idx0, cnt0 = synth.random_selection(B, Hkv, C, lens, seed=wl_l.seed + 99)
        st.set_selection(idx0.to(dev), cnt0.to(dev))
        st._kvd = kvd   # keep the cache alive with its state
        states.append(st)
        qs.append(q_next[0].to(wl.torch_dtype()).to(dev))
        outs.append(torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=dev))
    n = len(states)
    if n == 0:
        return {"layers": 0, "note": "not enough device memory for one layer"}

    def token():
        for l in range(n):
            states[l].step(qs[l], outs[l])

    for _ in range(2):
        token()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(main_s)
    for _ in range(tokens):
        token()
    for st in states[-len(side):]:   # the last selection of every side stream ends the window
        main_s.wait_event(st.ev_sel_done)
    b.record(main_s)
    torch.cuda.synchronize()
    period_us = a.elapsed_time(b) * 1e3 / tokens
    lens = synth.workloads.sequence_lengths(wl).tolist()
    step_b = step_bytes(wl, lens)["total"]
    res = {"layers": n, "requested_layers": layers, "side_streams": len(side), "tokens": tokens,
           "period_us": round(period_us, 1),
           "per_layer_us": round(period_us / n, 2), "gbs": round(step_b * n / (period_us / 1e6) / 1e9, 1),
           "note": "per token: attention of every layer on the main stream in layer order, prediction, scan and "
                   "selection of layer l on side stream l mod side_streams; no model weights or other layers' "
                   "compute"}
    del states
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- profiling launches
def profile_launches(args):
    """Builds the workload and launches one kernel --steps times, an L2 flush before
    each, for an ncu capture of that kernel alone (scan: the key scan as the library
    picks it; scan_cuda_cores: the CUDA-core scan on the same keys; attend: the
    sparse attention's stand-alone plan over a random selection; page_scan: the
    page-bound scan of the page-level path; decode: whole decode steps, for the
    selection or the predictor inside the step)."""
    import torch
    import query_predicted_token_b200 as asp
    import synth
    dev = torch.device("cuda", 0)
    wl = synth.workload(args.workload)
    B, Hq, Hkv, d, C = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.C
    kvd = synth.kv_cache(wl, dev)
    kv = asp.KV(kvd["k"], kvd["v"], kvd["seq_lens"], kvd["page_table"], t_max=wl.t_max)
    lens = kvd["seq_lens"].cpu().tolist()
    tail = 1 if kvd["page_table"] is not None else 0
    snap = [t - tail for t in lens]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    qpred = synth.query_history(wl, 1)[1][0].to(dev).contiguous()
    q = qpred.to(wl.torch_dtype())
    scores = torch.empty(B, Hkv, wl.t_max, device=dev)
    if args.profile == "decode":
        qhist, q_next = synth.query_history(wl, steps=1)
        st = asp.DecodeState(kv, Hq, asp.PredCfg(wl.W, wl.windows, wl.lam), C, qhist.to(dev).contiguous())
        i0, c0 = synth.random_selection(B, Hkv, C, lens, seed=wl.seed + 99)
        st.set_selection(i0.to(dev), c0.to(dev))
        qt = q_next[0].to(wl.torch_dtype()).to(dev)
        out = torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=dev)

        def fn():
            st.step(qt, out)
            st.s_main.wait_event(st.ev_sel_done)
    elif args.profile == "attend":
        idx, cnt = (x.to(dev) for x in synth.random_selection(B, Hkv, C, snap, seed=wl.seed + 99))
        tb = torch.tensor(snap, dtype=torch.int32, device=dev) if tail else None
        out = torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=dev)
        ws = torch.empty(max(16, asp.attend_workspace_bytes(B, Hq, Hkv, d, C, tail)), dtype=torch.uint8, device=dev)
        fn = lambda: asp.sparse_attend(q, kv, idx, cnt, C, out, None, tb, tail, ws)
    elif args.profile == "page_scan":
        meta = torch.empty(B, Hkv, math.ceil(wl.t_max / QUEST_PAGE), 2, d, dtype=wl.torch_dtype(), device=dev)
        asp.quest_build_meta(kv, QUEST_PAGE, meta)
        ps = torch.empty(B, Hkv, math.ceil(wl.t_max / QUEST_PAGE), device=dev)
        fn = lambda: asp.quest_page_scores(q, kv, meta, QUEST_PAGE, ps)
    elif args.profile == "scan_cuda_cores":
        fn = lambda: asp.score_keys_cuda_cores(qpred, kv, scores)
    else:
        fn = lambda: asp.score_keys(qpred, kv, scores)
    for _ in range(args.steps):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    assert asp.device_status() == 0
    print(f"profile {args.profile} {wl.name}: {args.steps} launches", flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
SUB_WORKLOADS = ("qwen3_32b_shaped_32k", "longcot_ragged_paged_b64")


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return profile_launches(args)
    import torch
    import query_predicted_token_b200 as asp
    import synth

    from query_predicted_token_b200.replicas import ReplicaGroup, rank_workload

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    group = ReplicaGroup("nccl", dev, timeout_s=120)
    world, rank = group.world, group.rank

    asp.lib()   # raises if the library is missing: there is no other path
    wl = rank_workload(synth.workload(args.workload), rank)   # each rank: its own batch
    B, Hq, Hkv, d, C = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.C
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peak, peak_kind = read_peaks()
    gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id
    with ClockSampler(gpu_id) as clocks:
        head, x = decode_record(wl, dev, args, flush, peak, peak_kind, headline=True, group=group)
        t_rank, t_e2e = group.slowest(sum(x["step_ms"]) / 1e3, sum(x["e2e_ms"]) / 1e3)
        ms_per_step = statistics.mean(x["step_ms"])
        io = (x["h2d"], x["d2h"])
        (total_bytes,) = group.total(x["acct"]["total"] * args.steps)   # ragged batches differ per rank
        group.barrier()
        extra = {}
        if world == 1 and not args.no_compare:
            # the pages' two baselines on the same cache and query
            extra["page_level"] = page_level_record(wl, x["kvd"], x["kv"], x["q_t"], x["s_main"], flush,
                                                    max(5, min(args.steps, 20)), peak, peak_kind)
            extra["full_attention"] = full_attention_record(wl, x["kvd"], x["kv"], x["q_t"], x["s_main"], flush,
                                                            max(5, min(args.steps, 20)), peak)
            extra["recall"] = recall_analysis(wl, x["kv"], dev)
        del x
        torch.cuda.empty_cache()
        subs = {}
        if world == 1 and not args.no_workloads:
            for name in SUB_WORKLOADS:
                rec, y = decode_record(synth.workload(name), dev, args, flush, peak, peak_kind, headline=False)
                del y
                torch.cuda.empty_cache()
                subs[name] = rec
        stack = None
        if world == 1 and args.layers > 1:
            stack = multi_layer_period(wl, args.layers, max(3, min(args.steps, 10)), dev, args.side_streams)
    group.barrier()
    value = total_bytes / t_rank / 1e9
    e2e_value = total_bytes / t_e2e / 1e9

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            gbs, sample, n, t = time_oracle(wl, args.cpu_seconds)
            cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle", "sample": sample}
        if "page_level" in extra:
            subs["quest_page_scan_8b_32k"] = extra["page_level"]
        if stack and "page_level" in extra and stack.get("layers"):
            # one layer's measured step times the layer count
            stack["page_level_period_us_from_one_layer"] = round(extra["page_level"]["step_us"] * stack["layers"], 1)
            stack["full_attention_period_us_from_one_layer"] = round(
                extra["full_attention"]["step_us"] * stack["layers"], 1)
        # the decode step's attention launches a merge when its plan splits the rows,
        # and the step launches the next step's lag factorisation when the selection's
        # CTAs (one per row) and the factorisation's (one per 4 query heads) fit on the
        # SMs together, for windows that are powers of two filling at most 32 lags
        dec_ws = int(asp.lib().asp_decode_workspace_bytes(B, Hq, Hkv, d, C, 0))
        splits = dec_ws > B * Hkv * 2048 * 4
        win = sorted(wl.windows)
        nv = 9 if max(win) + 1 <= 9 else (17 if max(win) + 1 <= 17 else 33)
        factor = (all(w & (w - 1) == 0 for w in win) and sum(win) <= 32 and max(win) == nv - 1 and
                  B * Hkv + -(-B * Hq // 4) <= torch.cuda.get_device_properties(0).multi_processor_count)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.kv_dtype == "bf16" else "f32", "data": "synthetic",
            "config": dict(head["config"], workload=wl.name,
                           l2="flushed before every step (512 MiB write outside the timed events); KV larger than L2",
                           parallelism=f"replicas x{world} (one decode batch per GPU, no collective)"),
            "step_us": head["step_us"], "step_us_p90": head["step_us_p90"], "kernel_us": head["kernel_us"],
            "step_bytes": head["step_bytes"], "ideal_step_us": head["ideal_step_us"],
            "roofline": head["roofline"], "roofline_attend": head["roofline_attend"],
            "step_frac_of_peak": round(value / world / peak, 4),
            "clocks": clocks.summary(),
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": io[0],
                    "d2h_bytes_per_step": io[1]},
            "gpu_launches": args.steps * (4 + (1 if splits else 0) + (1 if factor else 0)),
            "cpu_baseline": cpu,
            "workloads": subs or None,
            "comparison": {"full_attention": extra.get("full_attention"),
                           "page_level_step_us": extra["page_level"]["step_us"] if "page_level" in extra else None}
            if extra else None,
            "selection_recall": extra.get("recall"),
            "multi_layer": stack,
        }
        print(json.dumps(line), flush=True)
    group.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
