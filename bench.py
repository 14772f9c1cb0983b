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
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--layers", type=int, default=1,
                    help="also time a stack of this many layers (each with its own cache), steady-state period")
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


def read_traffic(kernel_file: str, launch_units: float):
    """Per-launch DRAM bytes of the score kernel from the committed ncu summary, if it
    was taken on the current source of that kernel (else None)."""
    import hashlib
    src = os.path.join(ROOT, "query_predicted_token_b200", "csrc", kernel_file)
    summ = os.path.join(ROOT, "profiles", "score_keys_qwen3_8b_shaped_32k.txt")
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


# ----------------------------------------------------------------------------- comparison paths
def comparison_paths(wl, kvd, kv, q_dev, stream, flush, steps):
    """Times, on the same cache and query, the page-level comparison path (page
    bound scan and page choice with the current query, then attention over the
    chosen pages' tokens) and full attention over every cached token.  The page
    bounds are built once beforehand (a serving system keeps them up to date as
    tokens arrive).  Returns a dict for the JSON line."""
    import torch
    import query_predicted_token_b200 as asp
    B, Hq, Hkv, d, C = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.C
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
    zero = torch.zeros(B, dtype=torch.int32, device=dev)
    ws_d = torch.empty(max(16, asp.attend_workspace_bytes(B, Hq, Hkv, d, 0, wl.t_max)), dtype=torch.uint8,
                       device=dev)
    with torch.cuda.stream(stream):
        asp.quest_build_meta(kv, QUEST_PAGE, meta, stream=stream)

    def quest_step():
        asp.quest_select(q_dev, kv, meta, QUEST_PAGE, C, ps, qidx, qcnt, stream=stream)
        asp.sparse_attend(q_dev, kv, qidx, qcnt, cp, out, workspace=ws_q, stream=stream)

    def dense_step():
        asp.sparse_attend(q_dev, kv, None, None, 0, out, None, zero, wl.t_max, ws_d, stream=stream)

    res = {}
    for name, fn, nbytes in (("page_level", quest_step, quest_step_bytes(wl, lens)["total"]),
                             ("full_attention", dense_step, dense_bytes(wl, lens))):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with torch.cuda.stream(stream):
            for k in range(-3, steps):
                flush.zero_()
                if k >= 0:
                    ev[k][0].record(stream)
                fn()
                if k >= 0:
                    ev[k][1].record(stream)
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
        res[name] = {"step_us": round(ms * 1e3, 2), "gbs": round(nbytes / (ms / 1e3) / 1e9, 1), "bytes": nbytes}
    res["note"] = ("same cache, query and L2 flush; page_level: page bounds scanned with the current query, "
                   f"{cp // QUEST_PAGE} pages of {QUEST_PAGE} kept, attention over their tokens; "
                   "full_attention: every cached token")
    return res


# ----------------------------------------------------------------------------- selection recall
def recall_analysis(wl, kv, dev):
    """Recall of the true next query's top-C set (untimed): the step's own
    selection (predicted query), the same step with raw ridge coefficients, and
    the current query reused one step late."""
    import torch
    import query_predicted_token_b200 as asp
    import synth
    from query_predicted_token_b200.recall import recall_report
    qhist, q_next = synth.query_history(wl, steps=2)
    q_t = q_next[0].to(wl.torch_dtype()).to(dev)
    q_true = q_next[1].to(wl.torch_dtype()).to(dev)     # the model's next query, as attention sees it
    B, Hq, d, C = wl.batch, wl.n_q_heads, wl.head_dim, wl.C
    chosen = {}
    for name, coef in (("predicted", "softmax"), ("predicted_raw_coefficients", "raw")):
        st = asp.DecodeState(kv, Hq, asp.PredCfg(wl.W, wl.windows, wl.lam, coef), C, qhist.to(dev).contiguous())
        out = torch.empty(B, Hq, d, dtype=wl.torch_dtype(), device=dev)
        st.step(q_t, out)
        torch.cuda.synchronize()
        chosen[name] = tuple(t.clone() for t in st.selection)
    res = recall_report(kv, C, q_true, {"current_query": q_t}, chosen)
    res = {k: round(v, 4) for k, v in res.items()}
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


# ----------------------------------------------------------------------------- GPU arm
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
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
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    s_main = st.s_main
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    acct = step_bytes(wl, lens)
    # the decode step's attention has a merge launch when its plan splits the rows:
    # its workspace then holds partials before the histogram
    dec_ws = int(asp.lib().asp_decode_workspace_bytes(B, Hq, Hkv, d, C, tail))
    splits = dec_ws > B * Hkv * 2048 * 4

    def one_step(k=None, e2e=False):
        with torch.cuda.stream(s_main):
            flush.zero_()                                   # L2 flush, outside the timed events
            if k is not None:
                ev[k][0].record(s_main)
            if e2e:
                q_t.copy_(q_host, non_blocking=True)
            st.step(q_t, out, lse)
            if e2e:   # the output is ready when the attention ends: read it back while the selection runs
                out_host.copy_(out, non_blocking=True)
            s_main.wait_event(st.ev_sel_done)
            if k is not None:
                ev[k][1].record(s_main)

    for _ in range(max(3, args.warmup)):
        one_step()
    torch.cuda.synchronize()
    group.barrier()
    gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id
    kern_ms = {n: [] for n in ("predict", "score", "select", "attend")}
    with ClockSampler(gpu_id) as clocks:
        # timed steps: no events between the kernels, so each kernel of the side
        # stream may launch while the previous one drains
        st.set_timing(False)
        torch.cuda.synchronize()
        for k in range(args.steps):
            one_step(k)
        torch.cuda.synchronize()
        step_ms = [a.elapsed_time(b) for a, b in ev]
        # the same steps again with events around every kernel, for the per-kernel
        # times and the scan's roofline
        st.set_timing(True)
        for k in range(args.steps):
            one_step()
            torch.cuda.synchronize()
            te = st.timing_events
            for i, n in enumerate(("predict", "score", "select", "attend")):
                kern_ms[n].append(te[2 * i].elapsed_time(te[2 * i + 1]))
        st.set_timing(False)
        torch.cuda.synchronize()
    assert asp.device_status() == 0
    # e2e: host query in, host output back, every step
    for k in range(args.steps):
        one_step(k, e2e=True)
    torch.cuda.synchronize()
    e2e_ms = [a.elapsed_time(b) for a, b in ev]
    # The key scan alone, for its roofline: the same kernel and grid through
    # asp_score_keys, launched back to back between two CUDA events on its stream
    # (the keys are larger than L2 and read with an evict-first hint, so each launch
    # streams them from HBM; one event pair per launch would add its ~6 µs floor).
    # The per-kernel events inside the step also hold the launch gap after the
    # predictor (events stop the programmatic dependent launch): `in_step_frac`.
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s_main):
        flush.zero_()
        for _ in range(2):
            asp.score_keys(st.qpred, kv, st.scores, stream=s_main)
        a0.record(s_main)
        for _ in range(args.steps):
            asp.score_keys(st.qpred, kv, st.scores, stream=s_main)
        a1.record(s_main)
    torch.cuda.synchronize()
    assert asp.device_status() == 0
    scan_alone_ms = a0.elapsed_time(a1) / args.steps
    # The sparse attention alone (its stand-alone plan, three CTAs per SM), the same
    # way, over the step's current selection: the second roofline row.
    sel_idx, sel_cnt = st.selection
    att_ws = torch.empty(max(16, int(asp.lib().asp_attend_workspace_bytes(B, Hq, Hkv, d, C, 0))),
                         dtype=torch.uint8, device=dev)
    with torch.cuda.stream(s_main):
        flush.zero_()
        for _ in range(2):
            asp.sparse_attend(q_t, kv, sel_idx, sel_cnt, C, out, workspace=att_ws, stream=s_main)
        a0.record(s_main)
        for _ in range(args.steps):
            asp.sparse_attend(q_t, kv, sel_idx, sel_cnt, C, out, workspace=att_ws, stream=s_main)
        a1.record(s_main)
    torch.cuda.synchronize()
    assert asp.device_status() == 0
    att_alone_ms = a0.elapsed_time(a1) / args.steps
    att_bytes = int(sel_cnt.sum().item()) * 2 * d * (2 if wl.kv_dtype == "bf16" else 4)
    # the pages' two baselines on the same cache and query: page-level selection, full attention
    compare = None if args.no_compare else comparison_paths(wl, kvd, kv, q_t, s_main, flush, args.steps)
    recall = None if args.no_compare else recall_analysis(wl, kv, dev)
    stack = (multi_layer_period(wl, args.layers, args.steps, dev, args.side_streams)
             if args.layers > 1 else None)
    if stack and compare and stack.get("layers"):
        for k in ("page_level", "full_attention"):   # one layer's measured step times the layer count
            stack[k + "_period_us_from_one_layer"] = round(compare[k]["step_us"] * stack["layers"], 1)

    t_rank, t_e2e = group.slowest(sum(step_ms) / 1e3, sum(e2e_ms) / 1e3)
    (total_bytes,) = group.total(acct["total"] * args.steps)   # ragged batches differ per rank
    group.barrier()
    value = total_bytes / t_rank / 1e9
    e2e_value = total_bytes / t_e2e / 1e9
    peak, peak_kind = read_peaks()
    score_ms = statistics.mean(kern_ms["score"])
    in_step = acct["score"] / (score_ms / 1e3) / 1e9
    achieved = acct["score"] / (scan_alone_ms / 1e3) / 1e9
    traffic = read_traffic("asp_score_tc.cu", 1.0) if wl.name == "qwen3_8b_shaped_32k" else None

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            gbs, sample, n, t = time_oracle(wl, args.cpu_seconds)
            cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle", "sample": sample}
        clk = clocks.summary()
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(statistics.mean(step_ms), 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.kv_dtype == "bf16" else "f32",
            "data": "synthetic",
            "config": {"workload": wl.name, "batch": B, "n_q_heads": Hq, "n_kv_heads": Hkv, "head_dim": d,
                       "T": wl.t_max, "ragged": wl.ragged, "paged": paged, "C": C, "W": wl.W,
                       "windows": list(wl.windows), "lambda": wl.lam,
                       "l2": "flushed before every step (512 MiB write outside the timed events); KV larger than L2",
                       "parallelism": f"replicas x{world} (one decode batch per GPU, no collective)"},
            "step_us": round(statistics.mean(step_ms) * 1e3, 2),
            "step_us_p90": round(sorted(step_ms)[int(0.9 * (len(step_ms) - 1))] * 1e3, 2),
            "kernel_us": {n: round(statistics.mean(v) * 1e3, 2) for n, v in kern_ms.items()},
            "step_bytes": acct["total"],
            "roofline": {"kernel": "score_tc_kernel (key scan)", "bound": "hbm", "achieved": round(achieved, 1),
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic, "algorithmic_bytes": acct["score"],
                         "timed": f"alone: {args.steps} back-to-back launches of the same kernel and grid "
                                  "through asp_score_keys between two CUDA events on its stream; keys larger "
                                  "than L2, read with an evict-first hint",
                         "us": round(scan_alone_ms * 1e3, 2),
                         "in_step_frac": round(in_step / peak, 4)},
            "roofline_attend": {"kernel": "attend_mma_kernel (sparse attention, stand-alone plan)", "bound": "hbm",
                                "achieved": round(att_bytes / (att_alone_ms / 1e3) / 1e9, 1), "peak": peak,
                                "peak_kind": peak_kind, "unit": "GB/s",
                                "frac": round(att_bytes / (att_alone_ms / 1e3) / 1e9 / peak, 4),
                                "algorithmic_bytes": att_bytes, "us": round(att_alone_ms * 1e3, 2),
                                "timed": f"alone: {args.steps} back-to-back asp_sparse_attend launches over the "
                                         "step's selection between two CUDA events"},
            "step_frac_of_peak": round(value / world / peak, 4),
            "clocks": clk,
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": q_host.numel() * q_host.element_size(),
                    "d2h_bytes_per_step": out.numel() * out.element_size()},
            "gpu_launches": args.steps * (4 + (1 if splits else 0)),
            "cpu_baseline": cpu,
            "comparison": compare,
            "selection_recall": recall,
            "multi_layer": stack,
        }
        print(json.dumps(line), flush=True)
    group.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
