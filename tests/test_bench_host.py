"""Host-side pieces of bench.py (CPU only): the DRAM traffic of the dominant
kernel is taken from the committed ncu summary only while that summary was
captured on the kernel's current source, and the step's algorithmic bytes add
up from the per-kernel accounting."""
from __future__ import annotations

import hashlib
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402

SCRATCH = os.path.join(ROOT, "_build", "test_bench_host")


def _fake_root(src_text: str, summary_hash: str, dram_bytes: int) -> str:
    """A directory laid out like the repository with one kernel source and one summary."""
    shutil.rmtree(SCRATCH, ignore_errors=True)
    os.makedirs(os.path.join(SCRATCH, "query_predicted_token_b200", "csrc"))
    os.makedirs(os.path.join(SCRATCH, "profiles"))
    with open(os.path.join(SCRATCH, "query_predicted_token_b200", "csrc", "kern.cu"), "w") as f:
        f.write(src_text)
    with open(os.path.join(SCRATCH, "profiles", "score_keys_qwen3_8b_shaped_32k.txt"), "w") as f:
        f.write("# a summary\n")
        f.write(f"source_sha256_16: {summary_hash}\n")
        f.write(f"dram_bytes_per_launch: {dram_bytes}\n")
    return SCRATCH


def test_traffic_is_reported_only_for_the_source_it_was_captured_on(monkeypatch):
    src = "// kernel v1\n"
    h = hashlib.sha256(src.encode()).hexdigest()[:16]
    monkeypatch.setattr(bench, "ROOT", _fake_root(src, h, 1000))
    assert bench.read_traffic("kern.cu", 2.5) == 2500.0
    # the kernel changed after the capture: no traffic figure
    monkeypatch.setattr(bench, "ROOT", _fake_root("// kernel v2\n", h, 1000))
    assert bench.read_traffic("kern.cu", 1.0) is None
    # no summary or no source: no traffic figure, no exception
    assert bench.read_traffic("missing.cu", 1.0) is None
    shutil.rmtree(SCRATCH, ignore_errors=True)


def test_step_bytes_add_up():
    for name in ("tiny_f32_t512", "qwen3_8b_shaped_32k", "longcot_ragged_paged_b64"):
        wl = synth.workload(name)
        lens = synth.workloads.sequence_lengths(wl).tolist()
        acct = bench.step_bytes(wl, lens)
        parts = sum(v for k, v in acct.items() if k != "total")
        assert acct["total"] == parts, name
        # the key scan reads every cached key once: d * e bytes per token and KV head
        e = 2 if wl.kv_dtype == "bf16" else 4
        assert acct["score"] >= sum(lens) * wl.n_kv_heads * wl.head_dim * e, name
