"""Host logic of the replicated (one batch per GPU) run, on CPU with gloo ranks.

The decode step has no data-path collective; what N > 1 adds is the rank's own
seeded batch, a barrier around the timed steps, the maximum over ranks of the
measured time and the sum over ranks of the bytes moved.  These tests run that
sequence as two spawned ``gloo`` processes on 127.0.0.1, and check that a rank
that fails before a collective ends the other rank's collective with an error
(a short process-group timeout) instead of leaving it waiting.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import socket
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402
from query_predicted_token_b200.replicas import ReplicaGroup, rank_seed, rank_workload  # noqa: E402

RAGGED = "longcot_ragged_paged_b64"


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_env(rank: int, world: int, port: int) -> None:
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))


def _rank_main(rank: int, world: int, port: int, q) -> None:
    """The collective sequence of the replicated bench, with fake per-rank times."""
    _rank_env(rank, world, port)
    try:
        g = ReplicaGroup("gloo", "cpu", timeout_s=60)
        wl = rank_workload(synth.workload(RAGGED), g.rank)
        lens = synth.workloads.sequence_lengths(wl).tolist()
        moved = bench.step_bytes(wl, lens)["total"] * 3          # 3 steps
        g.barrier()                                              # before the timed steps
        t_step, t_e2e = 1.0 + 0.5 * g.rank, 4.0 - g.rank          # each rank's own clock
        slow = g.slowest(t_step, t_e2e)
        total = g.total(moved)
        g.barrier()
        g.close()
        q.put((rank, "ok", slow, total, moved, lens))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, "error", repr(e), None, None, None))


def _send_and_exit(q, item, code: int) -> None:
    """Puts ``item`` and ends the process at once; the queue's feeder thread is
    joined first, or ``os._exit`` can end the process before the message is out."""
    q.put(item)
    q.close()
    q.join_thread()
    os._exit(code)


def _rank_dies(rank: int, world: int, port: int, q) -> None:
    """Rank 1 exits abruptly after joining (no teardown, so its sockets close at
    once); rank 0 then enters a collective."""
    _rank_env(rank, world, port)
    try:   # a loaded host can take seconds to connect: report a failure instead of going silent
        g = ReplicaGroup("gloo", "cpu", timeout_s=30)
        g.barrier()   # both ranks fully connected before one of them leaves
    except Exception as e:
        _send_and_exit(q, (rank, "setup failed", repr(e)), 1)
    if rank == 1:
        _send_and_exit(q, (rank, "raised", None), 3)
    t0 = time.monotonic()   # start-up time (spawn, imports) is not what is tested: time the collective
    try:
        g.slowest(1.0)
        item = (rank, "no error", time.monotonic() - t0)
    except Exception as e:
        item = (rank, "error", type(e).__name__, time.monotonic() - t0)
    _send_and_exit(q, item, 0)   # the group is broken: skip its teardown


def _run(target, world: int = 2, join_s: float = 120.0):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(world):
            item = q.get(timeout=join_s)
            results[item[0]] = item
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():      # only the processes this test started
                p.kill()
                p.join()
    return results


def test_rank_seeds():
    wl = synth.workload(RAGGED)
    assert rank_workload(wl, 0) == wl                 # rank 0 decodes the single-GPU batch
    seeds = {rank_seed(wl.seed, r) for r in range(8)}
    assert len(seeds) == 8
    w1 = rank_workload(wl, 1)
    assert (w1.batch, w1.n_q_heads, w1.n_kv_heads, w1.head_dim, w1.t_max, w1.C) == \
        (wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.t_max, wl.C)
    with pytest.raises(ValueError):
        rank_seed(wl.seed, -1)


def test_single_rank_is_identity(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    g = ReplicaGroup("gloo", "cpu")
    assert (g.world, g.rank, g.distributed) == (1, 0, False)
    g.barrier()
    assert g.slowest(1.5, 2.5) == [1.5, 2.5]
    assert g.total(7, 9) == [7, 9]
    g.close()


def test_bad_rank_rejected(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "2")
    with pytest.raises(ValueError):
        ReplicaGroup("gloo", "cpu")


def test_two_gloo_ranks_aggregate():
    res = _run(_rank_main)
    assert sorted(res) == [0, 1]
    for r in (0, 1):
        assert res[r][1] == "ok", res[r][2]
    # max over ranks of each time, identical on every rank
    assert res[0][2] == res[1][2] == [1.5, 4.0]
    # bytes: the sum of what each rank moved, identical on every rank
    assert res[0][3] == res[1][3] == [res[0][4] + res[1][4]]
    # the ranks decode different batches (ragged lengths drawn from their own seeds)
    assert res[0][5] != res[1][5]
    assert res[0][5] == synth.workloads.sequence_lengths(synth.workload(RAGGED)).tolist()


def test_dead_rank_ends_collective_with_error():
    # the survivor's collective fails when the dead rank's sockets close, well inside
    # the group's 30 s timeout
    res = _run(_rank_dies, join_s=120.0)
    assert res[1][1] == "raised"
    assert res[0][1] == "error", res[0]
    assert res[0][3] < 60.0, res[0]   # within the 30 s process-group timeout, with margin
