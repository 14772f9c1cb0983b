"""One decode replica per GPU: data parallelism over independent batches.

A decode step reads only its own batch's KV cache, query history and
selection, so N GPUs serve N disjoint batches of sequences with nothing
exchanged on the data path (weak scaling: per-GPU work is fixed as N grows).
The only collectives are measurement plumbing on the host side:

* a barrier before and after the timed steps, so every rank starts together;
* the maximum over ranks of the measured seconds (the job is as fast as its
  slowest replica);
* the sum over ranks of the bytes each replica moved (ragged batches differ).

Every rank calls these in the same order.  The process group gets a short
timeout, so that a rank that died or never joined ends the others' next
collective with an error instead of a wait without end.

One process per GPU, launched by ``torch.distributed.run`` (``RANK``,
``LOCAL_RANK``, ``WORLD_SIZE``, ``MASTER_ADDR``/``MASTER_PORT`` from the
environment); ``backend`` is ``"nccl"`` on GPUs and ``"gloo"`` for the CPU
tests of this logic.
"""
from __future__ import annotations

import datetime
import os
from typing import Sequence

import torch

# distinct, reproducible inputs per rank; rank 0 keeps the single-GPU draw
_RANK_SEED_STRIDE = 1_000_003


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s batch given the workload's ``seed``."""
    if rank < 0:
        raise ValueError(f"rank {rank} < 0")
    return int(seed) + _RANK_SEED_STRIDE * int(rank)


def rank_workload(wl, rank: int):
    """The workload rank ``rank`` decodes: same shapes, its own seeded batch."""
    return wl.replace(seed=rank_seed(wl.seed, rank))


class ReplicaGroup:
    """Rank bookkeeping and the host-side collectives of a replicated run.

    With ``WORLD_SIZE`` 1 (or unset) no process group is created and every
    collective is the identity.
    """

    def __init__(self, backend: str, device: torch.device, timeout_s: float = 120.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        if not 0 <= self.rank < self.world:
            raise ValueError(f"RANK {self.rank} outside [0, {self.world})")
        self.device = torch.device(device)
        self._dist = None
        if self.world > 1:
            import torch.distributed as dist
            kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
            if backend == "nccl":
                kw["device_id"] = self.device
            dist.init_process_group(backend, **kw)
            self._dist = dist

    @property
    def distributed(self) -> bool:
        return self._dist is not None

    def barrier(self) -> None:
        if self._dist is not None:
            self._dist.barrier()

    def _all_reduce(self, values: Sequence[float], dtype, op) -> list:
        if self._dist is None:
            return list(values)
        t = torch.tensor(list(values), dtype=dtype, device=self.device)
        self._dist.all_reduce(t, op=op)
        return t.tolist()

    def slowest(self, *seconds: float) -> list:
        """Element-wise maximum over ranks of the given times."""
        op = self._dist.ReduceOp.MAX if self._dist is not None else None
        return self._all_reduce(seconds, torch.float64, op)

    def total(self, *counts: int) -> list:
        """Element-wise sum over ranks of the given integer counts."""
        op = self._dist.ReduceOp.SUM if self._dist is not None else None
        return [int(x) for x in self._all_reduce(counts, torch.int64, op)]

    def close(self) -> None:
        if self._dist is not None:
            self._dist.barrier()
            self._dist.destroy_process_group()
            self._dist = None
