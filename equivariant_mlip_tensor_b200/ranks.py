"""Data-parallel plumbing: one process per GPU, each with its own batch.

The convolution of independent graphs shards by batch with no exchange on
the data path: every rank builds, stores and differentiates its own
molecules.  The only collectives are the host-side ones that time a run:
a barrier around the timed region, the slowest rank's time (max) and the
total number of edges processed (sum).  The same code runs over NCCL on
GPUs and over gloo on CPU tensors (the multi-process tests).
"""
import os
from dataclasses import dataclass
from datetime import timedelta


@dataclass(frozen=True)
class Ranks:
    world: int
    rank: int
    local: int

    @staticmethod
    def from_env():
        """RANK / LOCAL_RANK / WORLD_SIZE as set by torch.distributed.run (defaults: one process)."""
        return Ranks(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                     int(os.environ.get("LOCAL_RANK", "0")))


def shard_seed(base, rank):
    """Seed of a rank's batch: every rank draws different molecules."""
    return base + 1000 * rank


class Group:
    """The process group of a run and its timing collectives.

    backend "nccl" with a CUDA device for the benchmark, "gloo" with the CPU
    for tests.  With one process nothing is initialised and every collective
    is the identity.  Every rank must call the same collectives in the same
    order.
    """

    def __init__(self, ranks, backend, device, timeout_s=120):
        import torch.distributed as dist
        self.ranks, self.device, self._dist = ranks, device, dist
        self.active = ranks.world > 1
        if self.active and not dist.is_initialized():
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, rank=ranks.rank, world_size=ranks.world,
                                    timeout=timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.active:
            self._dist.barrier()

    def _reduce(self, v, op):
        if not self.active:
            return float(v)
        import torch
        t = torch.tensor([float(v)], dtype=torch.float64, device=self.device)
        self._dist.all_reduce(t, op=op)
        return float(t.item())

    def max(self, v):
        """The largest value over ranks (the slowest rank's time)."""
        return self._reduce(v, self._dist.ReduceOp.MAX)

    def sum(self, v):
        """The sum over ranks (work done by the whole job)."""
        return self._reduce(v, self._dist.ReduceOp.SUM)

    def close(self):
        if self.active and self._dist.is_initialized():
            self._dist.destroy_process_group()


def throughput(group, local_units, local_seconds, steps):
    """(units per second of the whole job, ms per step): all ranks' units over
    the slowest rank's time, as weak scaling reports it."""
    t = group.max(local_seconds)
    units = group.sum(local_units)
    return units * steps / t, 1e3 * t / steps
