"""Process-group plumbing for multi-GPU runs: one process per GPU.

The path shards without any exchange (every (sequence, KV head, tile) is
independent), so a run on N GPUs is N independent replicas, each rank
owning its own batch of sequences.  The only collectives are host-side
bookkeeping outside the data path: a barrier around the timed region and a
max / sum of scalars across ranks.
"""

from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as torch_dist


class Ranks:
    def __init__(self, backend: str | None = None, timeout_s: float = 120.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        if self.world > 1:
            if backend is None:
                backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local_rank)
            torch_dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.pg = True
            self.backend = backend
        else:
            self.backend = None

    def _tensor(self, value: float) -> torch.Tensor:
        dev = torch.device("cuda", self.local_rank) if self.backend == "nccl" else torch.device("cpu")
        return torch.tensor([float(value)], dtype=torch.float64, device=dev)

    def barrier(self) -> None:
        if self.pg:
            if self.backend == "nccl":
                torch_dist.barrier(device_ids=[self.local_rank])
            else:
                torch_dist.barrier()

    def max(self, value: float) -> float:
        if not self.pg:
            return float(value)
        t = self._tensor(value)
        torch_dist.all_reduce(t, op=torch_dist.ReduceOp.MAX)
        return float(t.item())

    def sum(self, value: float) -> float:
        if not self.pg:
            return float(value)
        t = self._tensor(value)
        torch_dist.all_reduce(t, op=torch_dist.ReduceOp.SUM)
        return float(t.item())

    def close(self) -> None:
        if self.pg:
            torch_dist.destroy_process_group()
            self.pg = False


def replica_seed_offset(rank: int) -> int:
    """Seed offset of a rank's replica batch (rank 0 keeps the workload's own seeds)."""
    return 7919 * rank
