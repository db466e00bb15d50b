"""Multi-process plumbing over torch.distributed (one process per GPU).

The hot path shards without data exchange: activation tensors, layers and expert
matrices are independent problems, so ranks run replicas of the same step.  Two
small reductions appear only when one calibration is split over token shards
(data parallel over the calibration set):

  * the per-tensor amax is a maximum over all tokens: all-reduce MAX of one float
    ([CAL] section 2 step 1, max calibration);
  * the local Hessian H_b = sum_t x_t,b^T x_t,b is a sum over tokens: all-reduce SUM
    of the [cols/16, 16, 16] FP32 blocks ([CAL] section 2 step 2), 1 KB per block.

Timing across ranks is the maximum of the per-rank device times.  NCCL serves CUDA
tensors, gloo CPU tensors (used by the CPU tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as tdist


def env() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str | None = None, timeout_s: float = 300.0) -> tuple[int, int, int]:
    """Joins the process group when launched with more than one rank.  The timeout
    bounds every collective, so ranks waiting on a lost peer end with an error."""
    ws, rank, local = env()
    if ws > 1 and not tdist.is_initialized():
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return ws, rank, local


def active() -> bool:
    return tdist.is_available() and tdist.is_initialized() and tdist.get_world_size() > 1


def barrier():
    if active():
        tdist.barrier()


def finalize():
    if active():
        tdist.barrier()
        tdist.destroy_process_group()


def _device() -> torch.device:
    if active() and tdist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def max_over_ranks(values: list[float]) -> list[float]:
    """Element-wise maximum of per-rank numbers (e.g. device times), on every rank."""
    if not active():
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=_device())
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def shard_rows(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous token shard [r0, r1) of rank among world ranks (sizes differ by <= 1)."""
    base, extra = divmod(n, world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


def allreduce_amax_(d_amax: torch.Tensor) -> torch.Tensor:
    """In place: the per-tensor amax over all ranks' token shards (MAX)."""
    if active():
        tdist.all_reduce(d_amax, op=tdist.ReduceOp.MAX)
    return d_amax


def allreduce_hessian_(H: torch.Tensor) -> torch.Tensor:
    """In place: the local Hessians summed over all ranks' token shards (SUM)."""
    if active():
        tdist.all_reduce(H, op=tdist.ReduceOp.SUM)
    return H
