"""Data parallelism for the int8-LoRA layer step: one process per GPU.

Each rank holds a replica of the frozen int8 kernels and of the LoRA factors
and processes its own rows (tokens); forward and dX are independent per
rank.  The only exchange is the sum of the LoRA gradients dA and dB (and
dbias) over ranks, one all-reduce of a flat fp32 buffer per step: with LoRA
only the adapter weights are trained ("Parameter-efficient fine-tuning of
GPT-2 with LoRA", "Why does LoRA reduce memory footprint?": gradients exist
only for the trainable parameters), so that buffer is small (4 r (K + N)
bytes per layer).
"""
from __future__ import annotations

import os
from datetime import timedelta
from typing import Tuple

import torch
import torch.distributed as dist


def env_rank() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str = "nccl", timeout_s: float = 120.0):
    """Initialises the default process group when WORLD_SIZE > 1."""
    rank, local, world = env_rank()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29500")
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=timeout_s),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s))
    return rank, local, world


def shard_rows(M_total: int, rank: int, world: int) -> Tuple[int, int]:
    """[begin, end) rows of rank `rank` when M_total rows are split evenly
    (the first M_total % world ranks take one extra row)."""
    base, extra = divmod(M_total, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def rank_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s private batch in weak-scaling runs."""
    return base + 1000 * rank


def allreduce_grads(flat: torch.Tensor, group=None) -> torch.Tensor:
    """Sums the flat LoRA-gradient buffer over ranks, in place."""
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over all ranks (timings)."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()
