"""Multi-process plumbing for running the layer on several GPUs of one node.

One process per GPU (torchrun).  Ranks hold contiguous token ranges of one
global batch and a full copy of the weights (data parallelism over tokens).
Positions, the capacity cut and the aux loss of the global batch need one
exchange per forward pass: every rank's per-expert token counts and sums of p
(the library's exchange record, 12 bytes per expert), all-gathered in rank
order (``exchange_records``; ncclAllGather over NVLink on GPUs).  The
measurement adds a barrier around the timed region and the maximum of the
per-rank device times.

Everything here is device agnostic (NCCL on GPUs, gloo on CPUs for the tests).
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class RankInfo:
    rank: int
    world_size: int
    local_rank: int

    @property
    def distributed(self) -> bool:
        return self.world_size > 1


def rank_info() -> RankInfo:
    """RANK / WORLD_SIZE / LOCAL_RANK from the environment (torchrun sets them)."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> RankInfo:
    """Join the process group when more than one rank is running."""
    info = rank_info()
    if info.distributed and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(info.local_rank)
            kw["device_id"] = torch.device("cuda", info.local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    elif backend == "nccl" and torch.cuda.is_available():
        torch.cuda.set_device(info.local_rank)
    return info


def barrier(info: RankInfo) -> None:
    if info.distributed:
        dist.barrier()


def max_over_ranks(info: RankInfo, value: float, device=None) -> float:
    """Largest value over all ranks (the slowest rank decides a timed region)."""
    if not info.distributed:
        return float(value)
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(info: RankInfo, units_per_rank: int, steps: int,
                         max_total_ms: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest time."""
    return info.world_size * units_per_rank * steps / (max_total_ms / 1e3)


def exchange_records(info: RankInfo, record: torch.Tensor) -> torch.Tensor:
    """All-gather of one equally sized 1-D record per rank: the records of all
    ranks, concatenated in rank order (a copy of ``record`` on a single rank)."""
    record = record.reshape(-1).contiguous()
    if not info.distributed:
        return record.clone()
    out = torch.empty(info.world_size * record.numel(), dtype=record.dtype,
                      device=record.device)
    dist.all_gather_into_tensor(out, record)
    return out


def alltoall_rows(info: RankInfo, rows: torch.Tensor, send_counts, recv_counts) -> torch.Tensor:
    """Row blocks between ranks: block g of ``rows`` (send_counts[g] rows) goes
    to rank g; the result holds recv_counts[g] rows from each rank g, in rank
    order (expert-parallel dispatch and return)."""
    if not info.distributed:
        return rows.clone()
    out = torch.empty((int(sum(recv_counts)),) + tuple(rows.shape[1:]), dtype=rows.dtype,
                      device=rows.device)
    dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=[int(c) for c in recv_counts],
                           input_split_sizes=[int(c) for c in send_counts])
    return out


def token_range(info: RankInfo, T_per_rank: int) -> tuple:
    """[start, stop) of this rank's tokens in a global batch of world * T_per_rank."""
    return info.rank * T_per_rank, (info.rank + 1) * T_per_rank


def rank_seed(info: RankInfo, base_seed: int = 0) -> int:
    """Seed of this rank's batch (independent batches; rank 0 keeps the base seed)."""
    return base_seed + info.rank


def finalize(info: RankInfo) -> None:
    if info.distributed and dist.is_initialized():
        dist.destroy_process_group()
