"""One process per GPU for the decode step: how ranks split the work and
agree on a time.

Every (request, head) page is independent and a step reads only its own
page, q, k, v and gates, so ranks need no exchange on the data path: each
rank owns its own batch of requests (weak scaling: the work per rank is
fixed as ranks are added) and runs the step on its own GPU.  Only the
measurement crosses ranks: a barrier before and after the timed region and
the maximum of the ranks' device times.

Works with any torch.distributed backend (NCCL on GPUs, gloo on CPU).
"""
import datetime
import os

import torch

from . import workloads as W

RANK_SEED_STRIDE = 7919   # seed offset between ranks' request batches


def rank_env():
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend, timeout_s=120, device_id=None):
    """Join the process group when world_size > 1; returns (world, rank, local)."""
    world, rank, local = rank_env()
    if world > 1 and not torch.distributed.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device_id is not None:
            kw["device_id"] = device_id
        torch.distributed.init_process_group(backend, **kw)
    return world, rank, local


def rank_workload(w: W.Workload, rank: int) -> W.Workload:
    """The batch of requests rank `rank` owns: same shape and format, its own seed."""
    return W.Workload(w.index, w.name, w.fmt, w.batch, w.heads, w.steps, w.gate_mu, w.gate_sigma,
                      w.seed + RANK_SEED_STRIDE * rank)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device="cpu"):
    """The largest of the ranks' values of x (every rank gets it)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank, world, steps, ms_max):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world * steps / (ms_max / 1000.0)


def finish(world):
    if world > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
