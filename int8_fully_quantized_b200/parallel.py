"""Data-parallel pieces of the INT8 linear layer (one process per GPU, torch.distributed).

Row-parallel work (quantize, LayerNorm_i8, GELU_i8, forward and input-gradient GEMMs) needs no
exchange: every rank owns its tokens and a full copy of the weight. The weight gradient is a
contraction over tokens, so each rank holds a partial dW. INT8 blocks with different scales do
not add, so the partial leaves the wgrad kernel in fp32, is summed across ranks (NCCL over
NVLink on GPUs, gloo on CPU), and is then re-quantized per 32x32 block. Step timing is the
maximum over ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world() -> tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(), dist.get_world_size()
    return 0, 1


def allreduce_wgrad_(dw_f32: torch.Tensor) -> torch.Tensor:
    """Sum the fp32 weight-gradient partials of all ranks in place (no-op on one rank)."""
    _, n = world()
    if n > 1:
        dist.all_reduce(dw_f32, op=dist.ReduceOp.SUM)
    return dw_f32


class WgradExchange:
    """Overlapped exchange of the fp32 weight-gradient partials of one data-parallel step.

    ``start(dw_f32)`` issues the all-reduce of a partial as soon as its wgrad kernel has been
    enqueued (asynchronously: NCCL runs it on its own stream, ordered after the wgrad, while the
    caller enqueues the rest of the backward on the compute stream). ``finish(requantize)`` waits
    for every started all-reduce, in the order they were started, and hands each summed partial to
    ``requantize`` (the per-block quantizer of the caller's choice, e.g. ``jf_quantize_block`` into
    the INT8 dW). On one rank there is nothing to sum: ``start`` only records the tensor.
    Every rank must start the same tensors in the same order (the collectives pair up by order)."""

    def __init__(self):
        self._pending = []

    def start(self, dw_f32: torch.Tensor, tag=None) -> None:
        _, n = world()
        handle = dist.all_reduce(dw_f32, op=dist.ReduceOp.SUM, async_op=True) if n > 1 else None
        self._pending.append((tag, dw_f32, handle))

    def finish(self, requantize) -> list:
        """Wait for the all-reduces and re-quantize each sum; returns requantize's results in order."""
        out = []
        for tag, dw, handle in self._pending:
            if handle is not None:
                handle.wait()
            out.append(requantize(tag, dw))
        self._pending = []
        return out


def max_over_ranks(value: float, device=None) -> float:
    """Largest value of a per-rank measurement (a step time) across ranks."""
    _, n = world()
    if n == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own tokens (weak scaling: the per-rank batch is fixed); the weight is
    drawn from the base seed on every rank so that all replicas agree."""
    return base_seed * 1000 + 1 + rank
