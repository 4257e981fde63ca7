"""Data-parallel replicas of the streamed step (one process per GPU).

Each rank streams its own copy of the frozen NF4 base from host memory and runs its own
batch; the only exchange is the mean of the LoRA gradients (one all-reduce of the flat fp32
gradient buffer per step) before the AdamW update, so every replica keeps identical LoRA
parameters.  torch.distributed carries the collective (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def average_gradients_(grads: torch.Tensor, group=None) -> torch.Tensor:
    """In-place mean of a flat gradient buffer over the ranks of `group`."""
    world = dist.get_world_size(group)
    if world > 1:
        dist.all_reduce(grads, op=dist.ReduceOp.SUM, group=group)
        grads.mul_(1.0 / world)
    return grads


def dp_step(step_no_update, grads: torch.Tensor, apply_update, group=None):
    """One data-parallel training step.

    step_no_update(): runs forward + backward on this rank's batch, leaves gradients in
    `grads` and returns the local loss; apply_update(): the optimizer step from `grads`.
    Returns (local loss, mean loss over ranks)."""
    loss = step_no_update()
    average_gradients_(grads, group)
    apply_update()
    t = torch.tensor([float(loss)], dtype=torch.float64, device=grads.device)
    if dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        t /= dist.get_world_size(group)
    return loss, float(t.item())


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Largest value of a per-rank measurement (timings are reported as the slowest rank)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
