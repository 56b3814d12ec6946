"""Data-parallel training step of the backward (HSA summary page, Implementation;
abstract page: the model is trained).

With independent sequences per rank, dQ, dK and dV of a rank's sequences
depend on that rank's data alone.  W_L is shared by every sequence, so its
gradient is the sum over all ranks' sequences: the one exchange of a
data-parallel backward is an all-reduce (sum) of dW_L, d x d fp32
(64 KiB at d = 128).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import backward

__all__ = ["allreduce_param_grads", "backward_dp"]


def allreduce_param_grads(dW: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the W_L gradient over the process group in place (no-op on one rank)."""
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=group)
    return dW


def backward_dp(Q, K, V, W_L, L, idx, score, keff, dO, S, k, tau=0.0, q_pos0=0, group=None, **kw):
    """hsa.backward on this rank's sequences, then the all-reduce of dW_L.
    Returns (dQ, dK, dV, dW_L) with dW_L summed over the group."""
    dQ, dK, dV, dW = backward(Q, K, V, W_L, L, idx, score, keff, dO, S, k, tau, q_pos0, **kw)
    allreduce_param_grads(dW, group)
    return dQ, dK, dV, dW
