"""Data-parallel BitLinear training step over token shards.

The path shards by tokens: every rank holds the same master W and its own
tokens x_r [M_r, K] with their output gradients dY_r [M_r, N]. S1 runs on
every rank on the replicated W (deterministic, so every rank holds the same
codes and gamma and nothing is exchanged for them); S2, the forward and dX
only touch the rank's own tokens. dW is a sum over tokens, so each rank's
``bl_backward`` yields a partial sum over its shard and the one exchange step
of the path is the sum of the partials over the ranks: an all-reduce of dW
(N*K elements; NCCL over NVLink on GPUs). After it every rank holds
dW = dY^T x_hat over all ranks' tokens, ready for a replicated optimiser.

One step, entered by every rank in the same order:
  1. ``bl_quantize``  (S1 + S2 on this rank's tokens)
  2. ``bl_forward``   (S3)
  3. ``bl_backward``  (S4: dX of this rank's tokens, its partial dW)
  4. all-reduce (sum) of dW over the process group

Only argument marshalling and the collective live here; the arithmetic runs
in the library's kernels (``DPOps`` names them, so that the host logic can be
exercised on CPU ranks with other callables).
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable

import torch
import torch.distributed as dist

from . import bitlinear as b

__all__ = ["DPOps", "dp_step"]


@dataclass
class DPOps:
    """The device operations of a step: the library's calls by default."""
    quantize: Callable = field(default=b.bl_quantize)
    forward: Callable = field(default=b.bl_forward)
    backward: Callable = field(default=b.bl_backward)


def dp_step(x, W, dY, bufs: b.StepBuffers, *, group=None, stream=None, ops: DPOps | None = None):
    """One data-parallel forward + backward of one BitLinear layer.

    x [M_r, K] bf16 and dY [M_r, N] bf16: this rank's tokens. W [N, K]: the
    replicated master. ``bufs`` holds this rank's outputs (y, dX of its
    tokens) and, after the call, the dW summed over every rank of ``group``
    (the default process group when one is initialised; a single process
    sums nothing). Returns bufs.
    """
    ops = ops or DPOps()
    ops.quantize(W, x, bufs.w_packed, bufs.gamma, bufs.xq, bufs.sx, bufs.workspace, stream)
    ops.forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, None, stream)
    ws = {} if bufs.bwd_workspace is None else {"workspace": bufs.bwd_workspace}  # x_hat scratch
    ops.backward(dY, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.dX, bufs.dW, False, stream, **ws)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        if stream is not None and bufs.dW.is_cuda:
            with torch.cuda.stream(stream):
                dist.all_reduce(bufs.dW, op=dist.ReduceOp.SUM, group=group)
        else:
            dist.all_reduce(bufs.dW, op=dist.ReduceOp.SUM, group=group)
    return bufs
