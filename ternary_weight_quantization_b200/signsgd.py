"""Data-parallel sign-gradient step with no master weights on the ranks.

"1BitTraining.md", "Why this always holds", closing paragraph: because the
straight-through gradient and the gradient of the quantised weight have the
same sign, a sign-based optimiser needs only the 2-bit weights on each device
and one bit of gradient per weight, streamed to one place that accumulates
them. Here that place is the holder rank, which alone keeps the master W.

One step, entered by every rank in the same order:
  1. every rank: the sign words of its dW (``bl_sign_pack`` on dW, or made
     by the backward itself with ``bl_backward_signs``; N*K/8 bytes)
  2. gather of the R ranks' words on the holder (torch.distributed; NCCL on
     GPUs, each rank sends N*K/8 bytes)
  3. holder: majority vote, the update of W and its new codes and gamma
     (``bl_signsgd_apply``: two launches, the vote, update and |W| sums in
     one sweep over W; or the three calls ``bl_sign_vote``,
     ``bl_signsgd_update``, ``bl_quantize_weight`` when ``SignOps.apply`` is
     None)
  4. broadcast of the new w_packed and gamma from the holder (N*K/4 + 4 bytes)

Only argument marshalling and the order of the collectives live here; every
step of the arithmetic runs in the library's kernels (``SignOps`` names them,
so that the host logic can be exercised on CPU ranks with other callables).
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable

import torch
import torch.distributed as dist

from . import bitlinear as b


@dataclass
class SignOps:
    """The device operations of a step: the library's calls by default."""
    sign_pack: Callable = field(default=b.bl_sign_pack)
    sign_vote: Callable = field(default=b.bl_sign_vote)
    update: Callable = field(default=b.bl_signsgd_update)
    quantize_weight: Callable = field(default=b.bl_quantize_weight)
    # the holder's vote + update + new codes in one call (None: the three
    # separate calls above)
    apply: Callable | None = field(default=b.bl_signsgd_apply)


@dataclass
class SignBuffers:
    """Scratch of one layer's step: this rank's words, and on the holder the
    gathered words of every rank and the vote's direction (used only by the
    three-call form of the holder's step)."""
    words: torch.Tensor
    gathered: torch.Tensor | None
    direction: torch.Tensor | None

    @staticmethod
    def allocate(N: int, K: int, world: int, is_holder: bool, device) -> "SignBuffers":
        words = torch.empty((N, K // 32), dtype=torch.int32, device=device)
        gathered = torch.empty((world, N, K // 32), dtype=torch.int32, device=device) if is_holder else None
        direction = torch.empty((N, K // 4), dtype=torch.uint8, device=device) if is_holder else None
        return SignBuffers(words, gathered, direction)


def _world():
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(), dist.get_rank()
    return 1, 0


def signsgd_dp_step(dW, w_packed, gamma, lr, *, master_W=None, workspace=None, holder: int = 0,
                    buffers: SignBuffers | None = None, ops: SignOps | None = None, words=None):
    """One sign-gradient step of one layer over the default process group.

    dW [N, K]: this rank's gradient (bf16 or f32) -- or dW None and words
    [N, K/32] int32: its sign words, already made (``bl_backward_signs``).
    w_packed [N, K/4] uint8 and gamma [1] f32: this rank's codes, replaced by
    the step's new ones. master_W [N, K] and workspace
    (``bl_quantize_weight``'s scratch): needed on the holder rank only.
    Returns (w_packed, gamma).
    """
    ops = ops or SignOps()
    world, rank = _world()
    if (dW is None) == (words is None):
        raise ValueError("pass exactly one of dW and words")
    N, K = w_packed.shape[0], w_packed.shape[1] * 4
    is_holder = rank == holder
    if is_holder and (master_W is None or workspace is None):
        raise ValueError("the holder rank needs master_W and workspace")
    buf = buffers or SignBuffers.allocate(N, K, world, is_holder, w_packed.device)

    if world > 1:
        if words is None:
            ops.sign_pack(dW, buf.words)
            words = buf.words
        dist.gather(words, list(buf.gathered.unbind(0)) if is_holder else None, dst=holder)
        votes = buf.gathered
    elif words is None:
        ops.sign_pack(dW, buf.gathered[0])  # a single rank votes on its own words
        votes = buf.gathered
    else:
        votes = words.unsqueeze(0)
    if is_holder:
        if ops.apply is not None:
            ops.apply(votes, master_W, lr, w_packed, gamma, workspace)
        else:
            ops.sign_vote(votes, buf.direction)
            ops.update(master_W, buf.direction, lr)
            ops.quantize_weight(master_W, w_packed, gamma, workspace)
    if world > 1:
        dist.broadcast(w_packed, src=holder)
        dist.broadcast(gamma, src=holder)
    return w_packed, gamma
