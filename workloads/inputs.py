"""Seeded synthetic BitLinear workloads (CPU torch tensors).

The pages measure on no public dataset; every input is drawn here from a
seeded ``torch.Generator`` on the CPU with the shapes and distributions of the
workloads named for the BitLinear layer ("bitnet-qat-train", Usage and
Measured behavior: 2560 -> 6912 at batch 8 x 512; "bitlinear.py",
``BitLinear.__init__``: kaiming-uniform(a = sqrt(5)) masters):

  tiny       M=32,   K=128,  N=256   W fp32 ~ N(0, 0.02^2), x, dY bf16 ~ N(0, 1)
  up_proj    M=4096, K=2560, N=6912  W bf16 kaiming-uniform, x, dY bf16 ~ N(0, 1)
  down_proj  M=2048, K=6912, N=2560  as up_proj, and x carries a seeded 1 %
                                     Bernoulli mask of entries scaled by 20

Seeds: x from seed ``base``, W from ``base + 100``, dY from ``base + 1``, the
outlier mask from ``base + 200``. Tensors are contiguous, row-major.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch

__all__ = ["Workload", "WORKLOADS", "STACKS", "make_inputs", "stack_inputs", "kaiming_uniform_bound"]


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    w_dtype: torch.dtype
    w_init: str          # "normal0.02" | "kaiming"
    outliers: bool = False


WORKLOADS = {
    "tiny": Workload("tiny", 32, 128, 256, torch.float32, "normal0.02"),
    "up_proj": Workload("up_proj", 4096, 2560, 6912, torch.bfloat16, "kaiming"),
    "down_proj": Workload("down_proj", 2048, 6912, 2560, torch.bfloat16, "kaiming", True),
}


# Layer stacks: 8 BitLinear layers alternating
# 2560 -> 6912 -> 2560 ... over x [4, 512, 2560].
STACKS = {
    "stack8": (2048, [2560, 6912] * 4 + [2560]),
}


def kaiming_uniform_bound(fan_in: int) -> float:
    """Bound of torch's kaiming_uniform_(a=sqrt(5)) for a [out, in] weight."""
    gain = math.sqrt(2.0 / (1.0 + 5.0))
    return math.sqrt(3.0) * gain / math.sqrt(fan_in)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def make_inputs(M: int, K: int, N: int, *, w_dtype=torch.bfloat16, w_init="kaiming",
                outliers=False, seed: int = 0):
    """Return (x [M,K] bf16, W [N,K] w_dtype, dY [M,N] bf16) on the CPU."""
    x = torch.randn(M, K, generator=_gen(seed), dtype=torch.float32)
    if outliers and x.numel():
        mask = torch.rand(M, K, generator=_gen(seed + 200)) < 0.01
        x = torch.where(mask, x * 20.0, x)
    if w_init == "normal0.02":
        w = torch.randn(N, K, generator=_gen(seed + 100), dtype=torch.float32) * 0.02
    elif w_init == "kaiming":
        b = kaiming_uniform_bound(K)
        w = (torch.rand(N, K, generator=_gen(seed + 100), dtype=torch.float32) * 2.0 - 1.0) * b
    elif w_init == "uniform1":
        w = torch.rand(N, K, generator=_gen(seed + 100), dtype=torch.float32) * 2.0 - 1.0
    else:
        raise ValueError(w_init)
    dy = torch.randn(M, N, generator=_gen(seed + 1), dtype=torch.float32)
    return (x.to(torch.bfloat16).contiguous(), w.to(w_dtype).contiguous(),
            dy.to(torch.bfloat16).contiguous())


def workload_inputs(name: str, seed: int = 0):
    wl = WORKLOADS[name]
    return make_inputs(wl.M, wl.K, wl.N, w_dtype=wl.w_dtype, w_init=wl.w_init,
                       outliers=wl.outliers, seed=seed)


__all__.append("workload_inputs")


def stack_inputs(M: int, dims, seed: int = 0):
    """(x [M, dims[0]] bf16, [W_l [dims[l+1], dims[l]] bf16 kaiming-uniform],
    dY [M, dims[-1]] bf16) on the CPU; W_l from seed + 100 + l."""
    x = torch.randn(M, dims[0], generator=_gen(seed), dtype=torch.float32)
    ws = []
    for l, (K, N) in enumerate(zip(dims[:-1], dims[1:])):
        b = kaiming_uniform_bound(K)
        w = (torch.rand(N, K, generator=_gen(seed + 100 + l), dtype=torch.float32) * 2.0 - 1.0) * b
        ws.append(w.to(torch.bfloat16).contiguous())
    dy = torch.randn(M, dims[-1], generator=_gen(seed + 1), dtype=torch.float32)
    return x.to(torch.bfloat16).contiguous(), ws, dy.to(torch.bfloat16).contiguous()


def gamma_midpoint_weights(case: str, w_dtype=torch.bfloat16, seed: int = 0):
    """W [2048, 1024] (2^21 elements) whose mean |W| lies on, just above or
    just below the midpoint 1 + 2^-24 between the fp32 neighbours 1 and
    1 + 2^-23. Every magnitude is a bf16 value; signs and positions are
    shuffled with ``seed``:

      2^20 ones and 2^19 twos (sum 2^21), then in the remaining 2^19 slots
      "tie":   one 2^-3                         sum = 2^21 + 2^-3
      "above": one 2^-3 and 2^18 of 2^-41       sum = 2^21 + 2^-3 + 2^-23
      "below": 2^-3 - 2^-11, 2^-11 - 2^-19 and 2^-19 - 2^-23
                                                sum = 2^21 + 2^-3 - 2^-23
      and zeros in the slots left.
    """
    n, k = 1 << 21, 1 << 19
    vals = torch.zeros(n, dtype=torch.float64)
    vals[: n - 2 * k] = 1.0
    vals[n - 2 * k: n - k] = 2.0
    rest = n - k
    if case in ("tie", "above"):
        vals[rest] = 2.0 ** -3
        if case == "above":
            vals[rest + 1: rest + 1 + (1 << 18)] = 2.0 ** -41
    elif case == "below":
        vals[rest] = 2.0 ** -3 - 2.0 ** -11
        vals[rest + 1] = 2.0 ** -11 - 2.0 ** -19
        vals[rest + 2] = 2.0 ** -19 - 2.0 ** -23
    else:
        raise ValueError(case)
    g = _gen(seed)
    perm = torch.randperm(n, generator=g)
    signs = torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0).to(torch.float64)
    w = (vals[perm] * signs).reshape(2048, 1024)
    return w.to(w_dtype).contiguous()


__all__.append("gamma_midpoint_weights")
