"""A stack of BitLinear layers trained through the library's calls.

The forward of every layer quantises its weight and its input
(``bl_quantize``) and runs the INT8 GEMM (``bl_forward``); between forward and
backward each layer keeps only its saved state -- the 2-bit codes, gamma, the
INT8 activations and their scales ("bitnet-qat-train", third intro bullet) --
so no bf16 copy of any layer's input or weight is kept. The backward walks the
layers in reverse (``bl_backward``): each layer's dX is the dY of the layer
below. Only argument marshalling happens here; every step runs in the
library's kernels.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import bitlinear as b


@dataclass
class _Layer:
    K: int
    N: int
    w_packed: torch.Tensor
    gamma: torch.Tensor
    workspace: torch.Tensor
    xq: torch.Tensor
    sx: torch.Tensor
    dW: torch.Tensor


@dataclass
class BitLinearStack:
    """Layers dims[0] -> dims[1] -> ... -> dims[-1] over M tokens."""
    M: int
    dims: list
    layers: list = field(default_factory=list)
    act: list = field(default_factory=list)   # two [M, max_dim] bf16 buffers (forward outputs)
    grad: list = field(default_factory=list)  # two [M, max_dim] bf16 buffers (backward dX)
    bwd_workspace: torch.Tensor | None = None  # x_hat scratch of the backward, shared by the layers

    @staticmethod
    def allocate(M, dims, dw_dtype=torch.bfloat16, device="cuda"):
        s = BitLinearStack(M=M, dims=list(dims))
        for K, N in zip(dims[:-1], dims[1:]):
            ws = b.bl_quantize_weight_workspace_size(N, K)
            s.layers.append(_Layer(
                K=K, N=N,
                w_packed=torch.empty((N, K // 4), dtype=torch.uint8, device=device),
                gamma=torch.empty(1, dtype=torch.float32, device=device),
                workspace=torch.empty(max(ws, 16), dtype=torch.uint8, device=device),
                xq=torch.empty((M, K), dtype=torch.int8, device=device),
                sx=torch.empty(M, dtype=torch.float32, device=device),
                dW=torch.empty((N, K), dtype=dw_dtype, device=device),
            ))
        big = M * max(dims)
        s.act = [torch.empty(big, dtype=torch.bfloat16, device=device) for _ in range(2)]
        s.grad = [torch.empty(big, dtype=torch.bfloat16, device=device) for _ in range(2)]
        need = max(b.bl_backward_workspace_size(M, N, K) for K, N in zip(dims[:-1], dims[1:]))
        s.bwd_workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
        return s

    def forward(self, x, weights, stream=None, on_layer=None):
        """x [M, dims[0]] bf16, weights[l] [dims[l+1], dims[l]]: returns the last
        layer's output (a view of an internal buffer). ``on_layer(l, y)``, if
        given, is called after layer l with its output (a view that the next
        layer but one overwrites)."""
        h = x
        for i, (L, W) in enumerate(zip(self.layers, weights)):
            y = self.act[i % 2][: self.M * L.N].view(self.M, L.N)
            b.bl_quantize(W, h, L.w_packed, L.gamma, L.xq, L.sx, L.workspace, stream)
            b.bl_forward(L.xq, L.sx, L.w_packed, L.gamma, y, None, stream)
            if on_layer is not None:
                on_layer(i, y)
            h = y
        return h

    def backward(self, dY, input_grad=True, stream=None, on_layer=None):
        """dY [M, dims[-1]] bf16: fills every layer's dW; returns dX of the first
        layer (a view of an internal buffer) or None when input_grad is False.
        ``on_layer(l, dy, dx)``, if given, is called after layer l with the
        output gradient it was given and its input gradient (views of internal
        buffers, or None for the first layer's dx when it is not wanted)."""
        g = dY
        for i in range(len(self.layers) - 1, -1, -1):
            L = self.layers[i]
            want_dx = input_grad or i > 0
            dX = self.grad[i % 2][: self.M * L.K].view(self.M, L.K) if want_dx else None
            b.bl_backward(g, L.xq, L.sx, L.w_packed, L.gamma, dX, L.dW, False, stream, workspace=self.bwd_workspace)
            if on_layer is not None:
                on_layer(i, g, dX)
            g = dX
        return g

    @staticmethod
    def check():
        """Synchronises the device and raises if a kernel recorded a device
        failure (a bounded pipeline wait that gave up) since the last reset."""
        status = b.bl_get_last_error()
        if status != 0:
            raise b.BitLinearError(status, "BitLinearStack", "device error word set")
