"""A small decoder LM whose projections are BitLinear layers run by the library.

"bitnet-qat-train" (Measured behavior, Training) trains a 4-layer transformer
LM with the layer. Here the attention q, k, v, o and the SwiGLU gate, up,
down projections of every block go through the C ABI: the forward quantises
the fp32 master and the bf16 activations (``bl_quantize``) and runs the INT8
GEMM (``bl_forward``), keeping only the 2-bit codes, gamma, the INT8
activations and their scales; the backward rebuilds the operands from that
state (``bl_backward``: dX in bf16, dW in fp32). The pages give no other part
of the model; embedding, RMSNorm, attention, the SwiGLU gating, the LM head,
the cross-entropy and AdamW are plain PyTorch on the GPU (fp32), outside the
library:

  pre-norm blocks  h += o(attn(norm(h))); h += down(silu(gate(m)) * up(m)),
                   m = norm(h); RMSNorm x / sqrt(mean(x^2) + eps) * g
  attention        causal softmax, `heads` heads, no positional encoding
  loss             mean next-token cross-entropy
  AdamW            decoupled decay on the 2-D weights, not on the norm gains
"""

from __future__ import annotations

import math

import torch

from . import bitlinear as b

__all__ = ["BitLinearFunction", "lm_loss", "adamw_step", "train_lm"]


class BitLinearFunction(torch.autograd.Function):
    """y [M, N] fp32 = BitLinear(x [M, K] fp32, W [N, K] fp32 master)."""

    @staticmethod
    def forward(ctx, x2d, w):
        M, K = x2d.shape
        N = w.shape[0]
        dev = x2d.device
        xb = x2d.to(torch.bfloat16).contiguous()
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
        gamma = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(max(b.bl_quantize_weight_workspace_size(N, K), 16), dtype=torch.uint8, device=dev)
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sx = torch.empty(M, dtype=torch.float32, device=dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        b.bl_quantize(w.contiguous(), xb, packed, gamma, xq, sx, ws)
        b.bl_forward(xq, sx, packed, gamma, y)
        ctx.save_for_backward(xq, sx, packed, gamma)
        return y.float()

    @staticmethod
    def backward(ctx, gy):
        xq, sx, packed, gamma = ctx.saved_tensors
        M, K = xq.shape
        N = packed.shape[0]
        dy = gy.to(torch.bfloat16).contiguous()
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dy.device)
        dW = torch.empty((N, K), dtype=torch.float32, device=dy.device)
        b.bl_backward(dy, xq, sx, packed, gamma, dX, dW)
        return dX.float(), dW


def _rmsnorm(x, g, eps):
    return x / torch.sqrt(torch.mean(x * x, dim=-1, keepdim=True) + eps) * g


def lm_loss(params: dict, ids: torch.Tensor, cfg) -> torch.Tensor:
    """Mean next-token cross-entropy of ids [B, S + 1] (fp32 parameters)."""
    B, S1 = ids.shape
    S, d, H = S1 - 1, cfg.d, cfg.heads
    dh = d // H
    x_ids, y_ids = ids[:, :S], ids[:, 1:]
    h = params["embed"][x_ids]
    causal = torch.ones(S, S, dtype=torch.bool, device=ids.device).tril()
    bl = BitLinearFunction.apply
    for i in range(cfg.layers):
        def p(n):
            return params[f"layer{i}.{n}"]
        a = _rmsnorm(h, p("attn_norm"), cfg.norm_eps).reshape(B * S, d)
        q, k, v = (bl(a, p(n)).reshape(B, S, H, dh).transpose(1, 2) for n in ("q", "k", "v"))
        scores = (q @ k.transpose(-1, -2)) / math.sqrt(dh)
        scores = scores.masked_fill(~causal, float("-inf"))
        o = (torch.softmax(scores, dim=-1) @ v).transpose(1, 2).reshape(B * S, d)
        h = h + bl(o, p("o")).reshape(B, S, d)
        m = _rmsnorm(h, p("mlp_norm"), cfg.norm_eps).reshape(B * S, d)
        h = h + bl(torch.nn.functional.silu(bl(m, p("gate"))) * bl(m, p("up")), p("down")).reshape(B, S, d)
    logits = _rmsnorm(h, params["final_norm"], cfg.norm_eps) @ params["head"].T
    return torch.nn.functional.cross_entropy(logits.reshape(B * S, -1), y_ids.reshape(-1))


def adamw_step(params: dict, grads: dict, state: dict, step: int, cfg):
    """One AdamW step in place (step counts from 1); no decay on norm gains."""
    b1, b2 = cfg.beta1, cfg.beta2
    bc1, bc2 = 1.0 - b1 ** step, 1.0 - b2 ** step
    with torch.no_grad():
        for name, p in params.items():
            g = grads[name]
            m, v = state.setdefault(name, (torch.zeros_like(p), torch.zeros_like(p)))
            m.mul_(b1).add_(g, alpha=1.0 - b1)
            v.mul_(b2).addcmul_(g, g, value=1.0 - b2)
            if not name.endswith("norm"):
                p.mul_(1.0 - cfg.lr * cfg.weight_decay)
            p.sub_(cfg.lr * (m / bc1) / (torch.sqrt(v / bc2) + cfg.eps))


def train_lm(init: dict, batches: torch.Tensor, cfg, device, steps: int | None = None, timing: bool = False):
    """Losses of `steps` AdamW steps from `init` on `batches` (token ids);
    with ``timing``, also the mean device time per step in ms (CUDA events)."""
    params = {n: t.to(device=device, dtype=torch.float32).contiguous().requires_grad_(True) for n, t in init.items()}
    ids_all = batches.to(device)
    state: dict = {}
    losses, times = [], []
    for t in range(steps if steps is not None else batches.shape[0]):
        if timing:
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
        loss = lm_loss(params, ids_all[t], cfg)
        grads = torch.autograd.grad(loss, list(params.values()))
        adamw_step(params, dict(zip(params.keys(), grads)), state, t + 1, cfg)
        if timing:
            e.record()
        losses.append(loss.detach())
        if timing:
            torch.cuda.synchronize(device)
            times.append(s.elapsed_time(e))
    if b.bl_get_last_error() != 0:
        raise RuntimeError("device error word set")
    out = [float(x) for x in losses]
    return (out, sum(times[1:]) / max(len(times) - 1, 1)) if timing else out
