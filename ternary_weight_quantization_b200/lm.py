"""A small decoder LM whose projections are BitLinear layers run by the library.

"bitnet-qat-train" (Measured behavior, Training) trains a 4-layer transformer
LM with the layer. Here the attention q, k, v, o and the SwiGLU gate, up,
down projections of every block go through the C ABI: the forward quantises
the fp32 master and the bf16 activations (``bl_quantize``) and runs the INT8
GEMM (``bl_forward``), keeping only the 2-bit codes, gamma, the INT8
activations and their scales; the backward rebuilds the operands from that
state (``bl_backward``: dX in bf16, dW in fp32). The pages give no other part
of the model; embedding, RMSNorm, attention, the SwiGLU gating, the LM head,
the cross-entropy and AdamW are plain PyTorch on the GPU, outside the
library, in the precision ``dtype`` (fp64 by default, the precision the LM
oracle keeps them in, so that a comparison of the two isolates the library's
calls; fp32 for a faster run):

  pre-norm blocks  h += o(attn(norm(h))); h += down(silu(gate(m)) * up(m)),
                   m = norm(h); RMSNorm x / sqrt(mean(x^2) + eps) * g
  attention        causal softmax, `heads` heads, no positional encoding
  loss             mean next-token cross-entropy
  AdamW            decoupled decay on the 2-D weights, not on the norm gains

Around each BitLinear call the model rounds as the calls require: its input
and its output gradient to bf16 (one rounding, straight from ``dtype``), the
master to fp32; y and dX come back in bf16 and dW in fp32. The embedding is a
one-hot product, so its gradient is a plain matrix product (the same sums on
every run) rather than an atomic scatter.
"""

from __future__ import annotations

import math

import torch

from . import bitlinear as b

__all__ = ["BitLinearFunction", "to_bf16_rn", "lm_loss", "adamw_step", "train_lm"]

_BF16_MIN_NORMAL = 2.0 ** -126


def to_bf16_rn(x: torch.Tensor) -> torch.Tensor:
    """Round a float64 (or float32) tensor to bf16 once, to nearest with ties to
    even. (A float64 -> bf16 cast through float32 rounds twice, which differs
    when the float32 value lands on a bf16 tie.) Finite inputs.

    Normal range: the float64 bit pattern is rounded at the 8th significant
    bit with an integer add of half a unit (less one, plus the kept lowest
    bit: ties go to even) and a mask; the result is exactly a bf16 value, so
    the cast that follows is exact. Below 2^-126 the bf16 quantum is 2^-133:
    the value is rounded on that grid with round-half-even.
    """
    if x.dtype == torch.float32:
        return x.to(torch.bfloat16)  # float32 -> bf16 is one rounding already
    x = x.to(torch.float64).contiguous()
    bits = x.view(torch.int64)
    keep = (bits >> 45) & 1
    rounded = ((bits + ((1 << 44) - 1) + keep) & ~((1 << 45) - 1)).view(torch.float64)
    tiny = torch.round(x * 2.0 ** 133) * 2.0 ** -133
    y = torch.where(x.abs() < _BF16_MIN_NORMAL, tiny, rounded)
    return y.to(torch.bfloat16)


class BitLinearFunction(torch.autograd.Function):
    """y [M, N] = BitLinear(x [M, K], W [N, K] master), in the dtype of x."""

    @staticmethod
    def forward(ctx, x2d, w):
        M, K = x2d.shape
        N = w.shape[0]
        dev = x2d.device
        xb = to_bf16_rn(x2d).contiguous()
        w32 = w.detach().to(torch.float32).contiguous()
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
        gamma = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(max(b.bl_quantize_weight_workspace_size(N, K), 16), dtype=torch.uint8, device=dev)
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sx = torch.empty(M, dtype=torch.float32, device=dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        b.bl_quantize(w32, xb, packed, gamma, xq, sx, ws)
        b.bl_forward(xq, sx, packed, gamma, y)
        ctx.save_for_backward(xq, sx, packed, gamma)
        ctx.out_dtype = x2d.dtype
        ctx.w_dtype = w.dtype
        return y.to(x2d.dtype)

    @staticmethod
    def backward(ctx, gy):
        xq, sx, packed, gamma = ctx.saved_tensors
        M, K = xq.shape
        N = packed.shape[0]
        dy = to_bf16_rn(gy).contiguous()
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dy.device)
        dW = torch.empty((N, K), dtype=torch.float32, device=dy.device)
        b.bl_backward(dy, xq, sx, packed, gamma, dX, dW)
        return dX.to(ctx.out_dtype), dW.to(ctx.w_dtype)


def _rmsnorm(x, g, eps):
    return x / torch.sqrt(torch.mean(x * x, dim=-1, keepdim=True) + eps) * g


def lm_loss(params: dict, ids: torch.Tensor, cfg) -> torch.Tensor:
    """Mean next-token cross-entropy of ids [B, S + 1] (parameters of one float dtype)."""
    B, S1 = ids.shape
    S, d, H = S1 - 1, cfg.d, cfg.heads
    dh = d // H
    x_ids, y_ids = ids[:, :S], ids[:, 1:]
    embed = params["embed"]
    one_hot = torch.nn.functional.one_hot(x_ids.reshape(-1), embed.shape[0]).to(embed.dtype)
    h = (one_hot @ embed).reshape(B, S, d)
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


def train_lm(init: dict, batches: torch.Tensor, cfg, device, steps: int | None = None, timing: bool = False,
             dtype=torch.float64):
    """Losses of `steps` AdamW steps from `init` on `batches` (token ids), with
    everything outside the BitLinear calls in ``dtype``; with ``timing``, also
    the mean device time per step in ms (CUDA events, first step excluded)."""
    params = {n: t.to(device=device, dtype=dtype).contiguous().requires_grad_(True) for n, t in init.items()}
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
