"""Plain CPU oracle of a small decoder LM trained with BitLinear layers.

TEST INFRASTRUCTURE ONLY: imported by the tests and by the committed script
that writes the stored loss curve under tests/golden/. The CUDA library and
its Python package share no code with this file, and neither imports the
other.

"bitnet-qat-train" (Measured behavior, Training) trains a 4-layer transformer
LM with the layer and tracks the loss of the eager fake-quant recipe on
identical batches and seeds. This is that recipe, in plain PyTorch CPU ops in
fp64, with every BitLinear (attention q, k, v, o and the SwiGLU gate, up,
down projections) computed by the BitLinear oracle (``bitlinear_ref``) and
rounded where the library's calls round: the layer's input and its output
gradient to bf16 (the calls take bf16), y and dX to bf16, dW to fp32, the fp32
masters ternarised. Everything else (embedding, RMSNorm, attention, SwiGLU
gating, LM head, cross-entropy) is fp64 autograd, and AdamW is written out.

Readings where the pages give no model:
  * pre-norm blocks: h += o(attn(norm(h))); h += down(silu(gate(m)) * up(m))
    with m = norm(h); RMSNorm x / sqrt(mean(x^2) + eps) * g, eps 1e-6;
  * causal softmax attention with 8 heads, no positional encoding;
  * embedding and LM head in full precision; the loss is the mean next-token
    cross-entropy;
  * AdamW as torch defines it (decoupled decay p *= 1 - lr * wd, then
    p -= lr * m_hat / (sqrt(v_hat) + eps)); decay on the 2-D weights, not on
    the RMSNorm gains.

Pinning: tests/test_oracle_lm_pins.py (first loss = ln V with the zero-init
head, finite-difference gradients of the model with the quantisers replaced
by identity, the BitLinear wiring against ``bitlinear_ref``, a closed-form
AdamW step, causality of the attention).
"""

from __future__ import annotations

import math

import numpy as np
import torch

from . import bitlinear_ref as ref

__all__ = ["BitLinearRef", "lm_loss", "adamw_step", "train"]

_BL_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def _bf16(x: np.ndarray) -> np.ndarray:
    return ref.bf16_bits_to_f32(ref.round_to_bf16_bits(x)).astype(np.float64)


class BitLinearRef(torch.autograd.Function):
    """y = x W^T through the BitLinear oracle; straight-through backward."""

    @staticmethod
    def forward(ctx, x, w):
        x32 = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(x.detach().numpy()))
        w32 = w.detach().numpy().astype(np.float32)
        codes, gamma = ref.ternarize(w32)
        q, sx = ref.quantize_activations(x32)
        y32 = ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma)
        ctx.state = (codes, gamma, q, sx)
        return torch.from_numpy(_bf16(y32)).to(x.dtype)

    @staticmethod
    def backward(ctx, gy):
        codes, gamma, q, sx = ctx.state
        dy = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(gy.detach().numpy()))
        x_hat = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.dequantize_activations(q, sx)))
        dx = _bf16(ref.backward_dx(dy, codes, gamma))
        dw = ref.backward_dw(dy, x_hat).astype(np.float32).astype(np.float64)
        return torch.from_numpy(dx).to(gy.dtype), torch.from_numpy(dw).to(gy.dtype)


def _linear(x2d, w, quantize: bool):
    return BitLinearRef.apply(x2d, w) if quantize else x2d @ w.T


def _rmsnorm(x, g, eps):
    return x / torch.sqrt(torch.mean(x * x, dim=-1, keepdim=True) + eps) * g


def lm_loss(params: dict, ids: torch.Tensor, cfg, quantize: bool = True, reduction: str = "mean") -> torch.Tensor:
    """Next-token cross-entropy of ids [B, S + 1] (fp64 parameters), averaged
    over the B * S positions (``reduction="none"``: one value per position)."""
    B, S1 = ids.shape
    S, d, H = S1 - 1, cfg.d, cfg.heads
    dh = d // H
    x_ids, y_ids = ids[:, :S], ids[:, 1:]
    h = params["embed"][x_ids]                                   # [B, S, d]
    causal = torch.ones(S, S, dtype=torch.bool).tril()
    for i in range(cfg.layers):
        p = lambda n: params[f"layer{i}.{n}"]  # noqa: E731
        a = _rmsnorm(h, p("attn_norm"), cfg.norm_eps).reshape(B * S, d)
        q, k, v = (_linear(a, p(n), quantize).reshape(B, S, H, dh).transpose(1, 2) for n in ("q", "k", "v"))
        scores = (q @ k.transpose(-1, -2)) / math.sqrt(dh)
        scores = scores.masked_fill(~causal, float("-inf"))
        att = torch.softmax(scores, dim=-1) @ v                   # [B, H, S, dh]
        o = att.transpose(1, 2).reshape(B * S, d)
        h = h + _linear(o, p("o"), quantize).reshape(B, S, d)
        m = _rmsnorm(h, p("mlp_norm"), cfg.norm_eps).reshape(B * S, d)
        gate = _linear(m, p("gate"), quantize)
        up = _linear(m, p("up"), quantize)
        h = h + _linear(torch.nn.functional.silu(gate) * up, p("down"), quantize).reshape(B, S, d)
    logits = _rmsnorm(h, params["final_norm"], cfg.norm_eps) @ params["head"].T
    return torch.nn.functional.cross_entropy(logits.reshape(B * S, -1), y_ids.reshape(-1), reduction=reduction)


def _decayed(name: str) -> bool:
    return not name.endswith("norm")


def adamw_step(params: dict, grads: dict, state: dict, step: int, cfg):
    """One AdamW step in place (step counts from 1)."""
    b1, b2 = cfg.beta1, cfg.beta2
    bc1, bc2 = 1.0 - b1 ** step, 1.0 - b2 ** step
    with torch.no_grad():
        for name, p in params.items():
            g = grads[name]
            m, v = state.setdefault(name, (torch.zeros_like(p), torch.zeros_like(p)))
            m.mul_(b1).add_(g, alpha=1.0 - b1)
            v.mul_(b2).add_(g * g, alpha=1.0 - b2)
            if _decayed(name):
                p.mul_(1.0 - cfg.lr * cfg.weight_decay)
            p.sub_(cfg.lr * (m / bc1) / (torch.sqrt(v / bc2) + cfg.eps))


def train(init: dict, batches: torch.Tensor, cfg, steps: int | None = None, quantize: bool = True,
          dtype=torch.float64):
    """Losses of `steps` AdamW steps from `init` (fp32 tensors) on `batches`.

    ``dtype`` is the precision of everything outside the BitLinear oracle
    (parameters, AdamW state, the other layers): fp64 by default; fp32 gives
    a run in the precision a GPU fp32 model keeps, to measure how far two
    precisions alone drift apart over the steps."""
    params = {n: t.detach().to(dtype).clone().requires_grad_(True) for n, t in init.items()}
    state: dict = {}
    losses = []
    for t in range(steps if steps is not None else batches.shape[0]):
        loss = lm_loss(params, batches[t], cfg, quantize)
        grads = torch.autograd.grad(loss, list(params.values()))
        losses.append(float(loss.detach()))
        adamw_step(params, dict(zip(params.keys(), grads)), state, t + 1, cfg)
    return losses, params
