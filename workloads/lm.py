"""Seeded synthetic inputs of the small decoder LM trained with BitLinear layers.

The workload: a 4-layer decoder LM, model width 512, 8 heads, SwiGLU width
1408, vocabulary 8192, sequences of 256 tokens in batches of 8, 50 AdamW steps
at learning rate 1e-3. "bitnet-qat-train" (Measured behavior, Training) trains
a 4-layer transformer LM with the layer on identical batches and seeds and
compares its loss with the eager recipe's over the first 50 steps; it gives no
model sizes, so the ones here are this workload's. Token ids are uniform
random; nothing here is a dataset.

Only random draws with fixed seeds and shapes live here:
  lm_batches  token ids [steps, batch, seq + 1] (inputs and next-token targets)
  lm_init     the initial parameters (fp32, CPU), by name:
                embed            [V, d]        N(0, 0.02^2)
                layer{i}.attn_norm, layer{i}.mlp_norm, final_norm   [d] ones
                layer{i}.{q,k,v,o}  [d, d]       kaiming-uniform U(+-1/sqrt(d))
                layer{i}.{gate,up}  [F, d]       kaiming-uniform U(+-1/sqrt(d))
                layer{i}.down       [d, F]       kaiming-uniform U(+-1/sqrt(F))
                head             [V, d]        zeros (so the first loss is ln V)
Seeds: ids from ``seed``, parameter p (in the order above) from seed + 1000 + p.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch

__all__ = ["LMConfig", "LM_CONFIG", "LM_TINY", "lm_batches", "lm_init", "lm_param_names", "BITLINEAR_NAMES"]


@dataclass(frozen=True)
class LMConfig:
    layers: int = 4
    d: int = 512
    heads: int = 8
    ffn: int = 1408
    vocab: int = 8192
    seq: int = 256
    batch: int = 8
    steps: int = 50
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.01
    norm_eps: float = 1e-6


LM_CONFIG = LMConfig()
# a small case of the same model for CPU checks (every width a multiple of 32)
LM_TINY = LMConfig(layers=2, d=64, heads=2, ffn=96, vocab=128, seq=16, batch=2, steps=3)

BITLINEAR_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def lm_param_names(cfg: LMConfig):
    names = ["embed"]
    for i in range(cfg.layers):
        names += [f"layer{i}.attn_norm", f"layer{i}.mlp_norm"]
        names += [f"layer{i}.{n}" for n in BITLINEAR_NAMES]
    return names + ["final_norm", "head"]


def _shape(cfg: LMConfig, name: str):
    leaf = name.split(".")[-1]
    if name in ("embed", "head"):
        return (cfg.vocab, cfg.d)
    if leaf in ("attn_norm", "mlp_norm") or name == "final_norm":
        return (cfg.d,)
    if leaf in ("q", "k", "v", "o"):
        return (cfg.d, cfg.d)
    if leaf in ("gate", "up"):
        return (cfg.ffn, cfg.d)
    if leaf == "down":
        return (cfg.d, cfg.ffn)
    raise KeyError(name)


def lm_init(cfg: LMConfig, seed: int = 0):
    params = {}
    for p, name in enumerate(lm_param_names(cfg)):
        shape = _shape(cfg, name)
        g = torch.Generator().manual_seed(seed + 1000 + p)
        leaf = name.split(".")[-1]
        if name == "embed":
            t = torch.randn(shape, generator=g) * 0.02
        elif name == "head":
            t = torch.zeros(shape)
        elif len(shape) == 1:
            t = torch.ones(shape)
        else:
            bound = 1.0 / math.sqrt(shape[1])
            t = (torch.rand(shape, generator=g) * 2.0 - 1.0) * bound
        params[name] = t.to(torch.float32).contiguous()
    return params


def lm_batches(cfg: LMConfig, seed: int = 0):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, cfg.vocab, (cfg.steps, cfg.batch, cfg.seq + 1), generator=g, dtype=torch.int64)
