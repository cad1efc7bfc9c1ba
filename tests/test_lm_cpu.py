"""The LM's host code on the CPU, without the library: with every BitLinear
replaced by a plain product, the model of ternary_weight_quantization_b200.lm
computes the same loss as the oracle's model with its quantisers off, and
the two AdamW steps agree. (The quantised path itself is checked on the GPU.)"""

import pytest
import torch

from oracle import lm_ref
from workloads.lm import LM_TINY, lm_batches, lm_init


def _params64(cfg, seed):
    init = lm_init(cfg, seed=seed)
    init["head"] = torch.randn(init["head"].shape, generator=torch.Generator().manual_seed(seed + 1)) * 0.05
    return {n: t.to(torch.float64) for n, t in init.items()}


def test_model_structure_matches_oracle(monkeypatch):
    from ternary_weight_quantization_b200 import lm as plm
    monkeypatch.setattr(plm.BitLinearFunction, "apply", staticmethod(lambda x, w: x @ w.T))
    cfg = LM_TINY
    params = _params64(cfg, 2)
    ids = lm_batches(cfg, seed=3)[0]
    a = plm.lm_loss(params, ids, cfg)
    b = lm_ref.lm_loss(params, ids, cfg, quantize=False)
    assert a.item() == pytest.approx(b.item(), rel=1e-12, abs=1e-12)


def test_adamw_steps_agree():
    from ternary_weight_quantization_b200 import lm as plm
    cfg = LM_TINY
    g = torch.Generator().manual_seed(4)
    p1 = {"layer0.q": torch.randn(8, 8, generator=g, dtype=torch.float64), "final_norm": torch.randn(8, generator=g, dtype=torch.float64)}
    p2 = {k: v.clone() for k, v in p1.items()}
    s1, s2 = {}, {}
    for step in range(1, 4):
        grads = {k: torch.randn(v.shape, generator=g, dtype=torch.float64) for k, v in p1.items()}
        plm.adamw_step(p1, grads, s1, step, cfg)
        lm_ref.adamw_step(p2, grads, s2, step, cfg)
    for k in p1:
        assert torch.allclose(p1[k], p2[k], rtol=1e-14, atol=1e-15)
