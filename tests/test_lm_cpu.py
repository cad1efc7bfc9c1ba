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


def test_single_rounding_to_bf16_matches_oracle():
    """The LM's fp64 -> bf16 cast (one rounding) against the oracle's."""
    import numpy as np
    from oracle import bitlinear_ref as ref
    from ternary_weight_quantization_b200.lm import to_bf16_rn
    rng = np.random.default_rng(11)
    vals = [rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
            rng.standard_normal(2000) * 1e-39, rng.standard_normal(2000) * 1e-44]
    # values just above and below bf16 ties, where rounding through fp32 first
    # would land on the tie and round to even instead of away
    base = (rng.integers(0x0080, 0x7F00, 4000).astype(np.uint32) << 16) | 0x8000   # finite fp32 bf16 ties
    ties = base.view(np.float32).astype(np.float64)
    vals += [ties * (1 + 2.0 ** -30), ties * (1 - 2.0 ** -30), ties, -ties * (1 + 2.0 ** -30)]
    vals.append(np.array([0.0, -0.0, 1.0 + 2.0 ** -8 + 2.0 ** -30, 2.0 ** -126, -2.0 ** -127, 2.0 ** -133 * 1.5]))
    x = np.concatenate(vals)
    got = to_bf16_rn(torch.from_numpy(x)).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref.round_to_bf16_bits(x))
