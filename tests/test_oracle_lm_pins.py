"""Pins of the LM oracle (oracle/lm_ref.py) on a small case, CPU only.

Each pin fixes what mathematics decides, not what the oracle computes:
the first loss with a zero head is ln V exactly; with the quantisers replaced
by identity the model's gradients equal central finite differences; the
BitLinear autograd function wires the pinned ``bitlinear_ref`` steps the
right way round; one AdamW step equals its closed form; a future token never
changes an earlier position's loss.
"""

import math

import numpy as np
import torch

from oracle import bitlinear_ref as ref
from oracle import lm_ref
from workloads.lm import LM_TINY, lm_batches, lm_init


def _params64(init):
    return {n: t.to(torch.float64).clone().requires_grad_(True) for n, t in init.items()}


def test_first_loss_is_ln_vocab_with_zero_head():
    cfg = LM_TINY
    losses, _ = lm_ref.train(lm_init(cfg), lm_batches(cfg), cfg, steps=1)
    assert abs(losses[0] - math.log(cfg.vocab)) < 1e-12


def test_gradients_match_finite_differences_without_quantisers():
    cfg = LM_TINY
    init = lm_init(cfg, seed=3)
    g = torch.Generator().manual_seed(4)
    init["head"] = torch.randn(init["head"].shape, generator=g) * 0.05  # nonzero head: every path live
    params = _params64(init)
    ids = lm_batches(cfg, seed=5)[0]
    loss = lm_ref.lm_loss(params, ids, cfg, quantize=False)
    grads = dict(zip(params, torch.autograd.grad(loss, list(params.values()))))
    rng = np.random.default_rng(6)
    for name in ["embed", "layer0.attn_norm", "layer0.q", "layer0.k", "layer0.v", "layer1.o",
                 "layer1.gate", "layer1.up", "layer1.down", "layer1.mlp_norm", "final_norm", "head"]:
        p = params[name]
        for _ in range(3):
            idx = tuple(int(rng.integers(0, s)) for s in p.shape)
            if name == "embed":  # pick a row that the batch uses
                idx = (int(ids[0, 0]),) + idx[1:]
            h = 1e-6
            with torch.no_grad():
                old = p[idx].item()
                p[idx] = old + h
                up = lm_ref.lm_loss(params, ids, cfg, quantize=False).item()
                p[idx] = old - h
                dn = lm_ref.lm_loss(params, ids, cfg, quantize=False).item()
                p[idx] = old
            fd = (up - dn) / (2 * h)
            assert abs(fd - grads[name][idx].item()) <= 1e-6 + 1e-4 * abs(fd), (name, idx)


def test_bitlinear_function_wiring():
    rng = np.random.default_rng(7)
    x = torch.from_numpy(rng.standard_normal((6, 64)))
    w = torch.from_numpy(rng.standard_normal((32, 64)) * 0.05)
    dy = torch.from_numpy(rng.standard_normal((6, 32)))
    xr, wr = x.clone().requires_grad_(True), w.clone().requires_grad_(True)
    y = lm_ref.BitLinearRef.apply(xr, wr)
    y.backward(dy)
    # the same chain written with the pinned oracle steps
    x32 = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(x.numpy()))
    codes, gamma = ref.ternarize(w.numpy().astype(np.float32))
    q, sx = ref.quantize_activations(x32)
    y_bits = ref.round_to_bf16_bits(ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma))
    assert np.array_equal(ref.round_to_bf16_bits(y.detach().numpy()), y_bits)
    dyb = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(dy.numpy()))
    assert np.array_equal(ref.round_to_bf16_bits(xr.grad.numpy()),
                          ref.round_to_bf16_bits(ref.backward_dx(dyb, codes, gamma)))
    x_hat = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.dequantize_activations(q, sx)))
    assert np.array_equal(wr.grad.numpy().astype(np.float32), ref.backward_dw(dyb, x_hat).astype(np.float32))
    assert xr.grad.shape == x.shape and wr.grad.shape == w.shape


def test_adamw_step_closed_form():
    cfg = LM_TINY
    p = {"w": torch.tensor([1.0, -2.0], dtype=torch.float64), "g_norm": torch.tensor([3.0], dtype=torch.float64)}
    grads = {"w": torch.tensor([0.5, 0.0], dtype=torch.float64), "g_norm": torch.tensor([-0.25], dtype=torch.float64)}
    lm_ref.adamw_step(p, grads, {}, 1, cfg)
    lr, wd, eps = cfg.lr, cfg.weight_decay, cfg.eps
    # step 1: m_hat = g, v_hat = g^2, so the step is lr * g / (|g| + eps)
    assert p["w"][0].item() == (1.0 * (1 - lr * wd)) - lr * 0.5 / (0.5 + eps)
    assert p["w"][1].item() == -2.0 * (1 - lr * wd)          # zero gradient: decay only
    assert p["g_norm"][0].item() == 3.0 + lr * 0.25 / (0.25 + eps)  # norm gains are not decayed


def test_attention_is_causal():
    cfg = LM_TINY
    init = lm_init(cfg, seed=8)
    init["head"] = torch.randn(init["head"].shape, generator=torch.Generator().manual_seed(9)) * 0.05
    params = _params64(init)
    ids = lm_batches(cfg, seed=10)[0][:1].clone()        # [1, S + 1]
    S = cfg.seq

    def per_position_losses(tok):
        with torch.no_grad():
            return lm_ref.lm_loss(params, tok, cfg, quantize=False, reduction="none")

    base = per_position_losses(ids)
    changed = ids.clone()
    # token S-1 is the last input and the target of position S-2
    changed[0, S - 1] = (changed[0, S - 1] + 1) % cfg.vocab
    after = per_position_losses(changed)
    assert torch.equal(base[: S - 2], after[: S - 2])         # earlier positions untouched
    assert base[S - 1] != after[S - 1]                        # the position that reads it
