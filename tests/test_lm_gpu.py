"""GPU: the decoder LM trained through the library tracks the LM oracle.

Bar: the first loss is ln V (zero-initialised head), and at every step the
loss of the model trained through the C ABI is within 0.01 of the LM oracle's
("bitnet-qat-train", Measured behavior, Training: the layer's LM tracks the
eager recipe's loss over the first 50 steps). The model keeps everything
outside the BitLinear calls in fp64, as the oracle does, so the two runs
differ only where the library's calls and the oracle's BitLinear steps do
(fp32 sums of dX and dW on the tensor cores against fp64 sums rounded once).
The small case runs the oracle live; the full-size case compares with the
stored oracle curve (tests/golden/make_lm_golden.py writes it).
"""

import json
import math
import os

import pytest
import torch

from tests.conftest import GOLDEN
from workloads.lm import LM_CONFIG, LM_TINY, lm_batches, lm_init

pytestmark = pytest.mark.gpu


def test_small_lm_tracks_live_oracle():
    from oracle import lm_ref
    from ternary_weight_quantization_b200.lm import train_lm
    cfg = LM_TINY
    init, batches = lm_init(cfg, seed=1), lm_batches(cfg, seed=1)
    gpu = train_lm(init, batches, cfg, torch.device("cuda"))
    orc, _ = lm_ref.train(init, batches, cfg)
    assert abs(gpu[0] - math.log(cfg.vocab)) < 1e-5
    assert max(abs(a - b) for a, b in zip(gpu, orc)) <= 0.01


def test_lm_first_loss_is_ln_vocab():
    from ternary_weight_quantization_b200.lm import train_lm
    cfg = LM_CONFIG
    losses = train_lm(lm_init(cfg, seed=0), lm_batches(cfg, seed=0), cfg, torch.device("cuda"), steps=1)
    assert abs(losses[0] - math.log(cfg.vocab)) < 1e-9


def test_lm_run_is_deterministic():
    from ternary_weight_quantization_b200.lm import train_lm
    cfg = LM_CONFIG
    a = train_lm(lm_init(cfg, seed=0), lm_batches(cfg, seed=0), cfg, torch.device("cuda"), steps=4)
    b = train_lm(lm_init(cfg, seed=0), lm_batches(cfg, seed=0), cfg, torch.device("cuda"), steps=4)
    assert a == b


def test_lm_tracks_stored_oracle_curve():
    from ternary_weight_quantization_b200.lm import train_lm
    with open(os.path.join(GOLDEN, "lm_oracle_losses.json")) as f:
        gold = json.load(f)
    cfg = LM_CONFIG
    assert gold["config"]["steps"] == cfg.steps and gold["seed"] == 0 and gold.get("dtype", "fp64") == "fp64"
    losses = train_lm(lm_init(cfg, seed=0), lm_batches(cfg, seed=0), cfg, torch.device("cuda"))
    diffs = [abs(a - b) for a, b in zip(losses, gold["losses"])]
    assert len(diffs) == cfg.steps
    worst = max(diffs)
    assert worst <= 0.01, f"max |dloss| {worst:.4g} at step {diffs.index(worst)}"
