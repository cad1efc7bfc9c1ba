"""Pins of the CPU oracle against what the pages and mathematics fix.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, the wrong rounding mode or scale)
fails at least one of them. None of these tests needs a GPU.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import bitlinear_ref as ref
from tests.conftest import GOLDEN

# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------


def _load_dyadic():
    with open(os.path.join(GOLDEN, "dyadic_bitlinear.json")) as f:
        return json.load(f)


def _torch_bf16_bits(x_f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------
# bf16 rounding: a library routine and a hand-built double-rounding case
# --------------------------------------------------------------------------


def test_bf16_rounding_matches_torch_on_f32():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        rng.standard_normal(2000).astype(np.float32) * np.float32(1e-38),   # subnormals
        rng.standard_normal(2000).astype(np.float32) * np.float32(1e37),    # near overflow
        # exact ties between two bf16 neighbours (bit 15 set, bits 0..14 clear)
        ((rng.integers(0, 2 ** 16, 4000, dtype=np.uint32) << 16) | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 3.3895314e38, -3.3895314e38, 1.0, -1.0], np.float32),
    ])
    vals = vals[np.isfinite(vals)]
    np.testing.assert_array_equal(ref.round_to_bf16_bits(vals), _torch_bf16_bits(vals))


def test_bf16_rounding_is_single_rounding_from_f64():
    # 1 + 2^-8 + 2^-30: rounding straight to bf16 (quantum 2^-7) goes up;
    # rounding to fp32 first would make an exact tie and go down to 1.0.
    x = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30, -(1.0 + 2.0 ** -8 + 2.0 ** -30)])
    out = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(x))
    np.testing.assert_array_equal(out, np.array([1.0078125, -1.0078125], np.float32))
    assert ref.bf16_bits_to_f32(ref.round_to_bf16_bits(np.array([1.0 + 2.0 ** -8])))[0] == 1.0


# --------------------------------------------------------------------------
# S1: ternarisation and packing
# --------------------------------------------------------------------------


def test_ternarize_hand_derived_fixture():
    g = _load_dyadic()
    w = np.array(g["W"], np.float32)
    codes, gamma = ref.ternarize(w)
    assert gamma.dtype == np.float32 and float(gamma) == g["gamma"]
    np.testing.assert_array_equal(codes, np.array(g["codes"], np.int8))
    np.testing.assert_array_equal(ref.pack_ternary(codes), np.array(g["packed"], np.uint8))
    np.testing.assert_array_equal(ref.unpack_ternary(ref.pack_ternary(codes), 8), codes)


def test_pack_roundtrip_and_field_values():
    rng = np.random.default_rng(2)
    c = rng.integers(-1, 2, size=(37, 64)).astype(np.int8)
    p = ref.pack_ternary(c)
    assert p.shape == (37, 16)
    np.testing.assert_array_equal(ref.unpack_ternary(p, 64), c)
    fields = np.stack([(p >> (2 * j)) & 3 for j in range(4)])
    assert not np.any(fields == 2)
    with pytest.raises(ValueError):
        ref.unpack_ternary(np.array([[0b10]], np.uint8), 4)


def test_ternarize_degenerate_tensors():
    codes, gamma = ref.ternarize(np.zeros((4, 32), np.float32))
    assert float(gamma) == float(np.float32(1e-5))
    assert not codes.any()
    # below the clamp floor every |w| / 1e-5 <= 0.5 -> code 0; above it, sign
    w = np.full((1, 32), 4e-6, np.float32)
    w[0, 0] = 6e-6
    codes, gamma = ref.ternarize(w)
    assert float(gamma) == float(np.float32(1e-5))
    assert codes[0, 0] == 1 and not codes[0, 1:].any()


@pytest.mark.parametrize("kind,expected", [
    ("gauss", 2.0 * 0.5 * (1.0 + math.erf(0.5 * math.sqrt(2.0 / math.pi) / math.sqrt(2.0))) - 1.0),
    ("uniform", 0.25),
])
def test_ternary_zero_fraction_closed_form(kind, expected):
    """Code statistics ("bitlinear.py", ternary_stats) against closed forms.

    Gaussian masters: gamma -> sigma*sqrt(2/pi), P(code 0) = P(|Z| <= gamma/2).
    Uniform(-b, b): gamma -> b/2, P(|w| <= b/4) = 1/4; codes +-1 equally likely.
    """
    rng = np.random.default_rng(3)
    n = 1 << 20
    w = (rng.standard_normal(n) if kind == "gauss" else rng.uniform(-1.0, 1.0, n)) * 0.02
    codes, _ = ref.ternarize(w.astype(np.float32).reshape(1024, 1024))
    frac0 = float(np.mean(codes == 0))
    sigma = math.sqrt(expected * (1 - expected) / n)
    assert abs(frac0 - expected) < 5 * sigma
    pos, neg = float(np.mean(codes == 1)), float(np.mean(codes == -1))
    assert abs(pos - neg) < 10 * math.sqrt(0.5 / n)


def test_ternarize_is_deterministic():
    rng = np.random.default_rng(4)
    w = rng.standard_normal((64, 96)).astype(np.float32)
    a = ref.ternarize(w)
    b = ref.ternarize(w.copy())
    np.testing.assert_array_equal(a[0], b[0])
    assert a[1].tobytes() == b[1].tobytes()


def test_gamma_uses_exact_mean():
    # Many tiny values after one big one: a naive fp32 running sum would drop
    # them; the exactly rounded fp64 mean keeps them.
    w = np.full(1 << 16, 1e-3, np.float32)
    w[0] = 1e4
    expected = np.float32((1e4 + ((1 << 16) - 1) * float(np.float32(1e-3))) / (1 << 16))
    assert ref.absmean_gamma(w.reshape(256, 256)) == expected


@pytest.mark.parametrize("case,expected", [("tie", 1.0), ("above", 1.0 + 2.0 ** -23), ("below", 1.0)])
@pytest.mark.parametrize("w_dtype", ["bf16", "f32"])
def test_gamma_at_an_fp32_midpoint(case, expected, w_dtype):
    """Tensors whose mean |W| is 1 + 2^-24 (the midpoint between the fp32
    neighbours 1 and 1 + 2^-23) exactly, or 2^-44 above or below it: the
    exactly rounded mean gives the closed forms (the tie to the even 1.0).
    Every magnitude >= 1 gets code +-1 with its sign, every smaller one 0."""
    from workloads import gamma_midpoint_weights
    w = gamma_midpoint_weights(case, torch.bfloat16 if w_dtype == "bf16" else torch.float32)
    wf = w.float().numpy()
    codes, gamma = ref.ternarize(wf)
    assert gamma == np.float32(expected)
    big = np.abs(wf) >= 1.0
    np.testing.assert_array_equal(codes[big], np.sign(wf[big]).astype(np.int8))
    assert not codes[~big].any()


# --------------------------------------------------------------------------
# S2: activation quantisation
# --------------------------------------------------------------------------


def test_activation_hand_derived_fixture():
    g = _load_dyadic()
    x = np.array(g["x"], np.float32)
    q, sx = ref.quantize_activations(x)
    np.testing.assert_array_equal(q, np.array(g["q"], np.int8))
    np.testing.assert_array_equal(sx, np.array(g["sx"], np.float32))


def test_activation_ties_and_reciprocal_scale():
    # absmax 1 -> inv = 127: -0.5 * 127 = -63.5 rounds to the even -64.
    x = np.array([[1.0, -0.5, 0.25, 0.0, 0.75, -1.0, 0.125, 0.375]], np.float32)
    q, sx = ref.quantize_activations(x)
    np.testing.assert_array_equal(q[0], [127, -64, 32, 0, 95, -127, 16, 48])
    assert sx[0].view(np.uint32) == 1006699012          # fp32(1/127) = 0x3C010204
    # all-zero token: the 1e-5 floor applies, q = 0, s_x = fp32(1e-5 / 127)
    q0, sx0 = ref.quantize_activations(np.zeros((1, 64), np.float32))
    assert not q0.any() and sx0[0].view(np.uint32) == 866719708


def test_activation_invariants_random():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((257, 384)).astype(np.float32)
    x[rng.random(x.shape) < 0.01] *= 20
    q, sx = ref.quantize_activations(x)
    assert q.min() >= -127 and q.max() <= 127
    am = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(q[np.arange(257), am]) == 127)
    # dequantised values stay within half a step of the input
    xh = q.astype(np.float64) * sx[:, None]
    assert np.all(np.abs(xh - x) <= 0.5 * sx[:, None] * (1 + 1e-5))


# --------------------------------------------------------------------------
# S3: forward
# --------------------------------------------------------------------------


def test_forward_hand_derived_fixture():
    g = _load_dyadic()
    q = np.array(g["q"], np.int8)
    codes = np.array(g["codes"], np.int8)
    acc = ref.forward_accumulate(q, codes)
    np.testing.assert_array_equal(acc, np.array(g["acc"]))
    y = ref.forward_output(acc, np.array(g["sx"], np.float32), np.float32(g["gamma"]))
    np.testing.assert_array_equal(y, np.array(g["y"], np.float32))


def test_forward_accumulate_brute_force_all_code_rows():
    """Every one of the 3^4 ternary rows of length 4 against a loop dot product."""
    rng = np.random.default_rng(6)
    rows = np.array(np.meshgrid(*[[-1, 0, 1]] * 4, indexing="ij")).reshape(4, -1).T
    codes = np.tile(rows, (1, 8)).astype(np.int8)           # [81, 32]
    q = rng.integers(-127, 128, size=(5, 32)).astype(np.int8)
    acc = ref.forward_accumulate(q, codes)
    for m in range(q.shape[0]):
        for n in range(codes.shape[0]):
            s = 0
            for k in range(32):
                s += int(q[m, k]) * int(codes[n, k])
            assert acc[m, n] == s


def test_forward_accumulate_extremes_exact():
    k = 8192
    q = np.full((2, k), 127, np.int8)
    q[1] = -127
    c = np.ones((3, k), np.int8)
    c[1] = -1
    c[2, ::2] = 0
    acc = ref.forward_accumulate(q, c)
    assert acc[0, 0] == 127 * k and acc[1, 0] == -127 * k and acc[0, 1] == -127 * k
    assert acc[0, 2] == 127 * (k // 2)


# --------------------------------------------------------------------------
# S4: straight-through backward
# --------------------------------------------------------------------------


def test_backward_hand_derived_fixture():
    g = _load_dyadic()
    dy = np.array(g["dY"], np.float32)
    codes = np.array(g["codes"], np.int8)
    xh = ref.dequantize_activations(np.array(g["q"], np.int8), np.array(g["sx"], np.float32))
    np.testing.assert_array_equal(xh, np.array(g["x_hat"], np.float32))
    np.testing.assert_array_equal(ref.backward_dx(dy, codes, np.float32(g["gamma"])), np.array(g["dX"]))
    np.testing.assert_array_equal(ref.backward_dw(dy, xh), np.array(g["dW"]))


def test_backward_adjoint_identity_and_loops():
    """<dY, x_hat W_hat^T> = <dX, x_hat> = <dW, W_hat> for the linear map.

    Non-square shapes make any transposed operand fail on shape or value.
    """
    rng = np.random.default_rng(7)
    M, K, N = 5, 12, 7
    x = rng.standard_normal((M, K)).astype(np.float32)
    w = rng.standard_normal((N, K)).astype(np.float32)
    dy = rng.standard_normal((M, N)).astype(np.float32)
    codes, gamma = ref.ternarize(w)
    q, sx = ref.quantize_activations(x)
    xh = ref.dequantize_activations(q, sx).astype(np.float64)
    wh = codes.astype(np.float64) * float(gamma)
    dx = ref.backward_dx(dy, codes, gamma)
    dw = ref.backward_dw(dy, xh)
    assert dx.shape == (M, K) and dw.shape == (N, K)
    lhs = float(np.sum(dy.astype(np.float64) * (xh @ wh.T)))
    assert math.isclose(lhs, float(np.sum(dx * xh)), rel_tol=1e-12)
    assert math.isclose(lhs, float(np.sum(dw * wh)), rel_tol=1e-12)
    for m in range(M):
        for k in range(K):
            s = sum(float(dy[m, n]) * float(codes[n, k]) for n in range(N)) * float(gamma)
            assert math.isclose(dx[m, k], s, rel_tol=1e-12, abs_tol=1e-12)
    for n in range(N):
        for k in range(K):
            s = sum(float(dy[m, n]) * xh[m, k] for m in range(M))
            assert math.isclose(dw[n, k], s, rel_tol=1e-12, abs_tol=1e-12)


def _fake_quant_linear_torch(x, w, w_eps=1e-8):
    """The eager fake-quant BitLinear of "bitlinear.py" (forward with the
    detach-based straight-through estimator), restated in torch fp64.
    ``w_eps`` is the recipe's additive term on the weight scale."""
    w_scale = w.abs().mean() + w_eps
    w_q = torch.clamp(torch.round(w / w_scale), -1, 1)
    w_ste = w + (w_q * w_scale - w).detach()
    x_scale = x.abs().amax(dim=-1, keepdim=True).clamp(min=1e-8)
    x_q = torch.clamp(torch.round(x * 127.0 / x_scale), -127, 127)
    x_ste = x + (x_q * x_scale / 127.0 - x).detach()
    return torch.nn.functional.linear(x_ste, w_ste), w_q, x_q


def test_matches_eager_fake_quant_formulation_fp64():
    """Oracle (integer accumulate, then scale) vs the eager fake-quant recipe
    (dequantise, then float matmul), gradients by torch autograd."""
    rng = np.random.default_rng(8)
    M, K, N = 9, 64, 24
    x64 = rng.standard_normal((M, K))
    w64 = rng.standard_normal((N, K)) * 0.02
    dy64 = rng.standard_normal((M, N))
    xt = torch.tensor(x64, requires_grad=True)
    wt = torch.tensor(w64, requires_grad=True)
    y_t, w_q, x_q = _fake_quant_linear_torch(xt, wt)
    y_t.backward(torch.tensor(dy64))

    codes, gamma = ref.ternarize(w64, np.float64)
    q, sx = ref.quantize_activations(x64, np.float64)
    np.testing.assert_array_equal(codes, w_q.detach().numpy().astype(np.int8))
    np.testing.assert_array_equal(q, x_q.detach().numpy().astype(np.int8))
    # the recipe adds 1e-8 to gamma where the oracle clamps: results that
    # carry gamma differ by about 1e-8 / gamma relative, nothing more
    tol = 4e-8 / float(gamma)
    y = ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma, np.float64)
    np.testing.assert_allclose(y, y_t.detach().numpy(), rtol=tol, atol=1e-12)
    xh = ref.dequantize_activations(q, sx, np.float64)
    np.testing.assert_allclose(ref.backward_dx(dy64, codes, gamma), xt.grad.numpy(), rtol=tol, atol=1e-12)
    np.testing.assert_allclose(ref.backward_dw(dy64, xh), wt.grad.numpy(), rtol=1e-9, atol=1e-12)


def test_worked_example_sign_equality():
    """The 3-layer 7->6->5->4 net of "1BitTraining.md", built from the oracle.

    The page claims that under the identity STE the gradient with respect to
    each latent weight equals the gradient with respect to the quantised
    weight, element by element (sign equality True for all three layers).
    The test builds the net from the oracle's steps in fp64, derives the
    quantised-weight gradients by hand through the chain rule, and checks
    them against torch autograd through the eager STE formulation.
    """
    printed = {}
    with open(os.path.join(GOLDEN, "p1_printed_output.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, *vals = line.split()
                printed[key] = vals
    rs = np.random.RandomState(0)
    W = [rs.randn(6, 7), rs.randn(5, 6), rs.randn(4, 5)]
    x0 = rs.randn(2, 7)
    target = rs.randn(2, 4)

    # forward through the oracle: quantise input of every layer, integer
    # accumulate, scale
    acts, quants = [], []
    h = x0
    for i, w in enumerate(W):
        codes, gamma = ref.ternarize(w, np.float64)
        q, sx = ref.quantize_activations(h, np.float64)
        acts.append(ref.dequantize_activations(q, sx, np.float64))
        quants.append((codes, gamma))
        h = ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma, np.float64)
    delta = h - target
    grads_q = [None] * 3
    for i in (2, 1, 0):
        codes, gamma = quants[i]
        grads_q[i] = ref.backward_dw(delta, acts[i])
        delta = ref.backward_dx(delta, codes, gamma)

    # the same net with latent weights as leaves, STE via autograd
    wts = [torch.tensor(w, requires_grad=True) for w in W]
    hh = torch.tensor(x0)
    for wt in wts:
        # no additive eps: the weight scales here are far above any floor
        hh, _, _ = _fake_quant_linear_torch(hh, wt, w_eps=0.0)
    loss = 0.5 * torch.sum((hh - torch.tensor(target)) ** 2)
    loss.backward()
    for i in range(3):
        g_fp = wts[i].grad.numpy()
        np.testing.assert_allclose(grads_q[i], g_fp, rtol=1e-9, atol=1e-12)
        same = bool(np.all(np.sign(g_fp) == np.sign(grads_q[i])))
        assert same == (printed[f"layer{i + 1}_sign_equality"][0] == "True")


def _page_listing_net(W, x0, target):
    """The 3-layer net of "1BitTraining.md" as its listing computes it,
    restated here: its quantisers return the dequantised values (activations
    scaled by 127 / max(max|x|, 1e-5) along the last axis, rounded, clipped
    to [-128, 127] and scaled back; weights multiplied by 1 / max(mean|w|,
    1e-5), rounded, clipped to [-1, 1] and scaled back), the forward uses only
    quantised weights and activations with no quantiser on the output, the
    loss is half the squared error, and the backward takes the quantisers'
    derivative as 1. Returns (loss, deltas, grads, codes, int8 codes), layer
    by layer from the input."""
    def act(x):
        s = 127.0 / np.maximum(np.abs(x).max(axis=-1, keepdims=True), 1e-5)
        r = np.clip(np.round(x * s), -128, 127)
        return r / s, r

    def wq(w):
        s = 1.0 / max(float(np.mean(np.abs(w))), 1e-5)
        r = np.clip(np.round(w * s), -1, 1)
        return r / s, r

    Qs, codes = zip(*(wq(w) for w in W))
    acts, ints = [], []
    h = x0
    for Q in Qs:
        a, r = act(h)
        acts.append(a)
        ints.append(r)
        h = a @ Q.T
    delta = h - target
    loss = 0.5 * float(np.sum(delta * delta))
    deltas, grads = [None] * 3, [None] * 3
    for i in (2, 1, 0):
        deltas[i] = delta
        grads[i] = delta.T @ acts[i]
        delta = delta @ Qs[i]
    return loss, deltas, grads, codes, ints


def test_worked_example_matches_page_listing():
    """The oracle-built 3-layer net against the page's own arithmetic: its
    quantisers (reciprocal weight scale, -128 clip) give the same codes, and
    the loss, every delta and every grad_Q agree to 1e-12 relative."""
    rs = np.random.RandomState(0)
    W = [rs.randn(6, 7), rs.randn(5, 6), rs.randn(4, 5)]
    x0 = rs.randn(2, 7)
    target = rs.randn(2, 4)
    p_loss, p_deltas, p_grads, p_codes, p_ints = _page_listing_net(W, x0, target)

    h = x0
    saved = []
    for i, w in enumerate(W):
        codes, gamma = ref.ternarize(w, np.float64)
        q, sx = ref.quantize_activations(h, np.float64)
        np.testing.assert_array_equal(codes, p_codes[i])
        np.testing.assert_array_equal(q, p_ints[i])
        saved.append((codes, gamma, ref.dequantize_activations(q, sx, np.float64)))
        h = ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma, np.float64)
    delta = h - target
    assert math.isclose(0.5 * float(np.sum(delta * delta)), p_loss, rel_tol=1e-12)
    for i in (2, 1, 0):
        codes, gamma, xh = saved[i]
        np.testing.assert_allclose(delta, p_deltas[i], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(ref.backward_dw(delta, xh), p_grads[i], rtol=1e-12, atol=1e-14)
        delta = ref.backward_dx(delta, codes, gamma)


def test_dw_accumulation_hand_derived():
    """bitlinear_step with dw_prev: dW = dw_prev + dY^T x_hat on the dyadic
    fixture, sums written out by hand (every term exact)."""
    g = _load_dyadic()
    x_bits = ref.round_to_bf16_bits(np.array(g["x"], np.float32))
    dy_bits = ref.round_to_bf16_bits(np.array(g["dY"], np.float32))
    prev = np.array([[0.25, 3.0, -4.5, -0.5, 1.0, 2.0, -5.0, 0.125],
                     [-11.875, -246.0, 0.75, 0.0, -0.125, 1.5, 0.5, -1.0]], np.float32)
    out = ref.bitlinear_step(x_bits, np.array(g["W"], np.float32), dy_bits, w_is_bf16=False, dw_prev=prev)
    expected = np.array([[34.0, -140.0, 0.0, 0.0, 1.25, 2.0, 0.0, 0.125],
                         [0.0, 0.0, -7.0, 0.25, 0.0, 1.5, 3.0, -1.0]])
    np.testing.assert_array_equal(out["dw_f64"], expected)
    np.testing.assert_array_equal(out["dw_f32"], expected.astype(np.float32))
    without = ref.bitlinear_step(x_bits, np.array(g["W"], np.float32), dy_bits, w_is_bf16=False)
    np.testing.assert_array_equal(without["dw_f64"], np.array(g["dW"]))


def test_dw_accumulation_loop():
    """dW[n, k] = dw_prev[n, k] + sum_m dY[m, n] x_hat[m, k], element by element."""
    rng = np.random.default_rng(12)
    M, K, N = 6, 32, 5
    x_bits = ref.round_to_bf16_bits(rng.standard_normal((M, K)))
    dy_bits = ref.round_to_bf16_bits(rng.standard_normal((M, N)))
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    prev = rng.standard_normal((N, K)).astype(np.float32)
    out = ref.bitlinear_step(x_bits, w, dy_bits, w_is_bf16=False, dw_prev=prev)
    dy = ref.bf16_bits_to_f32(dy_bits)
    xh = out["x_hat"]
    for n in range(N):
        for k in range(K):
            s = math.fsum([float(prev[n, k])] + [float(dy[m, n]) * float(xh[m, k]) for m in range(M)])
            assert math.isclose(out["dw_f64"][n, k], s, rel_tol=1e-12, abs_tol=1e-12)


# --------------------------------------------------------------------------
# the whole step with the product's roundings
# --------------------------------------------------------------------------


def test_bitlinear_step_shapes_and_saved_state():
    from workloads import make_inputs
    x, w, dy = make_inputs(32, 128, 256, w_dtype=torch.float32, w_init="normal0.02", seed=0)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    dyb = dy.view(torch.int16).numpy().view(np.uint16)
    out = ref.bitlinear_step(xb, w.numpy(), dyb, w_is_bf16=False)
    assert out["packed"].shape == (256, 32) and out["q"].shape == (32, 128)
    np.testing.assert_array_equal(ref.unpack_ternary(out["packed"], 128), out["codes"])
    assert out["y_bits"].shape == (32, 256) and out["dx_bits"].shape == (32, 128)
    assert out["dw_bits"].shape == (256, 128)
    # x_hat carries exactly the bf16 rounding of q * s_x
    xh32 = ref.dequantize_activations(out["q"], out["sx"])
    np.testing.assert_array_equal(out["x_hat"], ref.bf16_bits_to_f32(_torch_bf16_bits(xh32)))
