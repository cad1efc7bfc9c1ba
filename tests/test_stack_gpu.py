"""A stack of BitLinear layers through the library's calls against the oracle.

Each layer is checked on the inputs it was actually given: its forward on
the bf16 output of the layer below (the stack's x for the first layer), its
backward on the bf16 output gradient the layer above handed it (the stack's
dY for the top layer). With its true inputs every layer meets the single-layer
bars: codes, gamma, INT8 activations, scales and y bit-exact; dX and dW within
max rel 1e-2 and mean rel 1e-3 (rel_i = |g_i - o_i| / max(|o_i|, 1e-3 rms(o))).

The whole chain is also run through the oracle alone (each layer fed the
oracle's own output and gradient): the forward chain stays bit-exact, and the
chained input gradient stays within a normwise ||g - o|| / ||o|| of 1e-2
(there a lower layer's dY can differ from the oracle's by a bf16 rounding
flip of the layer above, so an elementwise bar would measure the chain, not
the layer).

Sizes: two small stacks in full, and the 8-layer 2560 <-> 6912 stack over
2048 tokens ("bitnet-qat-train", Measured behavior, Memory) on sampled tokens
and output rows (the oracle ternarises every full weight).
"""

import numpy as np
import pytest
import torch

from oracle import bitlinear_ref as ref
from workloads import STACKS, stack_inputs

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_REL = 1e-2, 1e-3


def bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def rel_err(gpu, orc):
    g = np.asarray(gpu, np.float64)
    o = np.asarray(orc, np.float64)
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    r = np.abs(g - o) / np.maximum(np.abs(o), 1e-3 * rms + 1e-30)
    norm = float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30))
    return float(r.max(initial=0.0)), float(r.mean()), norm


def assert_gate(gpu, orc, what):
    mx, mean, _ = rel_err(gpu, orc)
    assert mx <= MAX_REL and mean <= MEAN_REL, f"{what}: max rel {mx:.3e}, mean rel {mean:.3e}"


def bf16_vals(b16):
    return ref.bf16_bits_to_f32(b16).astype(np.float64)


def run_stack(M, dims, seed):
    """Runs the stack on the GPU and returns every layer's inputs, saved state
    and outputs as CPU arrays."""
    from ternary_weight_quantization_b200 import bitlinear as b
    from ternary_weight_quantization_b200.stack import BitLinearStack

    b.load_library()
    x, ws, dy = stack_inputs(M, dims, seed=seed)
    st = BitLinearStack.allocate(M, dims)
    ys, dys, dxs = {}, {}, {}
    st.forward(x.cuda(), [w.cuda() for w in ws], on_layer=lambda l, y: ys.__setitem__(l, bits(y)))
    st.backward(dy.cuda(), on_layer=lambda l, g, d: (dys.__setitem__(l, bits(g)), dxs.__setitem__(l, bits(d))))
    st.check()
    layers = []
    for l, L in enumerate(st.layers):
        layers.append({
            "w": ws[l], "x_bits": bits(x) if l == 0 else ys[l - 1], "y_bits": ys[l],
            "packed": L.w_packed.cpu().numpy(), "gamma": np.float32(L.gamma.item()),
            "q": L.xq.cpu().numpy(), "sx": L.sx.cpu().numpy(),
            "dy_bits": dys[l], "dx_bits": dxs[l], "dw": L.dW.float().cpu().numpy(),
        })
    return x, ws, dy, layers


@pytest.mark.parametrize("M,dims", [(40, [64, 96, 64, 128]), (300, [256, 544, 256])])
def test_stack_every_layer_on_its_inputs(M, dims):
    x, ws, dy, layers = run_stack(M, dims, seed=M)
    for l, g in enumerate(layers):
        codes, gamma = ref.ternarize(ref.bf16_bits_to_f32(bits(g["w"])))
        assert g["gamma"].tobytes() == gamma.tobytes(), f"gamma[{l}]"
        np.testing.assert_array_equal(g["packed"], ref.pack_ternary(codes), err_msg=f"codes[{l}]")
        q, sx = ref.quantize_activations(ref.bf16_bits_to_f32(g["x_bits"]))
        np.testing.assert_array_equal(g["q"], q, err_msg=f"xq[{l}]")
        np.testing.assert_array_equal(g["sx"], sx, err_msg=f"sx[{l}]")
        y = ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma)
        np.testing.assert_array_equal(g["y_bits"], ref.round_to_bf16_bits(y), err_msg=f"y[{l}]")
        dyv = bf16_vals(g["dy_bits"])
        xh = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.dequantize_activations(q, sx)))
        dw = bf16_vals(ref.round_to_bf16_bits(ref.backward_dw(dyv, xh)))
        assert_gate(g["dw"], dw, f"dW[{l}]")
        dx = bf16_vals(ref.round_to_bf16_bits(ref.backward_dx(dyv, codes, gamma)))
        assert_gate(bf16_vals(g["dx_bits"]), dx, f"dX[{l}]")
    np.testing.assert_array_equal(layers[-1]["dy_bits"], bits(dy))


@pytest.mark.parametrize("M,dims", [(40, [64, 96, 64, 128]), (300, [256, 544, 256])])
def test_stack_chain_against_oracle_chain(M, dims):
    x, ws, dy, layers = run_stack(M, dims, seed=M)
    h = ref.bf16_bits_to_f32(bits(x))
    saved = []
    for l, w in enumerate(ws):
        codes, gamma = ref.ternarize(ref.bf16_bits_to_f32(bits(w)))
        q, sx = ref.quantize_activations(h)
        y_bits = ref.round_to_bf16_bits(ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma))
        np.testing.assert_array_equal(layers[l]["y_bits"], y_bits, err_msg=f"chained y[{l}]")
        saved.append((codes, gamma))
        h = ref.bf16_bits_to_f32(y_bits)
    g = ref.bf16_bits_to_f32(bits(dy)).astype(np.float64)
    for l in range(len(ws) - 1, -1, -1):
        codes, gamma = saved[l]
        g = bf16_vals(ref.round_to_bf16_bits(ref.backward_dx(g, codes, gamma)))
    _, _, norm = rel_err(bf16_vals(layers[0]["dx_bits"]), g)
    assert norm <= 1e-2, f"chained input gradient: normwise {norm:.3e}"


def test_stack8_full_size_sampled():
    """The 8-layer 2560 <-> 6912 stack over 2048 tokens, every layer on its own
    inputs: gamma and all codes in full, the INT8 activations, y and dX on 48
    sampled tokens, dW on 48 sampled output rows."""
    M, dims = STACKS["stack8"]
    x, ws, dy, layers = run_stack(M, dims, seed=0)
    rng = np.random.default_rng(5)
    ms = np.sort(rng.choice(M, 48, replace=False))
    ms[0], ms[-1] = 0, M - 1
    for l, g in enumerate(layers):
        N, K = dims[l + 1], dims[l]
        ns = np.sort(rng.choice(N, 48, replace=False))
        codes, gamma = ref.ternarize(ref.bf16_bits_to_f32(bits(g["w"])))
        assert g["gamma"].tobytes() == gamma.tobytes(), f"gamma[{l}]"
        np.testing.assert_array_equal(g["packed"], ref.pack_ternary(codes), err_msg=f"codes[{l}]")
        q, sx = ref.quantize_activations(ref.bf16_bits_to_f32(g["x_bits"][ms]))
        np.testing.assert_array_equal(g["q"][ms], q, err_msg=f"xq[{l}]")
        np.testing.assert_array_equal(g["sx"][ms], sx, err_msg=f"sx[{l}]")
        y = ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma)
        np.testing.assert_array_equal(g["y_bits"][ms], ref.round_to_bf16_bits(y), err_msg=f"y[{l}]")
        dyv = bf16_vals(g["dy_bits"])
        dx = bf16_vals(ref.round_to_bf16_bits(ref.backward_dx(dyv[ms], codes, gamma)))
        assert_gate(bf16_vals(g["dx_bits"][ms]), dx, f"dX[{l}]")
        # dW rows from the GPU's saved INT8 state (bit-exact on the sampled tokens above)
        xh = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.dequantize_activations(g["q"], g["sx"])))
        dw = bf16_vals(ref.round_to_bf16_bits(ref.backward_dw(dyv[:, ns], xh)))
        assert_gate(g["dw"][ns], dw, f"dW[{l}]")
