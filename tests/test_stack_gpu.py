"""A stack of BitLinear layers through the library's calls against the oracle
chained the same way: each layer's forward output (bf16) is the next layer's
input, each layer's dX the dY of the layer below, and only the 2-bit / INT8
state is kept between forward and backward.

Bars: the forward chain is bit-exact (every layer's y is). The top layer's dW
has the single-layer bar (max rel 1e-2, mean rel 1e-3). A lower layer's dY is
the bf16 dX of the layer above, which differs from the oracle's own chain by
occasional bf16 rounding flips, and an output whose sum nearly cancels can
then show a large elementwise relative error; those layers (and the input
gradient) are held to mean rel 1e-3 and normwise rel ||g - o|| / ||o|| 1e-2.
"""

import numpy as np
import pytest
import torch

from oracle import bitlinear_ref as ref
from workloads import stack_inputs

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


def oracle_stack(x, ws, dy):
    """Forward and backward of the stack with the oracle's per-layer steps."""
    h = ref.bf16_bits_to_f32(bits(x))
    saved = []
    for w in ws:
        codes, gamma = ref.ternarize(ref.bf16_bits_to_f32(bits(w)))
        q, sx = ref.quantize_activations(h)
        y_bits = ref.round_to_bf16_bits(ref.forward_output(ref.forward_accumulate(q, codes), sx, gamma))
        saved.append((codes, gamma, q, sx))
        h = ref.bf16_bits_to_f32(y_bits)
    out_bits = y_bits
    g = ref.bf16_bits_to_f32(bits(dy))
    dws = [None] * len(ws)
    for l in range(len(ws) - 1, -1, -1):
        codes, gamma, q, sx = saved[l]
        xh = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.dequantize_activations(q, sx)))
        dws[l] = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.backward_dw(g, xh)))
        g = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.backward_dx(g, codes, gamma)))
    return out_bits, dws, g


@pytest.mark.parametrize("M,dims", [(40, [64, 96, 64, 128]), (300, [256, 544, 256])])
def test_stack_parity(M, dims):
    from ternary_weight_quantization_b200 import bitlinear as b
    from ternary_weight_quantization_b200.stack import BitLinearStack

    b.load_library()
    x, ws, dy = stack_inputs(M, dims, seed=M)
    st = BitLinearStack.allocate(M, dims)
    out = st.forward(x.cuda(), [w.cuda() for w in ws])
    out_bits = bits(out)
    dx = st.backward(dy.cuda())
    torch.cuda.synchronize()
    assert b.bl_get_last_error() == 0
    o_out, o_dws, o_dx = oracle_stack(x, ws, dy)
    np.testing.assert_array_equal(out_bits, o_out)          # forward chain bit-exact
    top = len(st.layers) - 1
    for l, L in enumerate(st.layers):
        mx, mean, norm = rel_err(L.dW.float().cpu().numpy(), o_dws[l])
        if l == top:
            assert mx <= MAX_REL and mean <= MEAN_REL, f"dW[{l}]: {mx:.2e} {mean:.2e}"
        else:
            assert mean <= MEAN_REL and norm <= MAX_REL, f"dW[{l}]: {mean:.2e} {norm:.2e}"
    mx, mean, norm = rel_err(dx.float().cpu().numpy(), o_dx)
    assert mean <= MEAN_REL and norm <= MAX_REL, f"dX: {mean:.2e} {norm:.2e}"
