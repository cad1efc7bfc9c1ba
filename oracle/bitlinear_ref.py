"""Plain CPU oracle of the BitNet b1.58 BitLinear training hot path.

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``. The CUDA library shares no code,
table or constant generator with this file, and neither imports the other.

What it computes, step by step, in the order the pages give it:

  S1  absmean ternarisation of the master weights and 2-bit packing
      ("1BitTraining.md", quantisation helpers: ``weight_quant``;
       "bitlinear.py", ``ternary_quantize``; "bitnet-qat-train", first bullet
       under the recipe: one fused ternarise + scale + pack pass)
  S2  per-token absmax INT8 activation quantisation
      ("1BitTraining.md", ``activation_quant``; "bitlinear.py",
       ``activation_quant_int8``)
  S3  forward  y = quant(x) . ternarize(W)^T . s_x . gamma, INT32-exact
      ("bitnet-qat-train", Semantics)
  S4  straight-through backward  dX = dY . W_hat,  dW = dY^T . x_hat, with
      W_hat and x_hat rebuilt from the saved 2-bit / INT8 state and gamma held
      constant ("bitnet-qat-train", Semantics; "1BitTraining.md", "Why this
      always holds": the quantiser's local Jacobian is taken as 1)

Readings where the pages leave a step open (each one is exercised by a pin in
the test suite):
  * weight scale: gamma = max(fp32(mean|W|), 1e-5), the clamp form of
    ``weight_quant``; mean|W| is the exactly rounded fp64 sum (``math.fsum``)
    divided by N*K in fp64, then rounded to fp32.
  * codes: rint_half_even(fp32(W / gamma)) clipped to [-1, 1], IEEE fp32
    division as in ``ternary_quantize``.
  * activations: a = max(max_k |x|, 1e-5), inv = fp32(127 / a),
    q = clip(rint_half_even(fp32(x * inv)), -127, 127), s_x = fp32(a / 127):
    the reciprocal form of ``activation_quant`` with the +-127 clip of
    ``activation_quant_int8``.
  * packing (no page gives the bit layout): element k of row n lives in byte
    n*K/4 + k/4 at bits 2*(k%4) .. 2*(k%4)+1, as a 2-bit two's-complement
    field (00 = 0, 01 = +1, 11 = -1; 10 never written).
  * forward epilogue: y = bf16_rn(fp32(acc) * fp32(s_x * gamma)).
  * x_hat = bf16_rn(fp32(q) * s_x); W_hat = code (exact in bf16) with gamma
    applied to dX after the sum.
  * dX and dW are summed in fp64 and rounded once to the output type.

Pinning: tests/test_oracle_pins.py checks every function here against values
and identities fixed by the pages or by mathematics (hand-derived dyadic
fixtures under tests/golden/, closed-form code statistics, brute-force integer
dot products, the adjoint identity of the linear map, the fake-quant
formulation of "bitlinear.py", and the sign-equality claim of
"1BitTraining.md").
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "EPS_W", "EPS_X", "QB",
    "bf16_bits_to_f32", "round_to_bf16_bits",
    "absmean_gamma", "ternarize", "pack_ternary", "unpack_ternary",
    "quantize_activations", "dequantize_activations",
    "forward_accumulate", "forward_output",
    "backward_dx", "backward_dw", "bitlinear_step",
]

# Clamp floors of the two scales ("1BitTraining.md", quantisation helpers).
EPS_W = np.float32(1e-5)
EPS_X = np.float32(1e-5)
# INT8 code range +-Q_b ("bitlinear.py", activation_quant_int8).
QB = 127


# --------------------------------------------------------------------------
# bf16 <-> float helpers (numpy has no bf16 type; bf16 is carried as uint16)
# --------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> the float32 values they denote (exact)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to bf16 (round to nearest, ties to even).

    Rounds once, directly from the input precision: each finite value is
    scaled by the power of two that puts bf16's last kept bit (8 significant
    bits; quantum 2^-133 below the normal range) at the units place, rounded
    half-to-even with ``np.rint``, scaled back and reinterpreted. Values whose
    rounded magnitude reaches 2^128 become +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.float64)
    finite = np.isfinite(x)
    xf = x[finite]
    mant, expo = np.frexp(xf)               # xf = mant * 2**expo, 0.5 <= |mant| < 1
    expo = np.where(xf == 0, 0, expo)
    q_exp = np.maximum(expo - 8, -133)      # exponent of the last kept bit
    r = np.ldexp(np.rint(np.ldexp(xf, -q_exp)), q_exp)
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, r), r)
    out[finite] = r
    out[~finite] = x[~finite]
    f32 = out.astype(np.float32)            # exact: every r is a bf16 value
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# S1: absmean ternarisation + 2-bit packing
# --------------------------------------------------------------------------

def absmean_gamma(w: np.ndarray, dtype=np.float32):
    """gamma = max(mean|W|, eps), per tensor.

    "1BitTraining.md" (``weight_quant``) scales by 1 / max(mean|w|, 1e-5);
    "bitlinear.py" (``ternary_quantize``) names mean(|w|) the absmean scale.
    The sum of |w| is taken exactly and rounded once to fp64 (``math.fsum``),
    divided by the element count in fp64 and rounded to ``dtype``.
    """
    a = np.abs(np.asarray(w, dtype=np.float64)).ravel()
    total = math.fsum(a.tolist()) if a.size else 0.0
    mean = total / float(a.size) if a.size else 0.0
    gamma = np.asarray(mean, dtype=np.float64).astype(dtype)
    return np.maximum(gamma, np.asarray(EPS_W, dtype=dtype))


def ternarize(w: np.ndarray, dtype=np.float32):
    """RoundClip(W / gamma, -1, 1) -> (codes int8 [N, K], gamma).

    "bitlinear.py", ``ternary_quantize``: w_q = clamp(round(w / scale), -1, 1).
    The division is IEEE in ``dtype`` and rounding is half-to-even (np.rint).
    """
    w = np.asarray(w).astype(dtype)
    gamma = absmean_gamma(w, dtype)
    scaled = (w / gamma).astype(dtype)
    codes = np.clip(np.rint(scaled), -1, 1).astype(np.int8)
    return codes, gamma


def pack_ternary(codes: np.ndarray) -> np.ndarray:
    """Pack ternary codes [N, K] (K % 4 == 0) into bytes [N, K/4].

    Element k of a row goes to byte k // 4 at bits 2*(k % 4); the field is the
    low two bits of the code's two's-complement form (0 -> 00, +1 -> 01,
    -1 -> 11). "bitnet-qat-train" states four codes per byte but no bit order.
    """
    c = np.asarray(codes, dtype=np.int8)
    n, k = c.shape
    assert k % 4 == 0
    fields = (c.astype(np.int16) & 3).astype(np.uint8).reshape(n, k // 4, 4)
    out = np.zeros((n, k // 4), dtype=np.uint8)
    for j in range(4):
        out |= (fields[:, :, j] << np.uint8(2 * j)).astype(np.uint8)
    return out


def unpack_ternary(packed: np.ndarray, k: int) -> np.ndarray:
    """Inverse of :func:`pack_ternary`; raises on the unused field 10."""
    p = np.asarray(packed, dtype=np.uint8)
    n = p.shape[0]
    assert p.shape[1] * 4 == k
    out = np.empty((n, k), dtype=np.int8)
    for j in range(4):
        f = (p >> np.uint8(2 * j)) & np.uint8(3)
        if np.any(f == 2):
            raise ValueError("packed ternary field 10 is not a valid code")
        out[:, j::4] = np.where(f == 3, -1, f.astype(np.int8))
    return out


# --------------------------------------------------------------------------
# S2: per-token absmax INT8 activation quantisation
# --------------------------------------------------------------------------

def quantize_activations(x: np.ndarray, dtype=np.float32):
    """Per-token absmax quantisation -> (q int8 [M, K], s_x [M]).

    "1BitTraining.md", ``activation_quant``: scale = 127 / max(max|x|, 1e-5)
    along the last axis, then round(x * scale); "bitlinear.py",
    ``activation_quant_int8``: clip to [-127, 127]. s_x = a / 127 is the
    dequantisation multiplier (x_hat = q * s_x).
    """
    x = np.asarray(x).astype(dtype)
    a = np.max(np.abs(x), axis=-1) if x.shape[-1] else np.zeros(x.shape[:-1], dtype)
    a = np.maximum(a.astype(dtype), np.asarray(EPS_X, dtype=dtype))
    inv = (np.asarray(QB, dtype=dtype) / a).astype(dtype)
    y = (x * inv[..., None]).astype(dtype)
    q = np.clip(np.rint(y), -QB, QB).astype(np.int8)
    sx = (a / np.asarray(QB, dtype=dtype)).astype(dtype)
    return q, sx


def dequantize_activations(q: np.ndarray, sx: np.ndarray, dtype=np.float32):
    """x_hat = q * s_x in ``dtype`` (the operand the dW contraction uses).

    "bitnet-qat-train", Semantics: x_hat is rebuilt from the saved INT8 state.
    For the bf16 product path the caller rounds the fp32 result to bf16.
    """
    return (np.asarray(q).astype(dtype) * np.asarray(sx, dtype=dtype)[:, None]).astype(dtype)


# --------------------------------------------------------------------------
# S3: forward
# --------------------------------------------------------------------------

def forward_accumulate(q: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k q[m, k] * c[n, k], exact ("bitnet-qat-train", Semantics).

    The product runs as an fp64 matmul: every operand and every partial sum is
    an integer of magnitude at most 127 * K < 2^53, so each fp64 operation is
    exact whatever order the library uses, and the result is the exact
    integer dot product. The result must fit INT32 (checked).
    """
    acc = np.asarray(q, dtype=np.float64) @ np.asarray(codes, dtype=np.float64).T
    acc = acc.astype(np.int64)
    if acc.size:
        assert np.abs(acc).max() < 2 ** 31, "accumulator exceeds INT32"
    return acc


def forward_output(acc: np.ndarray, sx: np.ndarray, gamma, dtype=np.float32) -> np.ndarray:
    """y[m, n] = acc[m, n] * (s_x[m] * gamma), each product rounded in ``dtype``."""
    scale = (np.asarray(sx, dtype=dtype) * np.asarray(gamma, dtype=dtype)).astype(dtype)
    return (np.asarray(acc).astype(dtype) * scale[:, None]).astype(dtype)


# --------------------------------------------------------------------------
# S4: straight-through backward
# --------------------------------------------------------------------------

def backward_dx(dy: np.ndarray, codes: np.ndarray, gamma) -> np.ndarray:
    """dX = dY . W_hat with W_hat = gamma * c, summed in fp64 (unrounded)."""
    return (np.asarray(dy, dtype=np.float64) @ np.asarray(codes, dtype=np.float64)) * float(gamma)


def backward_dw(dy: np.ndarray, x_hat: np.ndarray) -> np.ndarray:
    """dW = dY^T . x_hat, summed in fp64 (unrounded)."""
    return np.asarray(dy, dtype=np.float64).T @ np.asarray(x_hat, dtype=np.float64)


# --------------------------------------------------------------------------
# One whole fwd+bwd pass with the product path's roundings
# --------------------------------------------------------------------------

def bitlinear_step(x_bits, w, dy_bits, w_is_bf16: bool, dw_prev=None):
    """One BitLinear forward + backward, rounded the way the product stores it.

    x_bits, dy_bits: bf16 bit patterns (uint16) [M, K] and [M, N].
    w: master weights [N, K], as bf16 bits (``w_is_bf16``) or float32 values.
    dw_prev: optional previous dW (float32 values) that dW accumulates into.
    Returns a dict of every saved and produced tensor.
    """
    x = bf16_bits_to_f32(x_bits)
    dy = bf16_bits_to_f32(dy_bits)
    wf = bf16_bits_to_f32(w) if w_is_bf16 else np.asarray(w, dtype=np.float32)
    codes, gamma = ternarize(wf)
    q, sx = quantize_activations(x)
    acc = forward_accumulate(q, codes)
    y = forward_output(acc, sx, gamma)
    x_hat = bf16_bits_to_f32(round_to_bf16_bits(dequantize_activations(q, sx)))
    dx = backward_dx(dy, codes, gamma)
    dw = backward_dw(dy, x_hat)
    if dw_prev is not None:
        dw = dw + np.asarray(dw_prev, dtype=np.float64)
    return {
        "gamma": gamma, "codes": codes, "packed": pack_ternary(codes),
        "q": q, "sx": sx, "acc": acc,
        "y_bits": round_to_bf16_bits(y),
        "x_hat": x_hat,
        "dx_bits": round_to_bf16_bits(dx),
        "dw_f64": dw,
        "dw_bits": round_to_bf16_bits(dw),
        "dw_f32": dw.astype(np.float32),
    }
