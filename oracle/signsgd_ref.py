"""Plain CPU oracle of the master-free sign-gradient update (data parallel).

TEST INFRASTRUCTURE ONLY: imported by the tests and by the CPU-baseline leg
of ``bench.py``. The CUDA library shares no code with this file, and neither
imports the other.

What it computes, in the order of "1BitTraining.md", "Why this always holds"
(the closing paragraph on implications): since the straight-through
gradient and the gradient with respect to the quantised weight have the same
sign, a sign-based optimiser needs only the 2-bit weights on the device and
one bit of gradient per weight, sent to one place that accumulates them.

  G1  sign_bits         the 1-bit gradient of every weight, packed 32 to a word
  G2  majority_direction  the per-weight vote over the data-parallel ranks
  G3  signsgd_update    W <- W - lr * direction at the place that holds W,
                        after which S1 (``bitlinear_ref.ternarize``) makes the
                        next step's codes

Readings where the pages leave a step open:
  * the 1-bit gradient is the IEEE sign bit of dW (1 = negative; -0 counts as
    negative, +0 as positive), packed LSB-first: element 32*w + j of the
    flattened [N, K] tensor is bit j of word w.
  * the accumulation of R ranks' bits is a majority vote: direction +1 where
    more ranks saw a positive (sign bit 0) gradient, -1 where more saw a
    negative one, 0 on a tie (even R only).
  * the direction is stored in the 2-bit ternary packing of the weights
    (``bitlinear_ref.pack_ternary``).
  * the update runs in fp32 and is stored in the master dtype:
    W' = dtype_rn(fp32(fp32(W) - lr * d)); with d in {-1, 0, +1} the product
    lr * d is exact, so fp32 rounds once and bf16 masters round once more.
    Where d = 0 the step is +0: the weight is left bit for bit.

Pinning: tests/test_oracle_signsgd_pins.py checks these against a
hand-written bit pattern, an element-by-element math.copysign loop,
brute-force vote counts with Python integers and closed forms of the fp32
and bf16 update.
"""

from __future__ import annotations

import numpy as np

__all__ = ["sign_bits", "unpack_sign_bits", "majority_direction", "signsgd_update"]


def sign_bits(dw: np.ndarray) -> np.ndarray:
    """dW [N, K] (float32 values; K % 32 == 0) -> uint32 words [N, K/32].

    Bit j of word (n, w) is the sign bit of dW[n, 32 w + j].
    """
    d = np.asarray(dw, dtype=np.float32)
    n, k = d.shape
    assert k % 32 == 0
    neg = np.signbit(d).reshape(n, k // 32, 32).astype(np.uint64)
    weights = np.left_shift(np.uint64(1), np.arange(32, dtype=np.uint64))
    return (neg * weights).sum(axis=-1).astype(np.uint32)


def unpack_sign_bits(words: np.ndarray) -> np.ndarray:
    """Inverse of :func:`sign_bits` on the bits: [N, K/32] -> bool [N, K] (True = negative)."""
    w = np.asarray(words, dtype=np.uint32)
    n, kw = w.shape
    bits = (w[:, :, None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
    return bits.reshape(n, kw * 32).astype(bool)


def majority_direction(words_by_rank) -> np.ndarray:
    """R ranks' sign words (each [N, K/32]) -> direction codes int8 [N, K].

    Per weight: +1 if the positive votes outnumber the negative ones, -1 if
    the negative ones do, 0 on a tie.
    """
    ranks = [unpack_sign_bits(w) for w in words_by_rank]
    assert ranks, "at least one rank"
    neg = np.sum(np.stack(ranks).astype(np.int64), axis=0)
    pos = len(ranks) - neg
    return np.sign(pos - neg).astype(np.int8)


def signsgd_update(w: np.ndarray, direction: np.ndarray, lr, w_is_bf16: bool) -> np.ndarray:
    """W' = dtype_rn(fp32(W - lr * d)).

    w: float32 values of the masters (bf16 masters as their exact fp32 values).
    Returns float32 values; for bf16 masters the caller turns them into bf16
    bits with ``bitlinear_ref.round_to_bf16_bits`` (the second rounding).
    """
    wf = np.asarray(w, dtype=np.float32)
    d = np.asarray(direction)
    # lr * d is exact for d = +-1; where d = 0 the step is +0, so W is left
    # bit for bit (also -0, and whatever the sign of lr)
    step = np.where(d == 0, np.float32(0.0), np.float32(lr) * d.astype(np.float32)).astype(np.float32)
    return (wf - step).astype(np.float32)
