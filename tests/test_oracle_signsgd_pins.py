"""Pins of the sign-gradient oracle (oracle/signsgd_ref.py).

Each test fixes a fact the pages or mathematics decide, by a route other than
the oracle's own formula: a hand-written bit pattern, an element-by-element
loop with math.copysign, brute-force vote counts with Python integers, and
closed forms of the fp32 / bf16 update. No GPU needed.
"""

import math

import numpy as np
import pytest

from oracle import bitlinear_ref as ref
from oracle import signsgd_ref as sg


def test_sign_bits_hand_written_pattern():
    # negatives at flattened positions 1, 3 (-0.0), 4 (a subnormal), 31, 32, 63
    d = np.zeros((1, 64), dtype=np.float32)
    d[0, 0] = 1.0
    d[0, 1] = -2.5
    d[0, 2] = 0.0
    d[0, 3] = -0.0
    d[0, 4] = -1e-45
    d[0, 5] = 1e-45
    d[0, 31] = -3.0e38
    d[0, 32] = -1.0
    d[0, 63] = -7.0
    words = sg.sign_bits(d)
    assert words.dtype == np.uint32 and words.shape == (1, 2)
    assert int(words[0, 0]) == 0x8000001A
    assert int(words[0, 1]) == 0x80000001


def test_sign_bits_elementwise_loop():
    rng = np.random.default_rng(3)
    d = rng.standard_normal((5, 96)).astype(np.float32)
    d[rng.random(d.shape) < 0.1] = 0.0
    d[rng.random(d.shape) < 0.05] = -0.0
    words = sg.sign_bits(d)
    for n in range(d.shape[0]):
        for w in range(d.shape[1] // 32):
            expect = 0
            for j in range(32):
                if math.copysign(1.0, float(d[n, 32 * w + j])) < 0:
                    expect |= 1 << j
            assert int(words[n, w]) == expect
    assert np.array_equal(sg.unpack_sign_bits(words), np.array(
        [[math.copysign(1.0, float(v)) < 0 for v in row] for row in d]))


def _brute_vote(words_by_rank, n, k):
    out = np.zeros((n, k), dtype=np.int8)
    for i in range(n):
        for e in range(k):
            neg = sum((int(w[i, e // 32]) >> (e % 32)) & 1 for w in words_by_rank)
            pos = len(words_by_rank) - neg
            out[i, e] = 1 if pos > neg else (-1 if neg > pos else 0)
    return out


@pytest.mark.parametrize("ranks", [1, 2, 3, 4, 5, 8])
def test_majority_direction_brute_force(ranks):
    rng = np.random.default_rng(10 + ranks)
    n, k = 3, 64
    words = [rng.integers(0, 2 ** 32, size=(n, k // 32), dtype=np.uint64).astype(np.uint32) for _ in range(ranks)]
    got = sg.majority_direction(words)
    assert np.array_equal(got, _brute_vote(words, n, k))
    if ranks % 2 == 1:
        assert not np.any(got == 0)  # an odd number of votes never ties


def test_majority_direction_special_cases():
    a = np.array([[0x0000FFFF]], dtype=np.uint32)
    b = np.array([[0xFFFF0000]], dtype=np.uint32)
    # one rank: +1 where the sign bit is clear, -1 where it is set
    one = sg.majority_direction([a])[0]
    assert np.array_equal(one, np.array([-1] * 16 + [1] * 16, dtype=np.int8))
    # two ranks with opposite bits everywhere: all ties
    assert np.array_equal(sg.majority_direction([a, b])[0], np.zeros(32, dtype=np.int8))
    # three ranks, two of them negative at bit 0 only
    c = np.array([[1]], dtype=np.uint32)
    z = np.array([[0]], dtype=np.uint32)
    three = sg.majority_direction([c, c, z])[0]
    assert three[0] == -1 and np.all(three[1:] == 1)


def test_vote_of_agreeing_ranks_is_the_gradient_sign():
    # ranks whose gradients all share one sign pattern vote for exactly that
    # pattern: direction = sign(sum of the ranks' gradients) where nonzero
    rng = np.random.default_rng(5)
    base = rng.standard_normal((4, 64)).astype(np.float32)
    grads = [base * np.float32(s) for s in (0.5, 1.0, 3.0)]
    d = sg.majority_direction([sg.sign_bits(g) for g in grads])
    assert np.array_equal(d, np.sign(np.sum(grads, axis=0)).astype(np.int8))


def test_direction_packs_in_the_ternary_format():
    rng = np.random.default_rng(6)
    words = [rng.integers(0, 2 ** 32, size=(2, 4), dtype=np.uint64).astype(np.uint32) for _ in range(4)]
    d = sg.majority_direction(words)
    assert np.array_equal(ref.unpack_ternary(ref.pack_ternary(d), d.shape[1]), d)


def test_signsgd_update_closed_forms_f32():
    w = np.array([1.0, -0.0, 0.75, 1.0, -3.0], dtype=np.float32)
    d = np.array([0, 0, 1, 1, -1], dtype=np.int8)
    out = sg.signsgd_update(w, d, 0.25, w_is_bf16=False)
    assert out.view(np.uint32).tolist() == np.array([1.0, -0.0, 0.5, 0.75, -2.75], dtype=np.float32).view(np.uint32).tolist()
    # 1 - 2^-30 is not an fp32 value next to 1: it rounds back to 1
    assert sg.signsgd_update(np.array([1.0], np.float32), np.array([1], np.int8), 2.0 ** -30, False)[0] == 1.0
    # d = 0 leaves every value bit for bit, whatever lr
    r = np.random.default_rng(7).standard_normal(64).astype(np.float32)
    assert np.array_equal(sg.signsgd_update(r, np.zeros(64, np.int8), 123.0, False).view(np.uint32), r.view(np.uint32))
    # ... also with a negative lr, on -0
    mz = np.array([-0.0], dtype=np.float32)
    assert sg.signsgd_update(mz, np.array([0], np.int8), -1.0, False).view(np.uint32)[0] == 0x80000000


def test_signsgd_update_bf16_second_rounding():
    one = np.array([1.0], dtype=np.float32)
    # 1 - 2^-9 is exact in fp32 and halfway between the bf16 values 1 - 2^-8
    # (0x3F7F, odd) and 1.0 (0x3F80, even): ties to even keep 1.0
    out = sg.signsgd_update(one, np.array([1], np.int8), 2.0 ** -9, w_is_bf16=True)
    assert int(ref.round_to_bf16_bits(out)[0]) == 0x3F80
    out = sg.signsgd_update(one, np.array([1], np.int8), 2.0 ** -8, w_is_bf16=True)
    assert int(ref.round_to_bf16_bits(out)[0]) == 0x3F7F
    out = sg.signsgd_update(one, np.array([-1], np.int8), 2.0 ** -7, w_is_bf16=True)
    assert int(ref.round_to_bf16_bits(out)[0]) == 0x3F81  # 1 + 2^-7 exact in bf16
