"""The C ABI library loads and exports every symbol include/bitlinear.h
declares; host-side argument validation works without a GPU."""

import ctypes
import os
import re

import pytest

from ternary_weight_quantization_b200 import bitlinear as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bl_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = b.load_library()
    declared = _declared_symbols()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(b.SIGNATURES), "binding signatures drift from the header"


def test_version_and_status_strings():
    lib = b.load_library()
    assert lib.bl_version() >> 16 == 1
    for code, name in b.STATUS.items():
        assert lib.bl_status_string(code).decode() == name


def test_workspace_size():
    # the exact-sum arrival counter (128-byte line), 256 exact-sum bins, a
    # spacer line and one fp64 partial sum per summing CTA (at most 1024): the
    # same for every tensor
    assert b.bl_quantize_weight_workspace_size(0, 32) == 0
    assert b.bl_quantize_weight_workspace_size(256, 128) == 128 + 8 * 256 + 128 + 8 * 1024
    assert b.bl_quantize_weight_workspace_size(6912, 2560) == 128 + 8 * 256 + 128 + 8 * 1024


def test_backward_workspace_size():
    # x_hat as bf16 [M][K] where dW has at least 2048 features; nothing below
    assert b.bl_backward_workspace_size(4096, 6912, 2560) == 4096 * 2560 * 2
    assert b.bl_backward_workspace_size(7, 2048, 96) == 7 * 96 * 2
    assert b.bl_backward_workspace_size(2048, 2560, 6912) == 2048 * 6912 * 2
    assert b.bl_backward_workspace_size(4096, 2040, 2560) == 0
    assert b.bl_backward_workspace_size(0, 6912, 2560) == 0


FAKE = ctypes.c_void_p(0x10000)        # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


@pytest.mark.parametrize("call,expect", [
    (lambda L: L.bl_quantize_act(FAKE, 4, 33, FAKE, FAKE, None), 2),          # K % 32
    (lambda L: L.bl_quantize_act(FAKE, 4, 0, FAKE, FAKE, None), 2),
    (lambda L: L.bl_quantize_act(None, 4, 64, FAKE, FAKE, None), 1),          # null
    (lambda L: L.bl_quantize_act(MISALIGNED, 4, 64, FAKE, FAKE, None), 4),    # alignment
    (lambda L: L.bl_quantize_act(FAKE, -1, 64, FAKE, FAKE, None), 1),
    (lambda L: L.bl_quantize_weight(FAKE, 7, 8, 64, FAKE, FAKE, FAKE, 1 << 20, None), 3),  # dtype
    (lambda L: L.bl_quantize_weight(FAKE, 0, 8, 64, FAKE, FAKE, FAKE, 0, None), 8),        # workspace
    (lambda L: L.bl_quantize_weight(FAKE, 0, 0, 64, FAKE, FAKE, FAKE, 64, None), 1),
    (lambda L: L.bl_forward(FAKE, FAKE, FAKE, FAKE, 4, 8, 48, FAKE, None, None), 2),
    (lambda L: L.bl_forward(FAKE, FAKE, None, FAKE, 4, 8, 64, FAKE, None, None), 1),
    (lambda L: L.bl_forward(FAKE, FAKE, FAKE, FAKE, 4, 8, 64, FAKE, MISALIGNED, None), 4),
    (lambda L: L.bl_backward(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 12, 64, FAKE, FAKE, 0, 0, None), 2),  # N % 8
    (lambda L: L.bl_backward(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 16, 64, FAKE, FAKE, 9, 0, None), 3),
    (lambda L: L.bl_backward(FAKE, FAKE, FAKE, None, FAKE, 4, 16, 64, FAKE, None, 0, 0, None), 1),
    (lambda L: L.bl_backward_ws(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2048, 64, FAKE, FAKE, 0, 0, FAKE, 64, None),
     8),                                                                       # workspace too small
    (lambda L: L.bl_backward_ws(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2048, 64, FAKE, FAKE, 0, 0, MISALIGNED, 1 << 20,
                                None), 8),                                     # workspace misaligned
    (lambda L: L.bl_backward_signs_ws(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2048, 64, FAKE, None, FAKE, 1 << 20, None),
     1),                                                                       # no sign words
    (lambda L: L.bl_export_weights(FAKE, FAKE, 4, 64, None, FAKE, None), 1),
    (lambda L: L.bl_sign_pack(FAKE, 0, 4, 48, FAKE, None), 2),               # K % 32
    (lambda L: L.bl_sign_pack(FAKE, 5, 4, 64, FAKE, None), 3),
    (lambda L: L.bl_sign_pack(FAKE, 0, 4, 64, MISALIGNED, None), 4),
    (lambda L: L.bl_sign_vote(FAKE, 0, 4, 64, FAKE, None), 1),               # ranks
    (lambda L: L.bl_sign_vote(FAKE, 128, 4, 64, FAKE, None), 1),
    (lambda L: L.bl_sign_vote(FAKE, 2, 4, 64, None, None), 1),
    (lambda L: L.bl_signsgd_update(FAKE, 0, 4, 64, FAKE, float("inf"), None), 1),  # lr
    (lambda L: L.bl_signsgd_update(FAKE, 0, 4, 64, FAKE, float("nan"), None), 1),
    (lambda L: L.bl_signsgd_update(FAKE, 2, 4, 64, FAKE, 0.1, None), 3),
    (lambda L: L.bl_signsgd_update(FAKE, 0, 0, 64, FAKE, 0.1, None), 1),
    (lambda L: L.bl_signsgd_apply(FAKE, 0, FAKE, 0, 4, 64, 0.1, FAKE, FAKE, FAKE, 1 << 20, None), 1),  # ranks
    (lambda L: L.bl_signsgd_apply(FAKE, 2, FAKE, 0, 4, 64, float("nan"), FAKE, FAKE, FAKE, 1 << 20, None), 1),
    (lambda L: L.bl_signsgd_apply(FAKE, 2, FAKE, 0, 4, 64, 0.1, FAKE, FAKE, FAKE, 64, None), 8),  # workspace
    (lambda L: L.bl_signsgd_apply(FAKE, 2, FAKE, 0, 4, 48, 0.1, FAKE, FAKE, FAKE, 1 << 20, None), 2),  # K % 32
])
def test_host_validation_without_gpu(call, expect):
    lib = b.load_library()
    assert call(lib) == expect
    assert lib.bl_last_error_message().decode()


def test_empty_work_is_ok_without_gpu():
    lib = b.load_library()
    assert lib.bl_quantize_act(None, 0, 64, None, None, None) == 0
    assert lib.bl_forward(None, None, None, None, 0, 8, 64, None, None, None) == 0
    assert lib.bl_backward(None, None, None, None, None, 4, 16, 64, None, None, 0, 0, None) == 0
