"""The Python binding refuses CPU tensors: there is no CPU or PyTorch fallback
on the product path, every call fails loudly before reaching the library."""

import pytest
import torch

import ternary_weight_quantization_b200 as bl
from ternary_weight_quantization_b200 import bitlinear as b

M, K, N = 4, 64, 16
bf = lambda *s: torch.zeros(s, dtype=torch.bfloat16)   # noqa: E731
f32 = lambda *s: torch.zeros(s, dtype=torch.float32)   # noqa: E731
u8 = lambda *s: torch.zeros(s, dtype=torch.uint8)      # noqa: E731
i8 = lambda *s: torch.zeros(s, dtype=torch.int8)       # noqa: E731
i32 = lambda *s: torch.zeros(s, dtype=torch.int32)     # noqa: E731

CALLS = {
    "bl_quantize_weight": lambda: bl.bl_quantize_weight(bf(N, K), u8(N, K // 4), f32(1), u8(64)),
    "bl_quantize_act": lambda: bl.bl_quantize_act(bf(M, K), i8(M, K), f32(M)),
    "bl_quantize": lambda: bl.bl_quantize(bf(N, K), bf(M, K), u8(N, K // 4), f32(1), i8(M, K), f32(M), u8(64)),
    "bl_forward": lambda: bl.bl_forward(i8(M, K), f32(M), u8(N, K // 4), f32(1), bf(M, N)),
    "bl_backward": lambda: bl.bl_backward(bf(M, N), i8(M, K), f32(M), u8(N, K // 4), f32(1), bf(M, K), bf(N, K)),
    "bl_sign_pack": lambda: bl.bl_sign_pack(bf(N, K), i32(N, K // 32)),
    "bl_sign_vote": lambda: bl.bl_sign_vote(i32(2, N, K // 32), u8(N, K // 4)),
    "bl_signsgd_update": lambda: bl.bl_signsgd_update(f32(N, K), u8(N, K // 4), 0.1),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_cpu_tensors_are_refused(name):
    with pytest.raises(ValueError, match="CUDA tensor"):
        CALLS[name]()


def test_wrong_dtypes_are_refused_before_the_device_check():
    with pytest.raises(ValueError):
        b.bl_sign_pack(torch.zeros((N, K), dtype=torch.float16), i32(N, K // 32))
    with pytest.raises(ValueError):
        b.bl_signsgd_update(torch.zeros((N, K), dtype=torch.float16), u8(N, K // 4), 0.1)
