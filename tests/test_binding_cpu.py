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


class _FakeCuda:
    """Stands in for a CUDA tensor on a machine without one: the binding's
    checks read only these attributes before calling the library."""

    def __init__(self, shape, dtype, index):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", index)
        self.is_cuda = True

    def is_contiguous(self):
        return True

    def numel(self):
        return int(torch.tensor(self.shape).prod()) if len(self.shape) else 1

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()

    def data_ptr(self):
        raise AssertionError("the library must not be reached")


def _fake_calls(dev_of):
    """Every entry point with fake CUDA tensors; dev_of(i) gives the device of
    the i-th tensor argument of a call."""
    def t(i, *shape, dtype):
        return _FakeCuda(shape, dtype, dev_of(i))
    bf, u8, i8, f32, i32 = torch.bfloat16, torch.uint8, torch.int8, torch.float32, torch.int32
    return {
        "bl_quantize_weight": lambda: bl.bl_quantize_weight(t(0, N, K, dtype=bf), t(1, N, K // 4, dtype=u8),
                                                            t(2, 1, dtype=f32), t(3, 64, dtype=u8)),
        "bl_quantize_act": lambda: bl.bl_quantize_act(t(0, M, K, dtype=bf), t(1, M, K, dtype=i8), t(2, M, dtype=f32)),
        "bl_quantize": lambda: bl.bl_quantize(t(0, N, K, dtype=bf), t(1, M, K, dtype=bf), t(2, N, K // 4, dtype=u8),
                                              t(3, 1, dtype=f32), t(4, M, K, dtype=i8), t(5, M, dtype=f32),
                                              t(6, 64, dtype=u8)),
        "bl_forward": lambda: bl.bl_forward(t(0, M, K, dtype=i8), t(1, M, dtype=f32), t(2, N, K // 4, dtype=u8),
                                            t(3, 1, dtype=f32), t(4, M, N, dtype=bf)),
        "bl_backward": lambda: bl.bl_backward(t(0, M, N, dtype=bf), t(1, M, K, dtype=i8), t(2, M, dtype=f32),
                                              t(3, N, K // 4, dtype=u8), t(4, 1, dtype=f32), t(5, M, K, dtype=bf),
                                              t(6, N, K, dtype=bf)),
        "bl_sign_pack": lambda: bl.bl_sign_pack(t(0, N, K, dtype=bf), t(1, N, K // 32, dtype=i32)),
        "bl_sign_vote": lambda: bl.bl_sign_vote(t(0, 2, N, K // 32, dtype=i32), t(1, N, K // 4, dtype=u8)),
        "bl_signsgd_update": lambda: bl.bl_signsgd_update(t(0, N, K, dtype=f32), t(1, N, K // 4, dtype=u8), 0.1),
    }


@pytest.mark.parametrize("name", sorted(CALLS))
@pytest.mark.parametrize("odd", [0, 1, "last"])
def test_tensors_of_another_device_are_refused(monkeypatch, name, odd):
    """A tensor on a GPU other than the current one is refused with ValueError
    before the library is called (its kernels would get a foreign pointer)."""
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    n_args = {"bl_quantize_weight": 4, "bl_quantize_act": 3, "bl_quantize": 7, "bl_forward": 5,
              "bl_backward": 7, "bl_sign_pack": 2, "bl_sign_vote": 2, "bl_signsgd_update": 2}[name]
    bad = n_args - 1 if odd == "last" else odd
    with pytest.raises(ValueError, match="current CUDA device"):
        _fake_calls(lambda i: 1 if i == bad else 0)[name]()
