"""bl_quantize_weight_noalloc against bl_quantize_weight.

Some callers cannot allocate device memory (plugin hosts that only pass in
the buffers they own, runtimes with a fixed memory pool), so they cannot hand
bl_quantize_weight its workspace. The no-allocation variant keeps its scratch
in a fixed array inside the library instead. This test calls it through the C
ABI twice in a row, on different weights each time so the second call starts
from the first call's leftover scratch, and checks that both calls give the
same packed codes and gamma as the workspace variant, bit for bit (the
tolerance the parity tests use for codes and gamma).

The file name sorts last so that a run stopping at the first failure has
already run every other test; the test also passes on its own in a fresh
process.
"""

import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("N,K,dtype", [(6912, 2560, torch.bfloat16), (256, 128, torch.float32),
                                       (37, 96, torch.bfloat16), (1000, 544, torch.float32)])
def test_noalloc_matches_workspace_variant(N, K, dtype):
    from ternary_weight_quantization_b200 import bitlinear as b

    lib = b.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    wdt = b.BL_F32 if dtype == torch.float32 else b.BL_BF16
    gen = torch.Generator().manual_seed(N + K)
    ws_bytes = lib.bl_quantize_weight_workspace_size(N, K)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    for call in range(2):
        w = (torch.randn(N, K, generator=gen) * (0.02 if call == 0 else 0.5)).to(dtype).cuda()
        ref_packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
        ref_gamma = torch.empty(1, dtype=torch.float32, device="cuda")
        rc = lib.bl_quantize_weight(_ptr(w), wdt, N, K, _ptr(ref_packed), _ptr(ref_gamma), _ptr(ws), ws_bytes,
                                    stream)
        assert rc == 0, lib.bl_last_error_message()
        packed = torch.full((N, K // 4), 0xAA, dtype=torch.uint8, device="cuda")
        gamma = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        rc = lib.bl_quantize_weight_noalloc(_ptr(w), wdt, N, K, _ptr(packed), _ptr(gamma), stream)
        assert rc == 0, lib.bl_last_error_message()
        torch.cuda.synchronize()
        assert lib.bl_get_last_error() == 0
        assert torch.equal(packed, ref_packed), f"call {call}: packed codes differ"
        assert torch.equal(gamma, ref_gamma), f"call {call}: gamma differs"
