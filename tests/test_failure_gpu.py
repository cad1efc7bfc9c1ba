"""Failure detection on the GPU without a fault: a bounded pipeline wait that
runs out reports BL_ERR_TIMEOUT through the device error word, and the CUDA
context stays usable afterwards (a full parity step still passes)."""

import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    from ternary_weight_quantization_b200 import bitlinear as b
    from tests.test_parity_gpu import check_all, oracle_step, run_step
    from workloads import make_inputs

    lib = b.load_library()
    assert lib.bl_reset_error() == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.bl_selftest_timeout(stream) == 0
    assert lib.bl_get_last_error() == 7          # BL_ERR_TIMEOUT
    assert b"bound" in lib.bl_last_error_message()
    assert lib.bl_reset_error() == 0
    assert lib.bl_get_last_error() == 0
    x, w, dy = make_inputs(64, 256, 128, seed=23)
    check_all(run_step(x, w, dy), oracle_step(x, w, dy), 128)
