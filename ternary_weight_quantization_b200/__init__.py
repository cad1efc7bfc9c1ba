"""B200 (sm_100a) BitNet b1.58 BitLinear training hot path.

The computation lives in the CUDA library libbitlinear.so (C ABI declared in
include/bitlinear.h); ``bitlinear`` is its thin Python binding.
"""

from .bitlinear import (  # noqa: F401
    BL_BF16, BL_F32, BitLinearError, StepBuffers, bitlinear_step, bl_backward, bl_backward_signs, bl_backward_workspace_size, bl_export_weights,
    bl_forward, bl_get_last_error, bl_quantize, bl_quantize_act, bl_quantize_weight, bl_quantize_weight_workspace_size,
    bl_reset_error, bl_sign_pack, bl_sign_vote, bl_signsgd_apply, bl_signsgd_update, bl_version, load_library,
)
