"""Thin Python binding of libbitlinear.so (argument marshalling only).

Each function has the name of the C entry point it calls, takes torch CUDA
tensors, checks dtype / shape / contiguity, passes raw device pointers and
the current CUDA stream, and raises :class:`BitLinearError` on any status
other than BL_OK. Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and importing the library fails
loudly when the shared object is missing.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear.so")

BL_BF16 = 0
BL_F32 = 1

STATUS = {
    0: "BL_OK", 1: "BL_ERR_INVALID_ARG", 2: "BL_ERR_UNSUPPORTED_SHAPE", 3: "BL_ERR_DTYPE",
    4: "BL_ERR_ALIGNMENT", 5: "BL_ERR_ARCH", 6: "BL_ERR_CUDA", 7: "BL_ERR_TIMEOUT", 8: "BL_ERR_WORKSPACE",
}

# (name, restype, argtypes) of every symbol include/bitlinear.h declares
_VP, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "bl_version": (_I32, []),
    "bl_status_string": (ctypes.c_char_p, [_I32]),
    "bl_last_error_message": (ctypes.c_char_p, []),
    "bl_quantize_weight_workspace_size": (_SZ, [_I64, _I64]),
    "bl_quantize_weight": (_I32, [_VP, _I32, _I64, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bl_quantize_weight_noalloc": (_I32, [_VP, _I32, _I64, _I64, _VP, _VP, _VP]),
    "bl_quantize_act": (_I32, [_VP, _I64, _I64, _VP, _VP, _VP]),
    "bl_quantize": (_I32, [_VP, _I32, _I64, _I64, _VP, _I64, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "bl_forward": (_I32, [_VP, _VP, _VP, _VP, _I64, _I64, _I64, _VP, _VP, _VP]),
    "bl_backward": (_I32, [_VP, _VP, _VP, _VP, _VP, _I64, _I64, _I64, _VP, _VP, _I32, _I32, _VP]),
    "bl_backward_signs": (_I32, [_VP, _VP, _VP, _VP, _VP, _I64, _I64, _I64, _VP, _VP, _VP]),
    "bl_backward_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bl_backward_ws": (_I32, [_VP, _VP, _VP, _VP, _VP, _I64, _I64, _I64, _VP, _VP, _I32, _I32, _VP, _SZ, _VP]),
    "bl_backward_signs_ws": (_I32, [_VP, _VP, _VP, _VP, _VP, _I64, _I64, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bl_export_weights": (_I32, [_VP, _VP, _I64, _I64, _VP, _VP, _VP]),
    "bl_get_last_error": (_I32, []),
    "bl_reset_error": (_I32, []),
    "bl_selftest_timeout": (_I32, [_VP]),
    "bl_sign_pack": (_I32, [_VP, _I32, _I64, _I64, _VP, _VP]),
    "bl_sign_vote": (_I32, [_VP, _I32, _I64, _I64, _VP, _VP]),
    "bl_signsgd_update": (_I32, [_VP, _I32, _I64, _I64, _VP, ctypes.c_float, _VP]),
    "bl_signsgd_apply": (_I32, [_VP, _I32, _VP, _I32, _I64, _I64, ctypes.c_float, _VP, _VP, _VP, _SZ, _VP]),
}


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")
        self.status = status


_LIB = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libbitlinear.so and declare its C signatures (raises if absent)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m ternary_weight_quantization_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        lib = load_library()
        detail = lib.bl_last_error_message().decode(errors="replace")
        raise BitLinearError(status, where, detail)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    elif stream.device.index != torch.cuda.current_device():
        raise ValueError(f"stream of {stream.device} but the current CUDA device is cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(stream.cuda_stream)


def _on_current_device(*tensors):
    """Every tensor argument must live on the current CUDA device: the library
    launches on the current device (and the stream passed is that device's),
    so a tensor of another GPU would hand its kernels foreign pointers."""
    cur = torch.cuda.current_device()
    for t in tensors:
        if t is not None and t.device.index != cur:
            raise ValueError(f"tensor on {t.device} but the current CUDA device is cuda:{cur}; "
                             "call under torch.cuda.device(...) of the tensors' device")


def _need(t, dtype, shape, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ----------------------------------------------------------------- entry points

def bl_version() -> int:
    return load_library().bl_version()


def bl_quantize_weight_workspace_size(N: int, K: int) -> int:
    return load_library().bl_quantize_weight_workspace_size(N, K)


def bl_quantize_weight(W, w_packed, gamma, workspace, stream=None):
    """S1: W [N,K] bf16|f32 -> w_packed [N,K/4] uint8, gamma [1] f32."""
    N, K = W.shape
    if W.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("W must be bf16 or f32")
    _need(W, W.dtype, (N, K), "W")
    _need(w_packed, torch.uint8, (N, K // 4), "w_packed")
    _need(gamma, torch.float32, (1,), "gamma")
    _on_current_device(W, w_packed, gamma, workspace)
    wdt = BL_F32 if W.dtype == torch.float32 else BL_BF16
    _check(load_library().bl_quantize_weight(_ptr(W), wdt, N, K, _ptr(w_packed), _ptr(gamma), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _stream(stream)),
           "bl_quantize_weight")


def bl_quantize_act(x, xq, sx, stream=None):
    """S2: x [M,K] bf16 -> xq [M,K] int8, sx [M] f32."""
    M, K = x.shape
    _need(x, torch.bfloat16, (M, K), "x")
    _need(xq, torch.int8, (M, K), "xq")
    _need(sx, torch.float32, (M,), "sx")
    _on_current_device(x, xq, sx)
    _check(load_library().bl_quantize_act(_ptr(x), M, K, _ptr(xq), _ptr(sx), _stream(stream)), "bl_quantize_act")


def bl_quantize(W, x, w_packed, gamma, xq, sx, workspace, stream=None):
    """S1 + S2 in one call (same outputs as bl_quantize_weight then bl_quantize_act)."""
    N, K = W.shape
    M = x.shape[0]
    if W.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("W must be bf16 or f32")
    _need(W, W.dtype, (N, K), "W")
    _need(x, torch.bfloat16, (M, K), "x")
    _need(w_packed, torch.uint8, (N, K // 4), "w_packed")
    _need(gamma, torch.float32, (1,), "gamma")
    _need(xq, torch.int8, (M, K), "xq")
    _need(sx, torch.float32, (M,), "sx")
    _on_current_device(W, x, w_packed, gamma, xq, sx, workspace)
    wdt = BL_F32 if W.dtype == torch.float32 else BL_BF16
    _check(load_library().bl_quantize(_ptr(W), wdt, N, K, _ptr(x), M, _ptr(w_packed), _ptr(gamma), _ptr(xq),
                                      _ptr(sx), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream)),
           "bl_quantize")


def bl_forward(xq, sx, w_packed, gamma, y, debug_acc=None, stream=None):
    """S3: y [M,N] bf16 = xq . codes^T * sx * gamma (debug_acc [M,N] int32 optional)."""
    M, K = xq.shape
    N = w_packed.shape[0]
    _need(xq, torch.int8, (M, K), "xq")
    _need(sx, torch.float32, (M,), "sx")
    _need(w_packed, torch.uint8, (N, K // 4), "w_packed")
    _need(gamma, torch.float32, (1,), "gamma")
    _need(y, torch.bfloat16, (M, N), "y")
    if debug_acc is not None:
        _need(debug_acc, torch.int32, (M, N), "debug_acc")
    _on_current_device(xq, sx, w_packed, gamma, y, debug_acc)
    _check(load_library().bl_forward(_ptr(xq), _ptr(sx), _ptr(w_packed), _ptr(gamma), M, N, K, _ptr(y),
                                     _ptr(debug_acc), _stream(stream)), "bl_forward")


def bl_backward_workspace_size(M: int, N: int, K: int) -> int:
    return load_library().bl_backward_workspace_size(M, N, K)


def bl_backward(dY, xq, sx, w_packed, gamma, dX=None, dW=None, accumulate_dW=False, stream=None, workspace=None):
    """S4: dX [M,K] bf16 = gamma * dY . codes; dW [N,K] (bf16|f32) = dY^T . x_hat.
    workspace (bl_backward_workspace_size bytes): x_hat is made once there
    (bl_backward_ws) instead of rebuilt in every dW tile; same results."""
    M, N = dY.shape
    K = xq.shape[1]
    _need(dY, torch.bfloat16, (M, N), "dY")
    _need(xq, torch.int8, (M, K), "xq")
    _need(sx, torch.float32, (M,), "sx")
    _need(w_packed, torch.uint8, (N, K // 4), "w_packed")
    _need(gamma, torch.float32, (1,), "gamma")
    dwdt = BL_BF16
    if dX is not None:
        _need(dX, torch.bfloat16, (M, K), "dX")
    if dW is not None:
        if dW.dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("dW must be bf16 or f32")
        _need(dW, dW.dtype, (N, K), "dW")
        dwdt = BL_F32 if dW.dtype == torch.float32 else BL_BF16
    _on_current_device(dY, xq, sx, w_packed, gamma, dX, dW, workspace)
    lib = load_library()
    if workspace is None:
        _check(lib.bl_backward(_ptr(dY), _ptr(xq), _ptr(sx), _ptr(w_packed), _ptr(gamma), M, N, K,
                               _ptr(dX), _ptr(dW), dwdt, int(bool(accumulate_dW)), _stream(stream)),
               "bl_backward")
    else:
        _check(lib.bl_backward_ws(_ptr(dY), _ptr(xq), _ptr(sx), _ptr(w_packed), _ptr(gamma), M, N, K,
                                  _ptr(dX), _ptr(dW), dwdt, int(bool(accumulate_dW)), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)),
               "bl_backward_ws")


def bl_backward_signs(dY, xq, sx, w_packed, gamma, dX, dw_sign_words, stream=None, workspace=None):
    """S4 with G1 fused: dX [M,K] bf16 (or None) as bl_backward, and the sign
    words of dW, dw_sign_words [N, K/32] int32 (bit patterns), instead of dW.
    workspace: as bl_backward's."""
    M, N = dY.shape
    K = xq.shape[1]
    _need(dY, torch.bfloat16, (M, N), "dY")
    _need(xq, torch.int8, (M, K), "xq")
    _need(sx, torch.float32, (M,), "sx")
    _need(w_packed, torch.uint8, (N, K // 4), "w_packed")
    _need(gamma, torch.float32, (1,), "gamma")
    if dX is not None:
        _need(dX, torch.bfloat16, (M, K), "dX")
    _need(dw_sign_words, torch.int32, (N, K // 32), "dw_sign_words")
    _on_current_device(dY, xq, sx, w_packed, gamma, dX, dw_sign_words, workspace)
    lib = load_library()
    if workspace is None:
        _check(lib.bl_backward_signs(_ptr(dY), _ptr(xq), _ptr(sx), _ptr(w_packed), _ptr(gamma), M, N, K,
                                     _ptr(dX), _ptr(dw_sign_words), _stream(stream)),
               "bl_backward_signs")
    else:
        _check(lib.bl_backward_signs_ws(_ptr(dY), _ptr(xq), _ptr(sx), _ptr(w_packed), _ptr(gamma), M, N, K,
                                        _ptr(dX), _ptr(dw_sign_words), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream)),
               "bl_backward_signs_ws")


def bl_sign_pack(dW, sign_words, stream=None):
    """G1: sign_words [N, K/32] int32 (bit patterns) <- sign bits of dW [N, K] (bf16|f32)."""
    N, K = dW.shape
    if dW.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("dW must be bf16 or f32")
    _need(dW, dW.dtype, (N, K), "dW")
    _need(sign_words, torch.int32, (N, K // 32), "sign_words")
    _on_current_device(dW, sign_words)
    dt = BL_F32 if dW.dtype == torch.float32 else BL_BF16
    _check(load_library().bl_sign_pack(_ptr(dW), dt, N, K, _ptr(sign_words), _stream(stream)), "bl_sign_pack")


def bl_sign_vote(sign_words, direction, stream=None):
    """G2: direction [N, K/4] uint8 (2-bit packed) <- majority of sign_words [R, N, K/32] int32."""
    R, N, KW = sign_words.shape
    _need(sign_words, torch.int32, (R, N, KW), "sign_words")
    _need(direction, torch.uint8, (N, KW * 8), "direction")
    _on_current_device(sign_words, direction)
    _check(load_library().bl_sign_vote(_ptr(sign_words), R, N, KW * 32, _ptr(direction), _stream(stream)),
           "bl_sign_vote")


def bl_signsgd_update(W, direction, lr, stream=None):
    """G3: W [N, K] (bf16|f32) <- dtype_rn(fp32(W) - lr * direction), in place."""
    N, K = W.shape
    if W.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("W must be bf16 or f32")
    _need(W, W.dtype, (N, K), "W")
    _need(direction, torch.uint8, (N, K // 4), "direction")
    _on_current_device(W, direction)
    dt = BL_F32 if W.dtype == torch.float32 else BL_BF16
    _check(load_library().bl_signsgd_update(_ptr(W), dt, N, K, _ptr(direction), float(lr), _stream(stream)),
           "bl_signsgd_update")


def bl_signsgd_apply(sign_words, W, lr, w_packed, gamma, workspace, stream=None):
    """G2 + G3 + S1 fused on the holder: the majority direction of sign_words
    [R, N, K/32] int32 applied to W [N, K] (bf16|f32) in place, then W's new
    w_packed [N, K/4] uint8 and gamma [1] f32 (two launches)."""
    R, N, KW = sign_words.shape
    K = KW * 32
    if W.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("W must be bf16 or f32")
    _need(sign_words, torch.int32, (R, N, KW), "sign_words")
    _need(W, W.dtype, (N, K), "W")
    _need(w_packed, torch.uint8, (N, K // 4), "w_packed")
    _need(gamma, torch.float32, (1,), "gamma")
    _on_current_device(sign_words, W, w_packed, gamma, workspace)
    dt = BL_F32 if W.dtype == torch.float32 else BL_BF16
    _check(load_library().bl_signsgd_apply(_ptr(sign_words), R, _ptr(W), dt, N, K, float(lr), _ptr(w_packed),
                                           _ptr(gamma), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _stream(stream)),
           "bl_signsgd_apply")


def bl_export_weights(w_packed, gamma, stream=None):
    """Copy (w_packed, gamma) to host: returns (uint8 [N,K/4] CPU tensor, float gamma)."""
    N, Kq = w_packed.shape
    host = torch.empty((N, Kq), dtype=torch.uint8, pin_memory=True)
    hg = torch.empty(1, dtype=torch.float32, pin_memory=True)
    _check(load_library().bl_export_weights(_ptr(w_packed), _ptr(gamma), N, Kq * 4, _ptr(host), _ptr(hg),
                                            _stream(stream)), "bl_export_weights")
    return host, float(hg[0])


def bl_get_last_error() -> int:
    return load_library().bl_get_last_error()


def bl_reset_error() -> int:
    return load_library().bl_reset_error()


# ----------------------------------------------------------------- one whole step

@dataclass
class StepBuffers:
    """Device buffers of one BitLinear fwd+bwd (caller-owned, reused)."""
    w_packed: torch.Tensor
    gamma: torch.Tensor
    workspace: torch.Tensor
    xq: torch.Tensor
    sx: torch.Tensor
    y: torch.Tensor
    dX: torch.Tensor
    dW: torch.Tensor
    bwd_workspace: torch.Tensor | None = None  # x_hat scratch of the backward (bl_backward_ws)

    @staticmethod
    def allocate(M, N, K, dw_dtype=torch.bfloat16, device="cuda"):
        ws = bl_quantize_weight_workspace_size(N, K)
        return StepBuffers(
            w_packed=torch.empty((N, K // 4), dtype=torch.uint8, device=device),
            gamma=torch.empty(1, dtype=torch.float32, device=device),
            workspace=torch.empty(max(ws, 16), dtype=torch.uint8, device=device),
            xq=torch.empty((M, K), dtype=torch.int8, device=device),
            sx=torch.empty(M, dtype=torch.float32, device=device),
            y=torch.empty((M, N), dtype=torch.bfloat16, device=device),
            dX=torch.empty((M, K), dtype=torch.bfloat16, device=device),
            dW=torch.empty((N, K), dtype=dw_dtype, device=device),
            bwd_workspace=torch.empty(max(bl_backward_workspace_size(M, N, K), 16), dtype=torch.uint8, device=device),
        )


def bitlinear_step(x, W, dY, bufs: StepBuffers, stream=None):
    """One BitLinear forward + backward: S1 + S2 (bl_quantize) -> S3 -> S4 (four kernel launches)."""
    bl_quantize(W, x, bufs.w_packed, bufs.gamma, bufs.xq, bufs.sx, bufs.workspace, stream)
    bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, None, stream)
    bl_backward(dY, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.dX, bufs.dW, False, stream,
                workspace=bufs.bwd_workspace)
