// C ABI of the BitLinear library: argument validation on the host, dispatch
// to the kernels, and the per-device error word that bounded device waits
// write on timeout. See include/bitlinear.h for the contract of each call.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>

#include "../../include/bitlinear.h"
#include "bl_internal.h"

namespace {

__device__ int g_device_error = 0;

thread_local char g_msg[256] = "";

bl_status fail(bl_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the error word on the current device. Looked up on every
// call (a host-side table lookup once the module is loaded): a cached address
// would go stale if the caller reset the device and the module were loaded
// again at another address.
int* device_error_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

// Checks the current device is sm_100 and returns its error word.
bl_status current_device(int** err) {
  static int arch_ok[64] = {};  // 0 unknown, 1 ok, 2 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(BL_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= 64) return fail(BL_ERR_CUDA, "device index %d out of range", dev);
  if (arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    arch_ok[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  if (arch_ok[dev] != 1) return fail(BL_ERR_ARCH, "device %d is not sm_100", dev);
  *err = device_error_ptr();
  if (!*err) return fail(BL_ERR_CUDA, "cannot resolve the device error word");
  return BL_OK;
}

bl_status check_k(int64_t K) {
  if (K < 32 || K % 32 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "K=%lld must be a positive multiple of 32", (long long)K);
  if (K > (int64_t(1) << 30)) return fail(BL_ERR_UNSUPPORTED_SHAPE, "K=%lld too large", (long long)K);
  return BL_OK;
}

bl_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return BL_OK;
  const char* detail = bl::launch_detail();
  bl_status s = fail(BL_ERR_CUDA, "%s: %s%s%s", what, cudaGetErrorString(e), detail[0] ? "; " : "", detail);
  bl::clear_launch_detail();
  return s;
}

}  // namespace

extern "C" {

int bl_version(void) { return (1 << 16) | 0; }

const char* bl_status_string(bl_status s) {
  switch (s) {
    case BL_OK: return "BL_OK";
    case BL_ERR_INVALID_ARG: return "BL_ERR_INVALID_ARG";
    case BL_ERR_UNSUPPORTED_SHAPE: return "BL_ERR_UNSUPPORTED_SHAPE";
    case BL_ERR_DTYPE: return "BL_ERR_DTYPE";
    case BL_ERR_ALIGNMENT: return "BL_ERR_ALIGNMENT";
    case BL_ERR_ARCH: return "BL_ERR_ARCH";
    case BL_ERR_CUDA: return "BL_ERR_CUDA";
    case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT";
    case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE";
  }
  return "BL_ERR_UNKNOWN";
}

const char* bl_last_error_message(void) { return g_msg; }

size_t bl_quantize_weight_workspace_size(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0) return 0;
  return bl::quantize_workspace_bytes();
}

bl_status bl_quantize_weight(const void* W, bl_dtype w_dtype, int64_t N, int64_t K, uint8_t* w_packed,
                             float* gamma, void* workspace, size_t workspace_bytes, void* stream) {
  g_msg[0] = 0;
  if (N < 1) return fail(BL_ERR_INVALID_ARG, "N=%lld must be >= 1", (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (w_dtype != BL_BF16 && w_dtype != BL_F32) return fail(BL_ERR_DTYPE, "w_dtype %d", (int)w_dtype);
  if (!W || !w_packed || !gamma) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W) || !aligned16(w_packed) || !aligned16(gamma))
    return fail(BL_ERR_ALIGNMENT, "W, w_packed and gamma must be 16-byte aligned");
  const size_t need = bl_quantize_weight_workspace_size(N, K);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(BL_ERR_WORKSPACE, "workspace needs %zu bytes, 16-byte aligned", need);
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_quantize_weight(W, w_dtype == BL_F32, N, K, w_packed, gamma, workspace, err,
                                                static_cast<cudaStream_t>(stream)),
                     "bl_quantize_weight launch");
}

bl_status bl_quantize_weight_noalloc(const void* W, bl_dtype w_dtype, int64_t N, int64_t K, uint8_t* w_packed,
                                     float* gamma, void* stream) {
  g_msg[0] = 0;
  if (N < 1) return fail(BL_ERR_INVALID_ARG, "N=%lld must be >= 1", (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (w_dtype != BL_BF16 && w_dtype != BL_F32) return fail(BL_ERR_DTYPE, "w_dtype %d", (int)w_dtype);
  if (!W || !w_packed || !gamma) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W) || !aligned16(w_packed) || !aligned16(gamma))
    return fail(BL_ERR_ALIGNMENT, "W, w_packed and gamma must be 16-byte aligned");
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_quantize_weight_noalloc(W, w_dtype == BL_F32, N, K, w_packed, gamma, err,
                                                        static_cast<cudaStream_t>(stream)),
                     "bl_quantize_weight_noalloc launch");
}

bl_status bl_quantize_act(const void* x, int64_t M, int64_t K, int8_t* xq, float* sx, void* stream) {
  g_msg[0] = 0;
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M=%lld must be >= 0", (long long)M);
  if (bl_status s = check_k(K)) return s;
  if (M == 0) return BL_OK;
  if (!x || !xq || !sx) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(xq) || !aligned16(sx))
    return fail(BL_ERR_ALIGNMENT, "x, xq and sx must be 16-byte aligned");
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_quantize_act(x, M, K, xq, sx, static_cast<cudaStream_t>(stream)),
                     "bl_quantize_act launch");
}

bl_status bl_quantize(const void* W, bl_dtype w_dtype, int64_t N, int64_t K, const void* x, int64_t M,
                      uint8_t* w_packed, float* gamma, int8_t* xq, float* sx, void* workspace,
                      size_t workspace_bytes, void* stream) {
  g_msg[0] = 0;
  if (N < 1) return fail(BL_ERR_INVALID_ARG, "N=%lld must be >= 1", (long long)N);
  if (M < 0) return fail(BL_ERR_INVALID_ARG, "M=%lld must be >= 0", (long long)M);
  if (bl_status s = check_k(K)) return s;
  if (w_dtype != BL_BF16 && w_dtype != BL_F32) return fail(BL_ERR_DTYPE, "w_dtype %d", (int)w_dtype);
  if (!W || !w_packed || !gamma) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (M > 0 && (!x || !xq || !sx)) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W) || !aligned16(w_packed) || !aligned16(gamma) || (x && !aligned16(x)) ||
      (xq && !aligned16(xq)) || (sx && !aligned16(sx)))
    return fail(BL_ERR_ALIGNMENT, "tensors must be 16-byte aligned");
  const size_t need = bl_quantize_weight_workspace_size(N, K);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(BL_ERR_WORKSPACE, "workspace needs %zu bytes, 16-byte aligned", need);
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_quantize(W, w_dtype == BL_F32, N, K, x, M, w_packed, gamma, workspace, xq, sx, err,
                                         static_cast<cudaStream_t>(stream)),
                     "bl_quantize launch");
}

bl_status bl_forward(const int8_t* xq, const float* sx, const uint8_t* w_packed, const float* gamma, int64_t M,
                     int64_t N, int64_t K, void* y, int32_t* debug_acc, void* stream) {
  g_msg[0] = 0;
  if (M < 0 || N < 1) return fail(BL_ERR_INVALID_ARG, "M=%lld, N=%lld", (long long)M, (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return fail(BL_ERR_UNSUPPORTED_SHAPE, "M or N too large");
  if (M == 0) return BL_OK;
  if (!xq || !sx || !w_packed || !gamma || !y) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(xq) || !aligned16(sx) || !aligned16(w_packed) || !aligned16(gamma) || !aligned16(y) ||
      (debug_acc && !aligned16(debug_acc)))
    return fail(BL_ERR_ALIGNMENT, "tensors must be 16-byte aligned");
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_forward(xq, sx, w_packed, gamma, M, N, K, y, debug_acc, err,
                                        static_cast<cudaStream_t>(stream)),
                     "bl_forward launch");
}

// The checks and the launch shared by bl_backward, bl_backward_signs and
// their workspace forms. dw_signs: dW receives sign words.
static bl_status backward_common(const void* dY, const int8_t* xq, const float* sx, const uint8_t* w_packed,
                                 const float* gamma, int64_t M, int64_t N, int64_t K, void* dX, void* dW,
                                 bl_dtype dw_dtype, int accumulate_dW, int dw_signs, void* workspace,
                                 size_t workspace_bytes, void* stream, const char* what) {
  g_msg[0] = 0;
  if (M < 0 || N < 1) return fail(BL_ERR_INVALID_ARG, "M=%lld, N=%lld", (long long)M, (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (N % 8 != 0) return fail(BL_ERR_UNSUPPORTED_SHAPE, "N=%lld must be a multiple of 8", (long long)N);
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return fail(BL_ERR_UNSUPPORTED_SHAPE, "M or N too large");
  if (dw_signs) {
    if (!dW) return fail(BL_ERR_INVALID_ARG, "null dw_sign_words");
  } else {
    if (dW && dw_dtype != BL_BF16 && dw_dtype != BL_F32) return fail(BL_ERR_DTYPE, "dw_dtype %d", (int)dw_dtype);
    if (!dX && !dW) return BL_OK;
  }
  if (M > 0 && !dY) return fail(BL_ERR_INVALID_ARG, "null dY");
  if (dX && (!w_packed || !gamma)) return fail(BL_ERR_INVALID_ARG, "dX needs w_packed and gamma");
  if (dW && M > 0 && (!xq || !sx)) return fail(BL_ERR_INVALID_ARG, "dW needs xq and sx");
  if ((dY && !aligned16(dY)) || (xq && !aligned16(xq)) || (sx && !aligned16(sx)) ||
      (w_packed && !aligned16(w_packed)) || (gamma && !aligned16(gamma)) || (dX && !aligned16(dX)) ||
      (dW && !aligned16(dW)))
    return fail(BL_ERR_ALIGNMENT, "tensors must be 16-byte aligned");
  if (workspace && bl::backward_uses_xhat(N)) {
    const size_t need = bl_backward_workspace_size(M, N, K);
    if (workspace_bytes < need || !aligned16(workspace))
      return fail(BL_ERR_WORKSPACE, "workspace needs %zu bytes, 16-byte aligned", need);
  }
  // x_hat is only made when dW is computed from tokens and worth it
  void* xhat = (workspace && dW && M > 0 && bl::backward_uses_xhat(N)) ? workspace : nullptr;
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_backward(dY, xq, sx, w_packed, gamma, M, N, K, dX, dW,
                                         dw_signs ? 0 : dw_dtype == BL_F32, dw_signs ? 0 : accumulate_dW != 0,
                                         dw_signs, xhat, err, static_cast<cudaStream_t>(stream)),
                     what);
}

size_t bl_backward_workspace_size(int64_t M, int64_t N, int64_t K) {
  return (M > 0 && K > 0 && bl::backward_uses_xhat(N)) ? static_cast<size_t>(M) * static_cast<size_t>(K) * 2 : 0;
}

bl_status bl_backward(const void* dY, const int8_t* xq, const float* sx, const uint8_t* w_packed,
                      const float* gamma, int64_t M, int64_t N, int64_t K, void* dX, void* dW, bl_dtype dw_dtype,
                      int accumulate_dW, void* stream) {
  return backward_common(dY, xq, sx, w_packed, gamma, M, N, K, dX, dW, dw_dtype, accumulate_dW, 0, nullptr, 0,
                         stream, "bl_backward launch");
}

bl_status bl_backward_ws(const void* dY, const int8_t* xq, const float* sx, const uint8_t* w_packed,
                         const float* gamma, int64_t M, int64_t N, int64_t K, void* dX, void* dW, bl_dtype dw_dtype,
                         int accumulate_dW, void* workspace, size_t workspace_bytes, void* stream) {
  return backward_common(dY, xq, sx, w_packed, gamma, M, N, K, dX, dW, dw_dtype, accumulate_dW, 0, workspace,
                         workspace_bytes, stream, "bl_backward_ws launch");
}

bl_status bl_backward_signs(const void* dY, const int8_t* xq, const float* sx, const uint8_t* w_packed,
                            const float* gamma, int64_t M, int64_t N, int64_t K, void* dX, uint32_t* dw_sign_words,
                            void* stream) {
  return backward_common(dY, xq, sx, w_packed, gamma, M, N, K, dX, dw_sign_words, BL_BF16, 0, 1, nullptr, 0, stream,
                         "bl_backward_signs launch");
}

bl_status bl_backward_signs_ws(const void* dY, const int8_t* xq, const float* sx, const uint8_t* w_packed,
                               const float* gamma, int64_t M, int64_t N, int64_t K, void* dX,
                               uint32_t* dw_sign_words, void* workspace, size_t workspace_bytes, void* stream) {
  return backward_common(dY, xq, sx, w_packed, gamma, M, N, K, dX, dw_sign_words, BL_BF16, 0, 1, workspace,
                         workspace_bytes, stream, "bl_backward_signs_ws launch");
}

bl_status bl_export_weights(const uint8_t* w_packed, const float* gamma, int64_t N, int64_t K,
                            uint8_t* host_packed, float* host_gamma, void* stream) {
  g_msg[0] = 0;
  if (N < 1) return fail(BL_ERR_INVALID_ARG, "N=%lld must be >= 1", (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (!w_packed || !gamma || !host_packed || !host_gamma) return fail(BL_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (bl_status s = cuda_status(cudaMemcpyAsync(host_packed, w_packed, static_cast<size_t>(N * (K / 4)),
                                                cudaMemcpyDeviceToHost, st),
                                "export packed"))
    return s;
  if (bl_status s = cuda_status(cudaMemcpyAsync(host_gamma, gamma, sizeof(float), cudaMemcpyDeviceToHost, st),
                                "export gamma"))
    return s;
  return cuda_status(cudaStreamSynchronize(st), "export sync");
}

bl_status bl_sign_pack(const void* dW, bl_dtype dw_dtype, int64_t N, int64_t K, uint32_t* sign_words, void* stream) {
  g_msg[0] = 0;
  if (N < 1) return fail(BL_ERR_INVALID_ARG, "N=%lld must be >= 1", (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (dw_dtype != BL_BF16 && dw_dtype != BL_F32) return fail(BL_ERR_DTYPE, "dw_dtype %d", (int)dw_dtype);
  if (!dW || !sign_words) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(dW) || !aligned16(sign_words)) return fail(BL_ERR_ALIGNMENT, "dW and sign_words must be 16-byte aligned");
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_sign_pack(dW, dw_dtype == BL_F32, N, K, sign_words, static_cast<cudaStream_t>(stream)),
                     "bl_sign_pack");
}

bl_status bl_sign_vote(const uint32_t* sign_words, int ranks, int64_t N, int64_t K, uint8_t* direction,
                       void* stream) {
  g_msg[0] = 0;
  if (N < 1) return fail(BL_ERR_INVALID_ARG, "N=%lld must be >= 1", (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (ranks < 1 || ranks > 127) return fail(BL_ERR_INVALID_ARG, "ranks=%d must be in 1..127", ranks);
  if (!sign_words || !direction) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(sign_words) || !aligned16(direction))
    return fail(BL_ERR_ALIGNMENT, "sign_words and direction must be 16-byte aligned");
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_sign_vote(sign_words, ranks, N, K, direction, static_cast<cudaStream_t>(stream)),
                     "bl_sign_vote");
}

bl_status bl_signsgd_update(void* W, bl_dtype w_dtype, int64_t N, int64_t K, const uint8_t* direction, float lr,
                            void* stream) {
  g_msg[0] = 0;
  if (N < 1) return fail(BL_ERR_INVALID_ARG, "N=%lld must be >= 1", (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (w_dtype != BL_BF16 && w_dtype != BL_F32) return fail(BL_ERR_DTYPE, "w_dtype %d", (int)w_dtype);
  if (!(lr - lr == 0.0f)) return fail(BL_ERR_INVALID_ARG, "lr must be finite");
  if (!W || !direction) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W) || !aligned16(direction)) return fail(BL_ERR_ALIGNMENT, "W and direction must be 16-byte aligned");
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_signsgd_update(W, w_dtype == BL_F32, N, K, direction, lr,
                                               static_cast<cudaStream_t>(stream)),
                     "bl_signsgd_update");
}

bl_status bl_signsgd_apply(const uint32_t* sign_words, int ranks, void* W, bl_dtype w_dtype, int64_t N, int64_t K,
                           float lr, uint8_t* w_packed, float* gamma, void* workspace, size_t workspace_bytes,
                           void* stream) {
  g_msg[0] = 0;
  if (N < 1) return fail(BL_ERR_INVALID_ARG, "N=%lld must be >= 1", (long long)N);
  if (bl_status s = check_k(K)) return s;
  if (ranks < 1 || ranks > 127) return fail(BL_ERR_INVALID_ARG, "ranks=%d must be in 1..127", ranks);
  if (w_dtype != BL_BF16 && w_dtype != BL_F32) return fail(BL_ERR_DTYPE, "w_dtype %d", (int)w_dtype);
  if (!(lr - lr == 0.0f)) return fail(BL_ERR_INVALID_ARG, "lr must be finite");
  if (!sign_words || !W || !w_packed || !gamma) return fail(BL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(sign_words) || !aligned16(W) || !aligned16(w_packed) || !aligned16(gamma))
    return fail(BL_ERR_ALIGNMENT, "sign_words, W, w_packed and gamma must be 16-byte aligned");
  const size_t need = bl_quantize_weight_workspace_size(N, K);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(BL_ERR_WORKSPACE, "workspace needs %zu bytes, 16-byte aligned", need);
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_signsgd_apply(sign_words, ranks, W, w_dtype == BL_F32, N, K, lr, w_packed, gamma,
                                              workspace, err, static_cast<cudaStream_t>(stream)),
                     "bl_signsgd_apply");
}

bl_status bl_selftest_timeout(void* stream) {
  g_msg[0] = 0;
  int* err = nullptr;
  if (bl_status s = current_device(&err)) return s;
  return cuda_status(bl::launch_selftest_timeout(err, static_cast<cudaStream_t>(stream)), "bl_selftest_timeout");
}

bl_status bl_get_last_error(void) {
  g_msg[0] = 0;
  if (cudaError_t e = cudaDeviceSynchronize(); e != cudaSuccess) return cuda_status(e, "cudaDeviceSynchronize");
  int v = 0;
  if (cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)); e != cudaSuccess)
    return cuda_status(e, "read device error word");
  if (v == BL_ERR_TIMEOUT) return fail(BL_ERR_TIMEOUT, "a device pipeline wait exceeded its bound");
  return v == 0 ? BL_OK : fail(static_cast<bl_status>(v), "device error %d", v);
}

bl_status bl_reset_error(void) {
  g_msg[0] = 0;
  const int zero = 0;
  return cuda_status(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)), "reset device error word");
}

}  // extern "C"
