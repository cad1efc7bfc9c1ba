// Host-side launchers shared between the kernel translation units and the
// C ABI layer. Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace bl {

// Launches `kernel` as a programmatic dependent of the previous kernel in
// `stream` (the kernel itself waits for it before reading its inputs).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- S1: absmean ternarisation + 2-bit packing (with S2 in the same launches)
// Most CTAs of the sum launch of S1 (one fp64 partial sum each).
constexpr int kMaxQuantCtas = 1024;

// Workspace (each part on its own 128-byte lines): at 0 the arrivals at the
// exact-sum barrier (u32); at 128 256 uint64 exact-sum bins (one per exponent
// field); at 2304 one fp64 partial sum per CTA of the sum launch. The launch
// that makes the partial sums (the sum launch, or the sign-gradient apply
// pass) clears the first two parts and fills the third on every call, so the
// caller's workspace needs no initialisation.
constexpr size_t kWsArrive = 0;
constexpr size_t kWsBins = 128;
constexpr size_t kWsParts = kWsBins + 8 * 256 + 128;
constexpr size_t kWsBytes = kWsParts + 8 * static_cast<size_t>(kMaxQuantCtas);

// Bytes of the S1 workspace (exact-sum arrival counter and bins, one fp64
// partial sum per CTA of the sum launch); the same for every tensor size.
// Needs no initialisation.
size_t quantize_workspace_bytes();

// S1 on W [N,K] and, when M > 0, S2 on x [M,K]: a sum launch (|W| partial
// sums and the token rows) and a code launch (gamma and the codes). `err` is
// the device error word (an exact-sum barrier wait that gave up records a
// timeout there).
cudaError_t launch_quantize(const void* W, int w_is_f32, int64_t N, int64_t K, const void* x, int64_t M,
                            uint8_t* packed, float* gamma, void* workspace, int8_t* xq, float* sx, int* err,
                            cudaStream_t s);

// S1 alone (launch_quantize with M = 0).
cudaError_t launch_quantize_weight(const void* W, int w_is_f32, int64_t N, int64_t K, uint8_t* packed,
                                   float* gamma, void* workspace, int* err, cudaStream_t s);

// S1 with the workspace in a fixed device array (g_noalloc_ws in k_quant.cu).
cudaError_t launch_quantize_weight_noalloc(const void* W, int w_is_f32, int64_t N, int64_t K, uint8_t* packed,
                                           float* gamma, int* err, cudaStream_t s);

// The code launch of S1 alone, for a W whose |W| partial sums another kernel
// of the stream has just left in the workspace (nparts fp64 values at
// kWsParts, bins and arrival counter cleared). part_roundings bounds the
// roundings any term went through inside its partial sum (it sets the
// enclosure of S that gamma is formed from).
cudaError_t launch_quantize_codes(const void* W, int w_is_f32, int64_t N, int64_t K, int nparts,
                                  double part_roundings, uint8_t* packed, float* gamma, void* workspace, int* err,
                                  cudaStream_t s);

// ---- S2 alone: per-token absmax INT8
cudaError_t launch_quantize_act(const void* x, int64_t M, int64_t K, int8_t* xq, float* sx, cudaStream_t s);

// ---- S3 / S4 GEMMs (tcgen05)
cudaError_t launch_forward(const int8_t* xq, const float* sx, const uint8_t* w_packed, const float* gamma,
                           int64_t M, int64_t N, int64_t K, void* y, int32_t* debug_acc, int* err,
                           cudaStream_t s);

// Whether the backward makes x_hat in a workspace for dW with N features
// (else it rebuilds x_hat in every dW tile).
bool backward_uses_xhat(int64_t N);

// dX and/or dW (either output may be null) in one launch. With dw_signs, dW
// receives the sign words of dW ([N*K/32] uint32, element 32w + j at bit j of
// word w) instead of dW itself. With xhat_ws (bf16 [M][K], 16-byte aligned), a
// launch before the GEMMs writes x_hat there and dW's tiles load it instead of
// rebuilding it.
cudaError_t launch_backward(const void* dY, const int8_t* xq, const float* sx, const uint8_t* w_packed,
                            const float* gamma, int64_t M, int64_t N, int64_t K, void* dX, void* dW, int dw_is_f32,
                            int accumulate, int dw_signs, void* xhat_ws, int* err, cudaStream_t s);

// ---- Master-free sign-gradient update (k_signsgd.cu)
// Sign bits of dW [N,K] (bf16 or f32): out [N*K/32] words, element 32w+j -> bit j.
cudaError_t launch_sign_pack(const void* dW, int dw_is_f32, int64_t N, int64_t K, uint32_t* out, cudaStream_t s);
// Majority vote of `ranks` sign-word arrays (rank r at words + r*N*K/32) ->
// 2-bit packed direction [N, K/4].
cudaError_t launch_sign_vote(const uint32_t* words, int ranks, int64_t N, int64_t K, uint8_t* direction,
                             cudaStream_t s);
// W [N,K] (bf16 or f32) <- dtype_rn(fp32(W) - lr * direction), in place.
cudaError_t launch_signsgd_update(void* W, int w_is_f32, int64_t N, int64_t K, const uint8_t* direction, float lr,
                                  cudaStream_t s);

// The holder's whole step in two launches: vote of `ranks` sign-word arrays,
// the update of W in place, |W'| partial sums in the same sweep, then the
// code launch of S1 (new packed codes and gamma of W').
cudaError_t launch_signsgd_apply(const uint32_t* words, int ranks, void* W, int w_is_f32, int64_t N, int64_t K,
                                 float lr, uint8_t* packed, float* gamma, void* workspace, int* err, cudaStream_t s);

// One warp waiting on an mbarrier that is never completed (bounded wait test).
cudaError_t launch_selftest_timeout(int* err, cudaStream_t s);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Detail of the last host-side launch failure on this thread ("" if none).
const char* launch_detail();
void clear_launch_detail();

}  // namespace bl
