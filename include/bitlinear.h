/*
 * bitlinear.h -- C ABI of the B200 (sm_100a) BitNet b1.58 BitLinear training
 * hot path: absmean ternarisation with 2-bit packing, per-token absmax INT8
 * activation quantisation, the INT32-exact forward GEMM and the
 * straight-through backward GEMMs.
 *
 * Sources, cited by page title and section:
 *   "bitnet-qat-train" (kernel card): intro bullets (fused ternarise + scale +
 *       pack pass, INT8 tensor-core forward, saved 2-bit/INT8 state),
 *       Semantics, Requirements (K divisible by 32, bf16 activations, bf16 or
 *       f32 master weights), Usage (export of packed weights and scale).
 *   "1BitTraining.md": quantisation helpers (activation_quant, weight_quant).
 *   "bitlinear.py": ternary_quantize, activation_quant_int8, BitLinear.forward.
 *
 * Conventions shared by every entry point
 *   - Every tensor argument is a DEVICE pointer unless its name starts with
 *     host_. The caller allocates and owns every buffer; the library never
 *     allocates device memory and keeps no state except one error word per
 *     device (and the fixed scratch array of bl_quantize_weight_noalloc).
 *   - Tensors are dense, row-major, and 16-byte aligned at their base.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). All work is enqueued asynchronously on it; nothing here
 *     synchronises the host except bl_export_weights and bl_get_last_error.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and returned as a bl_status; bl_last_error_message() then holds a
 *     one-line description (thread-local).
 *   - Device-side failures (a pipeline wait that exceeded its time bound) are
 *     recorded in the device error word and reported by bl_get_last_error.
 *     No kernel traps or asserts.
 *   - Shapes: M = tokens, K = in_features, N = out_features.
 *     x [M,K] bf16, W [N,K] bf16|f32, dY [M,N] bf16.
 *   - Requires an sm_100 device (B200).
 *
 * Saved state between forward and backward ("bitnet-qat-train", third intro
 * bullet): (xq, sx, w_packed, gamma). The caller keeps it.
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bl_status {
    BL_OK = 0,
    BL_ERR_INVALID_ARG = 1,        /* null pointer or negative size */
    BL_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 32 != 0, K < 32, or N % 8 != 0 in backward */
    BL_ERR_DTYPE = 3,              /* unknown bl_dtype */
    BL_ERR_ALIGNMENT = 4,          /* a tensor base is not 16-byte aligned */
    BL_ERR_ARCH = 5,               /* current device is not sm_100 */
    BL_ERR_CUDA = 6,               /* a CUDA runtime/driver call failed */
    BL_ERR_TIMEOUT = 7,            /* a device pipeline wait exceeded its bound */
    BL_ERR_WORKSPACE = 8           /* workspace missing or too small */
} bl_status;

typedef enum bl_dtype {
    BL_BF16 = 0,
    BL_F32 = 1
} bl_dtype;

/* Library version, (major << 16) | minor. */
int bl_version(void);

/* Human-readable name of a status code (static string). */
const char* bl_status_string(bl_status status);

/* Description of the last host-side failure on the calling thread. */
const char* bl_last_error_message(void);

/*
 * Bytes of device workspace bl_quantize_weight and bl_quantize need for an
 * [N,K] tensor: an arrival counter and 256 exact-sum bins, and one fp64
 * partial sum of |W| per CTA of the summing launch (at most 1024), 10496
 * bytes for every non-empty tensor. Returns 0 for an empty tensor.
 */
size_t bl_quantize_weight_workspace_size(int64_t N, int64_t K);

/*
 * S1 -- absmean ternarisation + 2-bit packing ("1BitTraining.md",
 * weight_quant; "bitlinear.py", ternary_quantize; "bitnet-qat-train", first
 * intro bullet: one fused ternarise + scale + pack pass, no bf16 fake-quant
 * tensor).
 *
 *   gamma   = max(fp32(fp64(S / (N*K))), 1e-5)  S = sum|W| rounded once to fp64
 *   code    = clamp(rint_half_even(fp32(W / gamma)), -1, 1)
 *   packing : element k of row n -> byte n*K/4 + k/4, bits 2*(k%4)..+1,
 *             field 00 = 0, 01 = +1, 11 = -1 (10 never written)
 *
 * W         [N,K] master weights, w_dtype = BL_BF16 or BL_F32 (read only)
 * w_packed  [N,K/4] uint8 output
 * gamma     one float output (device); the dequantisation multiplier
 * workspace device scratch of at least bl_quantize_weight_workspace_size(N,K)
 *           bytes, 16-byte aligned; contents need no initialisation and are
 *           overwritten.
 * gamma is exact: the fp64 sum of |W| (per-CTA trees, then the CTAs' sums in
 * a fixed order) carries a bounded rounding error; gamma is formed at both
 * ends of that enclosure of the exact sum, and
 * where the two differ (about one tensor in 10^5) the library sums |W|
 * exactly in integers and rounds once. gamma therefore never depends on the
 * summation order or on the GPU, and the same W gives bit-identical outputs
 * on every call.
 * Launches: a summing launch (each CTA stores the fp64 sum of |W| over its
 * slice of W; nothing waits) and a coding launch that starts once the first
 * has completed (every CTA forms gamma from the partial sums and writes the
 * codes of its share, reading W again, mostly from L2). Only in the rare
 * exact-sum case do the coding CTAs (never more than can be resident at
 * once) meet at a grid-wide barrier; its wait is bounded: a barrier that
 * cannot complete -- e.g. SMs held by other work for seconds -- records
 * BL_ERR_TIMEOUT in the device error word.
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE (K % 32), BL_ERR_DTYPE,
 *         BL_ERR_ALIGNMENT, BL_ERR_WORKSPACE, BL_ERR_ARCH, BL_ERR_CUDA.
 */
bl_status bl_quantize_weight(const void* W, bl_dtype w_dtype, int64_t N, int64_t K,
                             uint8_t* w_packed, float* gamma,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * bl_quantize_weight without a workspace. The pages have no counterpart to
 * this call; it exists for callers that cannot allocate device memory --
 * plugin hosts that hand the library only the input and output buffers they
 * own, and runtimes whose device memory is a fixed pool reserved up front --
 * and so cannot pass the workspace bl_quantize_weight asks for.
 *
 * It computes exactly what bl_quantize_weight computes (same kernels, same
 * bit-identical outputs) and calls no allocator. Its scratch -- the arrival
 * counter, the exact-sum bins and the partial sums that bl_quantize_weight
 * keeps in the caller's workspace -- is a fixed array inside the library of
 * 10496 bytes, enough for a tensor of any size; each GPU that loads the library
 * keeps that array until the process exits.
 *
 * Each call looks up the array's device address on the current device (a
 * runtime query; the first one on a device loads the library's device code
 * there, so make the first call on each device before any stream capture).
 * The address is not cached, so a call after the caller reset the device
 * finds the array where the reloaded device code put it. All calls share the
 * one array and nothing in it needs to start at zero (each call clears its
 * counter and bins before use and overwrites the rest), but two calls whose
 * kernels overlap on the GPU -- on different streams of one device without
 * ordering between them -- race on it and may produce a wrong gamma and
 * codes or a barrier timeout: order them on one stream or with events.
 *
 * Arguments, outputs and errors: as bl_quantize_weight, without the
 * workspace pair.
 */
bl_status bl_quantize_weight_noalloc(const void* W, bl_dtype w_dtype, int64_t N, int64_t K,
                                     uint8_t* w_packed, float* gamma, void* stream);

/*
 * S2 -- per-token absmax INT8 quantisation ("1BitTraining.md",
 * activation_quant; "bitlinear.py", activation_quant_int8).
 *
 *   a     = max(max_k |x[m,k]|, 1e-5)
 *   xq    = clamp(rint_half_even(fp32(x * fp32(127 / a))), -127, 127)
 *   sx[m] = fp32(a / 127)                (x_hat = xq * sx)
 *
 * x  [M,K] bf16 (finite values), xq [M,K] int8 output, sx [M] float output.
 * M == 0 is a no-op. Errors: as bl_quantize_weight (no workspace).
 */
bl_status bl_quantize_act(const void* x, int64_t M, int64_t K,
                          int8_t* xq, float* sx, void* stream);

/*
 * S1 + S2 in one call: the same outputs as bl_quantize_weight(W, ...) followed
 * by bl_quantize_act(x, ...), bit for bit. The two steps are independent, so
 * S2 runs in S1's summing launch: each CTA quantises its share of the token
 * rows, then sums its slice of W, so that both streams share HBM in one
 * pass. (The pages run the two quantisers one after the other; this is a
 * scheduling choice only.)
 *
 * Arguments: those of bl_quantize_weight and bl_quantize_act. M == 0 skips
 * S2 (x, xq, sx may then be NULL). Errors: as bl_quantize_weight, plus those
 * of bl_quantize_act's arguments.
 */
bl_status bl_quantize(const void* W, bl_dtype w_dtype, int64_t N, int64_t K,
                      const void* x, int64_t M,
                      uint8_t* w_packed, float* gamma, int8_t* xq, float* sx,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * S3 -- forward ("bitnet-qat-train", Semantics):
 *
 *   acc[m,n] = sum_k xq[m,k] * code[n,k]            exact INT32 (tensor cores)
 *   y[m,n]   = bf16_rn(fp32(acc) * fp32(sx[m] * gamma))
 *
 * xq [M,K] int8, sx [M] float, w_packed [N,K/4] uint8, gamma one float.
 * y [M,N] bf16 output. debug_acc: NULL, or an [M,N] int32 output that
 * receives acc (parity checking).
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE (K % 32), BL_ERR_ALIGNMENT,
 *         BL_ERR_ARCH, BL_ERR_CUDA; device timeouts via bl_get_last_error.
 */
bl_status bl_forward(const int8_t* xq, const float* sx, const uint8_t* w_packed,
                     const float* gamma, int64_t M, int64_t N, int64_t K,
                     void* y, int32_t* debug_acc, void* stream);

/*
 * S4 -- straight-through backward ("bitnet-qat-train", Semantics; the
 * quantisers' Jacobian is taken as 1 and gamma as constant):
 *
 *   dX[m,k] = bf16_rn(gamma * sum_n dY[m,n] * code[n,k])          fp32 accumulate
 *   dW[n,k] = round(sum_m dY[m,n] * x_hat[m,k] (+ dW[n,k] if accumulate_dW))
 *   x_hat[m,k] = bf16_rn(fp32(xq[m,k]) * sx[m])
 *
 * Both operands are rebuilt in shared memory from the saved 2-bit / INT8
 * state; no bf16 copy of W_hat or x_hat is written to device memory (see
 * bl_backward_ws for the form that makes x_hat once in a workspace).
 * dY [M,N] bf16. dX [M,K] bf16 output or NULL (skipped). dW [N,K] output or
 * NULL (skipped), of dw_dtype (BL_BF16 or BL_F32); accumulate_dW != 0 adds to
 * the existing contents instead of overwriting them.
 * Requires N % 8 == 0 (dY rows must be 16-byte multiples for the TMA loads).
 * Errors: as bl_forward, plus BL_ERR_DTYPE.
 */
bl_status bl_backward(const void* dY, const int8_t* xq, const float* sx,
                      const uint8_t* w_packed, const float* gamma,
                      int64_t M, int64_t N, int64_t K,
                      void* dX, void* dW, bl_dtype dw_dtype, int accumulate_dW,
                      void* stream);

/*
 * bl_backward with a workspace for x_hat: the same dX and dW, bit for bit.
 * A first launch writes x_hat (bf16 [M][K], M*K*2 bytes) into the
 * workspace from xq and sx, converted exactly as above; dW's tiles then load
 * their x_hat operand by TMA instead of rebuilding it from xq and sx in every
 * tile (each element would be rebuilt once per 256-feature block of dW).
 * The workspace is transient scratch of this call (no saved state; it holds
 * nothing the caller needs afterwards), owned by the caller, 16-byte
 * aligned, of at least bl_backward_workspace_size(M, N, K) bytes, and needs
 * no initialisation; one call at a time per workspace. workspace == NULL: as
 * bl_backward. Where dW has fewer than 2048 features (8 blocks of 256, each
 * of which rebuilds x_hat once) the extra launch costs more than it saves:
 * the size is then 0 and the workspace is not used (any pointer, or NULL).
 * Errors: as bl_backward, plus BL_ERR_WORKSPACE.
 */
size_t bl_backward_workspace_size(int64_t M, int64_t N, int64_t K);
bl_status bl_backward_ws(const void* dY, const int8_t* xq, const float* sx,
                         const uint8_t* w_packed, const float* gamma,
                         int64_t M, int64_t N, int64_t K,
                         void* dX, void* dW, bl_dtype dw_dtype, int accumulate_dW,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Export of the packed weights and their scale for inference
 * ("bitnet-qat-train", Usage: export_inference returns w_packed, scale_wt).
 * Copies w_packed [N,K/4] and gamma (scale_wt = gamma, the dequantisation
 * multiplier) into HOST buffers and synchronises `stream`.
 */
bl_status bl_export_weights(const uint8_t* w_packed, const float* gamma,
                            int64_t N, int64_t K,
                            uint8_t* host_packed, float* host_gamma, void* stream);

/*
 * Master-free sign-gradient training, data parallel ("1BitTraining.md", "Why
 * this always holds", closing paragraph on implications: the straight-through
 * gradient and the gradient of the quantised weight have the same sign, so a
 * sign-based optimiser needs only the 2-bit weights on each device and one
 * bit of gradient per weight, sent to one place that accumulates them).
 * One step over R data-parallel ranks:
 *   every rank   bl_backward_signs -> dX and the sign words of dW (or
 *                bl_backward -> dW, then bl_sign_pack -> its sign words)
 *   exchange     the R ranks' sign words are gathered (N*K/8 bytes a rank)
 *   holder of W  bl_signsgd_apply: vote, update of W and the next codes and
 *                gamma in two launches (or the three calls bl_sign_vote,
 *                bl_signsgd_update, bl_quantize_weight), which go back to
 *                the ranks.
 */

/*
 * G1: the 1-bit gradient. sign_words [N*K/32] (uint32) receives the IEEE sign
 * bit of every element of dW [N,K] (dw_dtype BL_BF16 or BL_F32): element
 * 32*w + j of the flattened tensor is bit j of word w (1 = negative; -0.0
 * counts as negative). Reads N*K*(2|4) bytes, writes N*K/8.
 * Errors: BL_ERR_INVALID_ARG (null, N < 1), BL_ERR_UNSUPPORTED_SHAPE (K),
 *         BL_ERR_DTYPE, BL_ERR_ALIGNMENT, BL_ERR_ARCH, BL_ERR_CUDA.
 */
bl_status bl_sign_pack(const void* dW, bl_dtype dw_dtype, int64_t N, int64_t K,
                       uint32_t* sign_words, void* stream);

/*
 * S4 with G1 fused: bl_backward's dX (may be NULL) and, instead of dW, its
 * sign words -- dw_sign_words [N*K/32] uint32 in bl_sign_pack's layout,
 * written by the epilogue of the dW tiles straight from the fp32 sums (the
 * rounding of dW to bf16 or fp32 keeps the sign, -0 included, so the words
 * equal bl_sign_pack of bl_backward's dW bit for bit). dW is never written:
 * N*K/8 bytes leave the kernel instead of N*K*2, and no second pass reads dW
 * back. M == 0 writes all-zero words (dW = +0).
 * Arguments and errors: as bl_backward (no accumulation, no dtype).
 */
bl_status bl_backward_signs(const void* dY, const int8_t* xq, const float* sx,
                            const uint8_t* w_packed, const float* gamma,
                            int64_t M, int64_t N, int64_t K,
                            void* dX, uint32_t* dw_sign_words, void* stream);

/* bl_backward_signs with bl_backward_ws's x_hat workspace (same words, same
 * dX). Arguments and errors: as those two. */
bl_status bl_backward_signs_ws(const void* dY, const int8_t* xq, const float* sx,
                               const uint8_t* w_packed, const float* gamma,
                               int64_t M, int64_t N, int64_t K,
                               void* dX, uint32_t* dw_sign_words,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * G2: the accumulation. sign_words holds `ranks` arrays of N*K/32 words back
 * to back (rank r at sign_words + r*N*K/32), 1 <= ranks <= 127. direction
 * [N,K/4] receives, per weight, +1 where more ranks have a positive (sign bit
 * 0) gradient, -1 where more have a negative one, 0 on a tie, in the 2-bit
 * packing of w_packed (00 = 0, 01 = +1, 11 = -1).
 * Errors: as bl_sign_pack (BL_ERR_INVALID_ARG also for ranks out of range).
 */
bl_status bl_sign_vote(const uint32_t* sign_words, int ranks, int64_t N, int64_t K,
                       uint8_t* direction, void* stream);

/*
 * G3: the sign-gradient step where the master weights are held. In place on
 * W [N,K] (w_dtype BL_BF16 or BL_F32): W = dtype_rn(fp32(W) - lr * d) with d
 * the direction of bl_sign_vote; the fp32 subtraction rounds once (lr * d is
 * exact), bf16 masters round once more. Where d = 0 (or the unused field 10)
 * the weight is left bit for bit. lr must be finite.
 * Errors: as bl_sign_pack (BL_ERR_INVALID_ARG also for a non-finite lr).
 */
bl_status bl_signsgd_update(void* W, bl_dtype w_dtype, int64_t N, int64_t K,
                            const uint8_t* direction, float lr, void* stream);

/*
 * G2 + G3 + S1 on the holder, fused: the same W, w_packed and gamma as
 * bl_sign_vote, bl_signsgd_update and bl_quantize_weight called in turn, bit
 * for bit, in two launches. The first votes the `ranks` sign-word arrays
 * (layout of bl_sign_vote), updates W in place (bl_signsgd_update's rule) and
 * sums |W| of the updated weights in fp64 in the same sweep; the second is
 * bl_quantize_weight's code launch (gamma exactly as there, then the codes,
 * re-reading W from L2). Saves the direction array (N*K/4 bytes written and
 * read back), the vote launch and the re-read of W from HBM for its sum.
 * workspace: as bl_quantize_weight (bl_quantize_weight_workspace_size bytes,
 * 16-byte aligned, no initialisation; one call at a time per workspace).
 * Errors: as bl_signsgd_update and bl_quantize_weight (BL_ERR_INVALID_ARG
 * also for ranks out of 1..127, BL_ERR_WORKSPACE); a device wait that gave up
 * records BL_ERR_TIMEOUT (bl_get_last_error).
 */
bl_status bl_signsgd_apply(const uint32_t* sign_words, int ranks, void* W, bl_dtype w_dtype,
                           int64_t N, int64_t K, float lr, uint8_t* w_packed, float* gamma,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises the current device, then returns BL_OK or the first device
 * failure recorded since the last bl_reset_error (BL_ERR_TIMEOUT).
 */
bl_status bl_get_last_error(void);

/* Clears the current device's error word (synchronous). */
bl_status bl_reset_error(void);

/*
 * Failure-detection self-test: enqueues one warp that waits on a pipeline
 * barrier nothing ever completes, with the same bounded wait (2 s) every
 * pipeline kernel uses. The wait gives up, records BL_ERR_TIMEOUT in the
 * device error word and the kernel returns; bl_get_last_error then reports
 * BL_ERR_TIMEOUT and the CUDA context stays usable. Clear it with
 * bl_reset_error. Returns the launch status.
 */
bl_status bl_selftest_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
