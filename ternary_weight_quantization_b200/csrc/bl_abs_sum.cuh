// |w| widened to fp64 exactly and added to an fp64 accumulator: the partial
// sums of S = sum |W| that S1's gamma is formed from. Shared by the sum launch
// of S1 and by the sign-gradient pass that writes W and sums it in the same
// sweep; both feed the same code launch, whose enclosure of S counts the
// roundings these additions make.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace bl {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// |w| widened to fp64 exactly from its bit pattern with the sign cleared.
// Normal values take integer arithmetic only (a bf16's fp64 high word is
// b * 2^13 + 0x38000000: exponent re-bias 127 -> 1023; an fp32's is
// (b >> 3) + 0x38000000 with low word b << 29); zeros and subnormals (zero
// exponent field) take a separate, rarely taken path. Inputs are finite.
//
// 8 bf16 magnitudes of one 16-byte vector, added to acc in element order.
__device__ __forceinline__ double add_abs8_bf16(double acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t mn = 0xFFFFFFFFu;  // per half: smallest 15-bit magnitude
#pragma unroll
  for (int j = 0; j < 4; ++j) asm("min.u16x2 %0, %0, %1;" : "+r"(mn) : "r"(w[j] & 0x7FFF7FFFu));
  if (min(mn << 16, mn & 0xFFFF0000u) >= 0x00800000u) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc = __dadd_rn(acc, __hiloint2double(static_cast<int>(((w[j] & 0x7FFFu) << 13) + 0x38000000u), 0));
      acc = __dadd_rn(acc, __hiloint2double(static_cast<int>(((w[j] & 0x7FFF0000u) >> 3) + 0x38000000u), 0));
    }
    return acc;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    acc = __dadd_rn(acc, static_cast<double>(fabsf(bf16_lo(w[j]))));
    acc = __dadd_rn(acc, static_cast<double>(fabsf(bf16_hi(w[j]))));
  }
  return acc;
}

// 4 fp32 magnitudes of one 16-byte vector, added to acc in element order.
__device__ __forceinline__ double add_abs4_f32(double acc, const uint4& v) {
  const uint32_t w[4] = {v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu, v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu};
  if (min(min(w[0], w[1]), min(w[2], w[3])) >= 0x00800000u) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      acc = __dadd_rn(acc, __hiloint2double(static_cast<int>((w[j] >> 3) + 0x38000000u), static_cast<int>(w[j] << 29)));
    return acc;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) acc = __dadd_rn(acc, static_cast<double>(__uint_as_float(w[j])));
  return acc;
}

template <bool kF32>
__device__ __forceinline__ double add_abs(double acc, const uint4& v) {
  if constexpr (kF32) return add_abs4_f32(acc, v);
  else return add_abs8_bf16(acc, v);
}

}  // namespace bl
