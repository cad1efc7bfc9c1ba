// S1 and S2 of the BitLinear hot path on sm_100a: absmean ternarisation with
// 2-bit packing, and per-token absmax INT8 activation quantisation.
//
// Both are HBM-bound streaming passes with 16-byte vector loads and no
// intermediate tensors in device memory. S1 needs gamma before any code, so
// it is two passes over W: pass A (fp64 partial sums of |W|) and the code
// pass (gamma from the partials, codes packed 4 per byte). bl_quantize runs
// pass A (quant_pass_a_kernel), then one grid (quant_phase2_kernel) whose
// token blocks -- S2, independent of S1 -- start beside pass A and whose
// code-pass blocks wait for it; bl_quantize_weight and bl_quantize_act launch
// the same arithmetic separately.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kQuantThreads = 256;
// Upper bound on pass-A blocks: two 256-thread blocks per SM on a 148-SM
// B200. A fixed constant, so the fp64 reduction tree is the same on any GPU.
constexpr int kMaxPartials = 296;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// A "group" is 16 consecutive elements of the flattened [N,K] tensor. Its 16
// codes pack into one 32-bit word: element i of the group sits at bits 2i..2i+1
// (little-endian, so byte j of the word holds elements 4j..4j+3, LSB first).
template <bool kF32>
struct Group {
  static constexpr int kVecs = kF32 ? 4 : 2;  // uint4 per 16 elements
  uint4 v[kVecs];

  __device__ __forceinline__ void load(const uint4* __restrict__ base, int64_t g) {
#pragma unroll
    for (int i = 0; i < kVecs; ++i) v[i] = __ldg(base + g * kVecs + i);
  }

  // Element i (0..15) as fp32.
  __device__ __forceinline__ float elem(int i) const {
    if constexpr (kF32) {
      const uint4& q = v[i >> 2];
      const uint32_t w = (i & 3) == 0 ? q.x : (i & 3) == 1 ? q.y : (i & 3) == 2 ? q.z : q.w;
      return __uint_as_float(w);
    } else {
      const uint4& q = v[i >> 3];
      const int j = (i & 7) >> 1;
      const uint32_t w = j == 0 ? q.x : j == 1 ? q.y : j == 2 ? q.z : q.w;
      return (i & 1) ? bf16_hi(w) : bf16_lo(w);
    }
  }
};

// |w| widened to fp64 exactly from its bit pattern with the sign cleared.
// Zero and normal values take integer arithmetic only (a bf16's fp64 high
// word is b * 2^13 + 0x38000000: exponent re-bias 127 -> 1023; an fp32's is
// (b >> 3) + 0x38000000 with low word b << 29), leaving the conversion pipe
// free. Subnormals (nonzero with a zero exponent field) are converted with
// the conversion instruction on a separate, rarely taken path. Inputs are
// finite.
__device__ __forceinline__ uint32_t abs_bits(float x) { return __float_as_uint(x) & 0x7FFFFFFFu; }

__device__ __forceinline__ double normal_abs_to_f64(uint32_t b32) {
  if (b32 == 0) return 0.0;
  return __hiloint2double(static_cast<int>((b32 >> 3) + 0x38000000u), static_cast<int>(b32 << 29));
}

__device__ __forceinline__ bool is_subnormal(uint32_t b32) { return b32 - 1u < 0x007FFFFFu; }

// acc + sum of |element| over one group, in element order.
// bf16 groups whose 16 magnitudes all have a nonzero exponent field (no zero,
// no subnormal) take a short path: one packed 16-bit minimum per word finds
// them, and each fp64 high word is the 15-bit magnitude shifted into place
// plus the re-biased exponent offset. Other groups, and fp32 groups, take the
// per-element path below. Both give the same fp64 values in the same order.
template <bool kF32>
__device__ __forceinline__ double add_group(double acc, const Group<kF32>& a) {
  if constexpr (!kF32) {
    const uint32_t w[8] = {a.v[0].x, a.v[0].y, a.v[0].z, a.v[0].w, a.v[1].x, a.v[1].y, a.v[1].z, a.v[1].w};
    uint32_t mn = 0xFFFFFFFFu;  // per half: smallest 15-bit magnitude
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t m = w[j] & 0x7FFF7FFFu;
      asm("min.u16x2 %0, %0, %1;" : "+r"(mn) : "r"(m));
    }
    if (min(mn << 16, mn & 0xFFFF0000u) >= 0x00800000u) {
      // element 2j is the low half of word j, element 2j + 1 the high half
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        acc = __dadd_rn(acc, __hiloint2double(static_cast<int>(((w[j] & 0x7FFFu) << 13) + 0x38000000u), 0));
        acc = __dadd_rn(acc, __hiloint2double(static_cast<int>(((w[j] & 0x7FFF0000u) >> 3) + 0x38000000u), 0));
      }
      return acc;
    }
  }
  bool sub = false;
#pragma unroll
  for (int i = 0; i < 16; ++i) sub |= is_subnormal(abs_bits(a.elem(i)));
  if (sub) {
#pragma unroll
    for (int i = 0; i < 16; ++i) acc = __dadd_rn(acc, static_cast<double>(__uint_as_float(abs_bits(a.elem(i)))));
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) acc = __dadd_rn(acc, normal_abs_to_f64(abs_bits(a.elem(i))));
  }
  return acc;
}


// ---------------------------------------------------------------- S1 pass A
// partials[b] = sum of |w| over block b's contiguous range of groups, fp64.
// Each thread keeps four accumulators (group u of every four goes to
// accumulator u; leftover groups to accumulator 0), adds them as
// (a0 + a1) + (a2 + a3), then a fixed shuffle/smem tree. The groups are
// loaded kLoad at a time (4 or 2), the next batch while the current one is
// summed; the order of the additions does not depend on kLoad.
template <bool kF32, int kLoad>
__device__ __forceinline__ void absmean_block(const uint4* __restrict__ W, int64_t ngroups, int64_t per_block,
                                              int64_t block, double* __restrict__ partials) {
  static_assert(kLoad == 2 || kLoad == 4, "batches split a quad of groups");
  constexpr int T = kQuantThreads;
  constexpr int kPerQuad = 4 / kLoad;
  const int64_t g0 = block * per_block;
  const int64_t g1 = min(g0 + per_block, ngroups);
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  const int64_t gt = g0 + threadIdx.x;
  // full quads of this thread: groups gt + (4q + u) T, u = 0..3, all < g1
  const int64_t nquads = gt + 3 * T < g1 ? (g1 - 1 - 3 * T - gt) / (4 * T) + 1 : 0;
  const int64_t nbatch = nquads * kPerQuad;
  if (nbatch > 0) {
    Group<kF32> a[kLoad];
#pragma unroll
    for (int v = 0; v < kLoad; ++v) a[v].load(W, gt + v * T);
    for (int64_t b = 0; b < nbatch; ++b) {
      const int64_t bn = b + 1;
      Group<kF32> nxt[kLoad];
      if (bn < nbatch) {
        const int64_t base = gt + (bn / kPerQuad) * 4 * T + (bn % kPerQuad) * kLoad * T;
#pragma unroll
        for (int v = 0; v < kLoad; ++v) nxt[v].load(W, base + v * T);
      }
      const int u0 = static_cast<int>(b % kPerQuad) * kLoad;
#pragma unroll
      for (int v = 0; v < kLoad; ++v) {
        if constexpr (kLoad == 4) {
          acc[v] = add_group(acc[v], a[v]);
        } else {
          // accumulator u0 + v (u0 is 0 or 2)
          if (u0 == 0) acc[v] = add_group(acc[v], a[v]);
          else acc[2 + v] = add_group(acc[2 + v], a[v]);
        }
      }
#pragma unroll
      for (int v = 0; v < kLoad; ++v) a[v] = nxt[v];
    }
  }
  for (int64_t g = gt + nquads * 4 * T; g < g1; g += T) {
    Group<kF32> a;
    a.load(W, g);
    acc[0] = add_group(acc[0], a);
  }
  double t = __dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) t = __dadd_rn(t, __shfl_xor_sync(0xffffffffu, t, off));
  __shared__ double warp_sums[kQuantThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = t;
  __syncthreads();
  if (threadIdx.x == 0) {
    double sum = 0.0;
#pragma unroll
    for (int w = 0; w < kQuantThreads / 32; ++w) sum = __dadd_rn(sum, warp_sums[w]);
    partials[block] = sum;
  }
}

template <bool kF32>
__global__ void __launch_bounds__(kQuantThreads) absmean_partials_kernel(const uint4* __restrict__ W,
                                                                         int64_t ngroups, int64_t per_block,
                                                                         double* __restrict__ partials) {
  pdl_wait_primary();       // W may come from the previous kernel (e.g. an optimizer step)
  pdl_launch_dependents();  // the code pass may start loading W while this pass finishes
  absmean_block<kF32, 4>(W, ngroups, per_block, blockIdx.x, partials);
}

// ---------------------------------------------------------------- S1 code pass
// Launched as a programmatic dependent of pass A: each thread first loads its
// first groups of W (pass A only started after W's producer finished, and it
// does not write W), then waits for pass A,
// then every block reduces the partials in the same fixed order (so all
// blocks hold the same gamma) and writes the codes of its range of groups.
//
// Code rule: code = clamp(rint_half_even(fp32(w / gamma)), -1, 1) is nonzero
// exactly when fp32(|w| / gamma) > 0.5, i.e. when the exact quotient exceeds
// 0.5 + 2^-25 (the midpoint between 0.5 and the next float, which rounds to
// the even 0.5). With T = gamma * (0.5 + 2^-25) computed exactly in fp64 and
// thr the largest float <= T, that is |w| > thr: one compare, no division.
template <bool kF32>
__device__ __forceinline__ uint32_t pack_group(const Group<kF32>& a, float thr) {
  if constexpr (!kF32) {
    // bf16: for a 15-bit magnitude b (the bf16 bits with the sign cleared)
    // and thr > 0, |w| > thr <=> (b << 16) > bits(thr) <=> b > bits(thr) >> 16,
    // so both halves of a word are compared with one subtraction: per half,
    // 0x8000 + tb - b keeps bit 15 clear exactly when b > tb (no borrow
    // crosses the halves since b <= 0x7FFF). Field bit 0 = nonzero, bit 1 =
    // nonzero and negative.
    const uint32_t tb = __float_as_uint(thr) >> 16;
    const uint32_t bias = (tb | (tb << 16)) + 0x80008000u;
    const uint32_t w[8] = {a.v[0].x, a.v[0].y, a.v[0].z, a.v[0].w, a.v[1].x, a.v[1].y, a.v[1].z, a.v[1].w};
    uint32_t acc[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t nz = ~(bias - (w[j] & 0x7FFF7FFFu)) & 0x80008000u;  // bits 15, 31
      const uint32_t nn = nz & w[j];
      // word j of a four-word half: low element's field to bits 4j', 4j'+1,
      // high element's to 16 + 4j', 17 + 4j' (j' = j % 4)
      const int sh = 4 * (j & 3);
      acc[j >> 2] |= (nz >> (15 - sh)) | (nn >> (14 - sh));
    }
    // high elements' fields from bits 16.. down to 4j' + 2
    const uint32_t lo = (acc[0] & 0x3333u) | ((acc[0] >> 14) & 0xCCCCu);
    const uint32_t hi = (acc[1] & 0x3333u) | ((acc[1] >> 14) & 0xCCCCu);
    return lo | (hi << 16);
  } else {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float w = a.elem(i);
      const uint32_t nz = fabsf(w) > thr ? 1u : 0u;
      const uint32_t neg = __float_as_uint(w) >> 31;
      word |= (nz * (1u | (neg << 1))) << (2 * i);  // 00 = 0, 01 = +1, 11 = -1
    }
    return word;
  }
}

// Code-pass block `block` of `nblocks`: threads stride over the groups
// (consecutive threads, consecutive groups), two groups per batch, the next
// batch loaded while the current one is packed; the first batch is loaded
// before the wait for pass A.
template <bool kF32>
__device__ __forceinline__ void code_pass_block(const uint4* __restrict__ W, int64_t ngroups,
                                                const double* __restrict__ partials, int nparts, int64_t numel,
                                                uint32_t* __restrict__ packed, float* __restrict__ gamma_out,
                                                int64_t block, int64_t nblocks) {
  const int64_t stride = nblocks * kQuantThreads;
  int64_t g = block * kQuantThreads + threadIdx.x;
  Group<kF32> a[2];
#pragma unroll
  for (int u = 0; u < 2; ++u)
    if (g + u * stride < ngroups) a[u].load(W, g + u * stride);

  pdl_wait_primary();  // pass A has finished and its partial sums are visible
  pdl_launch_dependents();

  __shared__ double red[kQuantThreads / 32];
  __shared__ float s_thr;
  double t = 0.0;
  for (int i = threadIdx.x; i < nparts; i += kQuantThreads) t = __dadd_rn(t, partials[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) t = __dadd_rn(t, __shfl_xor_sync(0xffffffffu, t, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = t;
  __syncthreads();
  if (threadIdx.x == 0) {
    double sum = 0.0;
#pragma unroll
    for (int w = 0; w < kQuantThreads / 32; ++w) sum = __dadd_rn(sum, red[w]);
    const double mean = __ddiv_rn(sum, static_cast<double>(numel));
    const float gamma = fmaxf(__double2float_rn(mean), 1e-5f);
    s_thr = __double2float_rd(__dmul_rn(static_cast<double>(gamma), 0.5 + 0x1p-25));
    if (block == 0) *gamma_out = gamma;
  }
  __syncthreads();
  const float thr = s_thr;

  for (; g < ngroups; g += 2 * stride) {
    const int64_t gn = g + 2 * stride;
    Group<kF32> b[2];
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (gn + u * stride < ngroups) b[u].load(W, gn + u * stride);
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (g + u * stride < ngroups) packed[g + u * stride] = pack_group(a[u], thr);
#pragma unroll
    for (int u = 0; u < 2; ++u) a[u] = b[u];
  }
}

template <bool kF32>
__global__ void __launch_bounds__(kQuantThreads, kF32 ? 2 : 4) ternarize_pack_kernel(const uint4* __restrict__ W,
                                                                          int64_t ngroups,
                                                                          const double* __restrict__ partials,
                                                                          int nparts, int64_t numel,
                                                                          uint32_t* __restrict__ packed,
                                                                          float* __restrict__ gamma_out) {
  code_pass_block<kF32>(W, ngroups, partials, nparts, numel, packed, gamma_out, blockIdx.x, gridDim.x);
}

// ---------------------------------------------------------------- S2
// One warp per token. The row stays in registers between the absmax and the
// quantisation: VPL = ceil(K / 256) 16-byte vectors per lane (K <= 8192).
//
// q = rint_half_even(fp32(x * inv)) uses the 1.5 * 2^23 shifter: adding it
// rounds |x * inv| <= 127.0001 to an integer (ties to even), and the low byte
// of the sum's bit pattern is that integer in two's complement. |q| <= 127
// holds without a clamp because |x| <= a and inv = fp32(127 / a).
__device__ __forceinline__ uint32_t quant4(float a, float b, float c, float d, float inv) {
  const float kShift = 12582912.0f;  // 1.5 * 2^23
  const uint32_t qa = __float_as_uint(__fadd_rn(__fmul_rn(a, inv), kShift));
  const uint32_t qb = __float_as_uint(__fadd_rn(__fmul_rn(b, inv), kShift));
  const uint32_t qc = __float_as_uint(__fadd_rn(__fmul_rn(c, inv), kShift));
  const uint32_t qd = __float_as_uint(__fadd_rn(__fmul_rn(d, inv), kShift));
  const uint32_t ab = __byte_perm(qa, qb, 0x0040);
  const uint32_t cd = __byte_perm(qc, qd, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

__device__ __forceinline__ uint2 quant8(const uint4& v, float inv) {
  uint2 r;
  r.x = quant4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y), inv);
  r.y = quant4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w), inv);
  return r;
}

// Running maximum of the 15-bit magnitudes of 8 bf16 values, per 16-bit
// half of `m`. For finite values the magnitude bit patterns order like the
// magnitudes, so this is |x|'s maximum without unpacking to fp32 (which also
// keeps a row's unpacked values from staying live until the quantisation).
__device__ __forceinline__ uint32_t max_mag_u16x2(uint32_t m, uint32_t w) {
  asm("max.u16x2 %0, %0, %1;" : "+r"(m) : "r"(w & 0x7FFF7FFFu));
  return m;
}

__device__ __forceinline__ uint32_t absmax8(const uint4& v, uint32_t m) {
  m = max_mag_u16x2(m, v.x);
  m = max_mag_u16x2(m, v.y);
  m = max_mag_u16x2(m, v.z);
  m = max_mag_u16x2(m, v.w);
  return m;
}

// The larger of the two halves as an fp32 value.
__device__ __forceinline__ float absmax_value(uint32_t m) { return __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16); }

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  return m;
}

constexpr int kActRowsPerBlock = 4;

// VPL = ceil(nv / 32), so only the last vector of a lane can lie past the row.
template <int VPL>
__device__ __forceinline__ void load_row(const uint4* __restrict__ row, int nv, int lane, uint4 (&v)[VPL]) {
  const uint4* p = row + lane;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    v[i] = (i < VPL - 1 || lane + 32 * i < nv) ? __ldg(p + 32 * i) : make_uint4(0u, 0u, 0u, 0u);
}

template <int VPL>
__device__ __forceinline__ void quant_row(const uint4 (&v)[VPL], int nv, int lane, int64_t m,
                                          int8_t* __restrict__ xq, float* __restrict__ sx) {
  uint32_t mx = 0u;
#pragma unroll
  for (int i = 0; i < VPL; ++i) mx = absmax8(v[i], mx);
  const float a = fmaxf(warp_max(absmax_value(mx)), 1e-5f);
  const float inv = __fdiv_rn(127.0f, a);
  if (lane == 0) sx[m] = __fdiv_rn(a, 127.0f);
  uint2* out = reinterpret_cast<uint2*>(xq + m * static_cast<int64_t>(nv) * 8) + lane;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if (i < VPL - 1 || lane + 32 * i < nv) out[32 * i] = quant8(v[i], inv);
}

// Warps stride over rows (first row m, then m + stride, ...); with short rows
// (kPrefetch) the next row's loads are issued before the current row is
// quantised.
template <int VPL, bool kPrefetch>
__device__ __forceinline__ void act_rows(const uint4* __restrict__ x, int64_t M, int nv, int8_t* __restrict__ xq,
                                         float* __restrict__ sx, int64_t m, int64_t stride) {
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  uint4 v[VPL];
  load_row<VPL>(x + m * nv, nv, lane, v);
  while (true) {
    const int64_t mn = m + stride;
    if constexpr (kPrefetch) {
      uint4 vn[VPL];
      if (mn < M) load_row<VPL>(x + mn * nv, nv, lane, vn);
      quant_row<VPL>(v, nv, lane, m, xq, sx);
      if (mn >= M) break;
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = vn[i];
    } else {
      quant_row<VPL>(v, nv, lane, m, xq, sx);
      if (mn >= M) break;
      load_row<VPL>(x + mn * nv, nv, lane, v);
    }
    m = mn;
  }
}

template <int VPL, bool kPrefetch>
__global__ void __launch_bounds__(32 * kActRowsPerBlock) act_quant_kernel(const uint4* __restrict__ x, int64_t M,
                                                                          int nv, int8_t* __restrict__ xq,
                                                                          float* __restrict__ sx) {
  pdl_wait_primary();
  pdl_launch_dependents();
  act_rows<VPL, kPrefetch>(x, M, nv, xq, sx,
                           static_cast<int64_t>(blockIdx.x) * kActRowsPerBlock + (threadIdx.x >> 5),
                           static_cast<int64_t>(gridDim.x) * kActRowsPerBlock);
}

// One row per warp, read twice: absmax, then quantisation (the second read
// mostly hits L1/L2).
__device__ __forceinline__ void act_rows_two_pass(const uint4* __restrict__ x, int64_t M, int nv,
                                                  int8_t* __restrict__ xq, float* __restrict__ sx, int64_t m,
                                                  int64_t stride) {
  const int lane = threadIdx.x & 31;
  for (; m < M; m += stride) {
    const uint4* row = x + m * nv;
    uint32_t mx = 0u;
#pragma unroll 4
    for (int j = lane; j < nv; j += 32) mx = absmax8(__ldg(row + j), mx);
    const float a = fmaxf(warp_max(absmax_value(mx)), 1e-5f);
    const float inv = __fdiv_rn(127.0f, a);
    if (lane == 0) sx[m] = __fdiv_rn(a, 127.0f);
    uint2* out = reinterpret_cast<uint2*>(xq + m * static_cast<int64_t>(nv) * 8);
#pragma unroll 4
    for (int j = lane; j < nv; j += 32) out[j] = quant8(__ldg(row + j), inv);
  }
}

// bl_quantize, launch 1: pass A alone (two groups loaded per batch, so that
// it fits beside two more 256-thread blocks on an SM).
template <bool kF32>
__global__ void __launch_bounds__(kQuantThreads, kF32 ? 2 : 4) quant_pass_a_kernel(const uint4* __restrict__ W,
                                                                        int64_t ngroups, int64_t per_block,
                                                                        double* __restrict__ partials) {
  pdl_wait_primary();
  pdl_launch_dependents();  // launch 2 may start beside this pass
  absmean_block<kF32, 2>(W, ngroups, per_block, blockIdx.x, partials);
}

// bl_quantize, launch 2 (a programmatic dependent of launch 1): blocks
// 0 .. act_blocks-1 quantise tokens (S2); the rest run the code pass. The token
// blocks do not wait for launch 1: x was complete before launch 1 passed its
// own dependency wait (and launch 2 only starts after that point), and launch
// 1 neither reads xq / s_x nor writes x. So they run beside pass A, and the
// code-pass blocks -- which do wait -- follow; since they wait, this grid
// still completes only after launch 1 has. Rows of up to 2560 elements stay
// in registers (VPL <= 10, the most that fits the 64 registers a thread has at
// four blocks per SM), longer ones are read twice (VPL = 0).
constexpr int kFusedMaxVpl = 10;

template <bool kF32, int VPL>
__global__ void __launch_bounds__(kQuantThreads, kF32 ? 2 : 4) quant_phase2_kernel(
    const uint4* __restrict__ W, int64_t ngroups, const double* __restrict__ partials, int nparts, int64_t numel,
    uint32_t* __restrict__ packed, float* __restrict__ gamma_out, const uint4* __restrict__ x, int64_t M, int nv,
    int8_t* __restrict__ xq, float* __restrict__ sx, int act_blocks) {
  if (static_cast<int>(blockIdx.x) < act_blocks) {
    pdl_launch_dependents();
    constexpr int kWarps = kQuantThreads / 32;
    const int64_t m = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const int64_t stride = static_cast<int64_t>(act_blocks) * kWarps;
    if constexpr (VPL > 0)
      act_rows<VPL, false>(x, M, nv, xq, sx, m, stride);
    else
      act_rows_two_pass(x, M, nv, xq, sx, m, stride);
    return;
  }
  code_pass_block<kF32>(W, ngroups, partials, nparts, numel, packed, gamma_out, blockIdx.x - act_blocks,
                        gridDim.x - act_blocks);
}

// Rows longer than 8192 elements: absmax pass, then a second read (from L2).
__global__ void __launch_bounds__(32 * kActRowsPerBlock) act_quant_long_kernel(const uint4* __restrict__ x,
                                                                               int64_t M, int nv,
                                                                               int8_t* __restrict__ xq,
                                                                               float* __restrict__ sx) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t m = static_cast<int64_t>(blockIdx.x) * kActRowsPerBlock + (threadIdx.x >> 5);
  if (m >= M) return;
  const uint4* row = x + m * nv;
  uint32_t mx = 0u;
  for (int j = lane; j < nv; j += 32) mx = absmax8(__ldg(row + j), mx);
  const float a = fmaxf(warp_max(absmax_value(mx)), 1e-5f);
  const float inv = __fdiv_rn(127.0f, a);
  if (lane == 0) sx[m] = __fdiv_rn(a, 127.0f);
  uint2* out = reinterpret_cast<uint2*>(xq + m * static_cast<int64_t>(nv) * 8);
  for (int j = lane; j < nv; j += 32) out[j] = quant8(__ldg(row + j), inv);
}

}  // namespace

// Fixed device scratch for bl_quantize_weight_noalloc: room for the largest
// number of fp64 partial sums pass A ever writes (kMaxPartials), 2368 bytes.
// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) double g_noalloc_partials[kMaxPartials];

// Blocks of the code pass: four per SM, fewer for small tensors.
static unsigned code_pass_blocks(int64_t ngroups) {
  const int64_t want = (ngroups + kQuantThreads - 1) / kQuantThreads;
  const int64_t cap = static_cast<int64_t>(4) * device_sm_count();
  return static_cast<unsigned>(want < cap ? want : cap);
}

int weight_partials_count(int64_t numel) {
  const int64_t ngroups = numel / 16;
  const int64_t want = (ngroups + kQuantThreads - 1) / kQuantThreads;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kMaxPartials, want)));
}

template <bool kF32>
static cudaError_t launch_weight_passes(const uint4* w, int64_t ngroups, int64_t per_block, int nparts, int64_t numel,
                                        uint32_t* out, float* gamma, double* partials, cudaStream_t s) {
  cudaError_t e = launch_pdl(absmean_partials_kernel<kF32>, dim3(nparts), dim3(kQuantThreads), 0, s, w, ngroups,
                             per_block, partials);
  if (e != cudaSuccess) return e;
  return launch_pdl(ternarize_pack_kernel<kF32>, dim3(code_pass_blocks(ngroups)), dim3(kQuantThreads), 0, s, w,
                    ngroups, static_cast<const double*>(partials), nparts, numel, out, gamma);
}

cudaError_t launch_quantize_weight(const void* W, int w_is_f32, int64_t N, int64_t K, uint8_t* packed,
                                   float* gamma, double* partials, cudaStream_t s) {
  const int64_t numel = N * K;  // multiple of 32
  const int64_t ngroups = numel / 16;
  const int nparts = weight_partials_count(numel);
  const int64_t per_block = (ngroups + nparts - 1) / nparts;
  const uint4* w = static_cast<const uint4*>(W);
  uint32_t* out = reinterpret_cast<uint32_t*>(packed);
  cudaError_t e = w_is_f32 ? launch_weight_passes<true>(w, ngroups, per_block, nparts, numel, out, gamma, partials, s)
                           : launch_weight_passes<false>(w, ngroups, per_block, nparts, numel, out, gamma, partials, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

size_t noalloc_scratch_bytes() { return sizeof(g_noalloc_partials); }

// Device address of g_noalloc_partials on the current device. Host code only
// holds a stand-in for the array's name, so the address is looked up with the
// device current, on every call: a cached address would go stale if the
// caller reset the device and the module were loaded again elsewhere. The
// first lookup on a device loads the module there (so it belongs before any
// stream capture); later ones are host-side table lookups.
static cudaError_t noalloc_scratch_ptr(double** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_partials);
  if (e != cudaSuccess) return e;
  *out = static_cast<double*>(p);
  return cudaSuccess;
}

cudaError_t launch_quantize_weight_noalloc(const void* W, int w_is_f32, int64_t N, int64_t K, uint8_t* packed,
                                           float* gamma, cudaStream_t s) {
  if (static_cast<size_t>(weight_partials_count(N * K)) * sizeof(double) > sizeof(g_noalloc_partials))
    return cudaErrorInvalidValue;
  double* scratch = nullptr;
  const cudaError_t e = noalloc_scratch_ptr(&scratch);
  if (e != cudaSuccess) return e;
  return launch_quantize_weight(W, w_is_f32, N, K, packed, gamma, scratch, s);
}

template <int VPL>
static void launch_act(const uint4* xv, int64_t M, int nv, int8_t* xq, float* sx, cudaStream_t s) {
  constexpr bool kPrefetch = VPL <= 12;
  static int per_sm[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  int occ = (dev >= 0 && dev < 64) ? per_sm[dev] : 0;
  if (!occ) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, act_quant_kernel<VPL, kPrefetch>,
                                                      32 * kActRowsPerBlock, 0) != cudaSuccess || occ < 1)
      occ = 1;
    cudaGetLastError();
    if (dev >= 0 && dev < 64) per_sm[dev] = occ;
  }
  const int64_t want = (M + kActRowsPerBlock - 1) / kActRowsPerBlock;
  const int64_t cap = static_cast<int64_t>(occ) * device_sm_count();
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  launch_pdl(act_quant_kernel<VPL, kPrefetch>, dim3(grid), dim3(32 * kActRowsPerBlock), 0, s, xv, M, nv, xq, sx);
}

// bl_quantize: pass A (quant_pass_a_kernel), then the token blocks and the
// code pass in one grid (quant_phase2_kernel). Rows longer than 8192
// elements take the separate launches.
template <bool kF32, int VPL>
static cudaError_t launch_quantize_fused(const uint4* w, int64_t N, int64_t K, const uint4* xv, int64_t M,
                                         uint32_t* packed, float* gamma, double* partials, int8_t* xq, float* sx,
                                         cudaStream_t s) {
  const int64_t numel = N * K;
  const int64_t ngroups = numel / 16;
  const int nparts = weight_partials_count(numel);
  const int64_t per_block = (ngroups + nparts - 1) / nparts;
  // token blocks: two per SM beside pass A, no more than the rows need
  const int64_t rows_blocks = (M + kQuantThreads / 32 - 1) / (kQuantThreads / 32);
  const int64_t act_blocks = std::min<int64_t>(static_cast<int64_t>(2) * device_sm_count(), rows_blocks);
  const int64_t code_blocks = code_pass_blocks(ngroups);
  const int nv = static_cast<int>(K / 8);
  cudaError_t e = launch_pdl(quant_pass_a_kernel<kF32>, dim3(static_cast<unsigned>(nparts)), dim3(kQuantThreads), 0,
                             s, w, ngroups, per_block, partials);
  if (e != cudaSuccess) return e;
  return launch_pdl(quant_phase2_kernel<kF32, VPL>, dim3(static_cast<unsigned>(act_blocks + code_blocks)),
                    dim3(kQuantThreads), 0, s, w, ngroups, static_cast<const double*>(partials), nparts, numel, packed,
                    gamma, xv, M, nv, xq, sx, static_cast<int>(act_blocks));
}

cudaError_t launch_quantize_act(const void* x, int64_t M, int64_t K, int8_t* xq, float* sx, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  const int nv = static_cast<int>(K / 8);
  const uint4* xv = static_cast<const uint4*>(x);
  const int per_lane = (nv + 31) / 32;
  switch (per_lane) {
#define BL_ACT_CASE(n) \
  case n:              \
    launch_act<n>(xv, M, nv, xq, sx, s); \
    break;
    BL_ACT_CASE(1) BL_ACT_CASE(2) BL_ACT_CASE(3) BL_ACT_CASE(4) BL_ACT_CASE(5) BL_ACT_CASE(6) BL_ACT_CASE(7)
    BL_ACT_CASE(8) BL_ACT_CASE(9) BL_ACT_CASE(10) BL_ACT_CASE(11) BL_ACT_CASE(12) BL_ACT_CASE(13)
    BL_ACT_CASE(14) BL_ACT_CASE(15) BL_ACT_CASE(16) BL_ACT_CASE(17) BL_ACT_CASE(18) BL_ACT_CASE(19)
    BL_ACT_CASE(20) BL_ACT_CASE(21) BL_ACT_CASE(22) BL_ACT_CASE(23) BL_ACT_CASE(24) BL_ACT_CASE(25)
    BL_ACT_CASE(26) BL_ACT_CASE(27) BL_ACT_CASE(28) BL_ACT_CASE(29) BL_ACT_CASE(30) BL_ACT_CASE(31)
    BL_ACT_CASE(32)
#undef BL_ACT_CASE
    default: {
      const unsigned grid = static_cast<unsigned>((M + kActRowsPerBlock - 1) / kActRowsPerBlock);
      launch_pdl(act_quant_long_kernel, dim3(grid), dim3(32 * kActRowsPerBlock), 0, s, xv, M, nv, xq, sx);
    }
  }
  return cudaGetLastError();
}

cudaError_t launch_quantize(const void* W, int w_is_f32, int64_t N, int64_t K, const void* x, int64_t M,
                            uint8_t* packed, float* gamma, double* partials, int8_t* xq, float* sx, cudaStream_t s) {
  const int nv = static_cast<int>(K / 8);
  const int per_lane = (nv + 31) / 32;
  if (M == 0 || per_lane > 32) {
    cudaError_t e = launch_quantize_weight(W, w_is_f32, N, K, packed, gamma, partials, s);
    if (e != cudaSuccess) return e;
    return launch_quantize_act(x, M, K, xq, sx, s);
  }
  const uint4* w = static_cast<const uint4*>(W);
  const uint4* xv = static_cast<const uint4*>(x);
  uint32_t* out = reinterpret_cast<uint32_t*>(packed);
  cudaError_t e = cudaSuccess;
  switch (per_lane <= kFusedMaxVpl ? per_lane : 0) {
#define BL_Q_CASE(n)                                                                                  \
  case n:                                                                                             \
    e = w_is_f32 ? launch_quantize_fused<true, n>(w, N, K, xv, M, out, gamma, partials, xq, sx, s)    \
                 : launch_quantize_fused<false, n>(w, N, K, xv, M, out, gamma, partials, xq, sx, s); \
    break;
    BL_Q_CASE(0) BL_Q_CASE(1) BL_Q_CASE(2) BL_Q_CASE(3) BL_Q_CASE(4) BL_Q_CASE(5) BL_Q_CASE(6)
    BL_Q_CASE(7) BL_Q_CASE(8) BL_Q_CASE(9) BL_Q_CASE(10)
#undef BL_Q_CASE
    default:
      break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bl
