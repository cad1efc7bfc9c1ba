// S1 and S2 of the BitLinear hot path on sm_100a: absmean ternarisation with
// 2-bit packing, and per-token absmax INT8 activation quantisation.
//
// S1 needs the mean |W| of the whole tensor before any code can be written,
// and S2 is independent of it. One persistent launch does both with W read
// from HBM once: each CTA (at most one per SM, all resident together) copies
// its contiguous slice of W into shared memory with bulk asynchronous copies
// (TMA, issued all at once at entry), sums |W| of the slice in fp64 as the
// copies land, publishes the partial sum and meets the other CTAs at a
// grid-wide barrier (a counter in the workspace, bounded wait); then every
// CTA forms gamma from all partial sums in one fixed order and writes the
// codes of its slice from shared memory. The part of a slice that does not
// fit in shared memory is summed from registers and read again (from L2) for
// its codes. Other warps of the same CTAs quantise the tokens (S2) while the
// slice copies are in flight. A one-thread launch before it clears the
// workspace's counters, so the caller's workspace needs no initialisation.
//
// gamma = max(fp32(fp64(fp64(S) / numel)), 1e-5) with S = sum |W| (exactly
// rounded to fp64, "1BitTraining.md" weight_quant / "bitlinear.py"
// ternary_quantize with the fp64 accumulation the reading fixes). The fp64
// tree sum carries a bounded rounding error, so gamma is formed at both ends
// of an enclosure of S; as the chain of roundings is monotone, when the two
// agree that value is the exact gamma (all but about one tensor in 10^5).
// Otherwise the CTAs compute S exactly -- integer sums of the significands
// per exponent field, combined as one wide integer and rounded once -- so
// gamma never depends on the reduction order or on the GPU's SM count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------- S1 geometry
constexpr int kQThreads = 512;                 // 16 warps per CTA
constexpr int kQWarps = kQThreads / 32;
constexpr int kChunkBytes = 16384;             // one bulk copy of the slice
constexpr int kMaxOnchipBytes = 220 * 1024;    // slice bytes held in shared memory
constexpr int kMaxChunks = kMaxOnchipBytes / kChunkBytes + 1;

// Workspace (each part on its own 128-byte lines): at 0 the arrivals at the
// partial-sum and at the exact-sum barrier (u32 each); at 128 the gamma flag
// (1: gamma published, 2: the exact sum is needed) and gamma's bits; at 256
// the next token row to claim; at 512 one fp64 partial sum per CTA; then 256
// uint64 exact-sum bins (one per exponent field).
constexpr size_t kWsArrive = 0;
constexpr size_t kWsFlag = 128;
constexpr size_t kWsRows = 256;
constexpr size_t kWsPartials = 512;
constexpr size_t kWsBins = kWsPartials + 8 * static_cast<size_t>(kMaxQuantCtas);
constexpr size_t kWsBytes = kWsBins + 8 * 256;

// ---------------------------------------------------------------- |W| in fp64
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

// Exact-sum bins: bin e collects the integer significands (hidden bit
// included; none for e = 0) of the elements whose exponent field is e, so
// that sum |W| = sum_e bin[e] * 2^(max(e, 1) - 127 - p), p = 7 (bf16) or 23.
template <bool kF32>
__device__ __forceinline__ void bin_abs(unsigned long long* bins, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if constexpr (kF32) {
      const uint32_t b = w[j] & 0x7FFFFFFFu, e = b >> 23, m = (b & 0x7FFFFFu) | (e ? 0x800000u : 0u);
      if (m) atomicAdd(&bins[e], static_cast<unsigned long long>(m));
    } else {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t b = (w[j] >> (16 * h)) & 0x7FFFu, e = b >> 7, m = (b & 0x7Fu) | (e ? 0x80u : 0u);
        if (m) atomicAdd(&bins[e], static_cast<unsigned long long>(m));
      }
    }
  }
}

// S = sum_e bins[e] * 2^(max(e, 1) - 127 - p), rounded once to fp64 (to
// nearest, ties to even). The bins are added as one unsigned integer of six
// 64-bit limbs, V = sum_e bins[e] << (max(e, 1) - 1), so S = V * 2^(-126 - p);
// V's top 53 bits are then rounded with the round and sticky bits below.
__device__ double exact_sum_from_bins(const unsigned long long* bins, int p) {
  unsigned long long limb[6] = {0, 0, 0, 0, 0, 0};
  for (int e = 0; e < 255; ++e) {
    const unsigned long long v = __ldcg(bins + e);
    if (!v) continue;
    const int sh = (e > 0 ? e : 1) - 1, q = sh >> 6, r = sh & 63;
    const unsigned long long add[2] = {v << r, r ? (v >> (64 - r)) : 0ull};
    unsigned long long carry = 0;
    for (int i = q; i < 6; ++i) {
      const unsigned long long a = (i - q) < 2 ? add[i - q] : 0ull;
      const unsigned long long s1 = limb[i] + a;
      const unsigned long long c1 = s1 < a ? 1ull : 0ull;
      const unsigned long long s2 = s1 + carry;
      const unsigned long long c2 = s2 < carry ? 1ull : 0ull;
      limb[i] = s2;
      carry = c1 + c2;
      if (i - q >= 1 && !carry) break;
    }
  }
  int top = -1;
  for (int i = 5; i >= 0 && top < 0; --i)
    if (limb[i]) top = 64 * i + 63 - __clzll(static_cast<long long>(limb[i]));
  if (top < 0) return 0.0;
  auto bit = [&](int pos) -> unsigned long long { return pos < 0 ? 0ull : (limb[pos >> 6] >> (pos & 63)) & 1ull; };
  unsigned long long m = 0;
  int exp2 = -126 - p;  // S = m * 2^exp2 after the loop below
  if (top <= 52) {
    m = limb[0];
  } else {
    const int lo = top - 52;
    for (int pos = top; pos >= lo; --pos) m = (m << 1) | bit(pos);
    const unsigned long long round = bit(lo - 1);
    bool sticky = false;
    for (int pos = lo - 2; pos >= 0 && !sticky; --pos) sticky = bit(pos) != 0;
    if (round && (sticky || (m & 1ull))) {
      ++m;
      if (m >> 53) {
        m >>= 1;
        exp2 += 1;
      }
    }
    exp2 += lo;
  }
  // m < 2^53 converts exactly; the power of two is a normal fp64 (exp2 in
  // [-201, 200]), so the product is exact
  return __dmul_rn(static_cast<double>(m), __hiloint2double((exp2 + 1023) << 20, 0));
}

// gamma from S: max(fp32(fp64(S / numel)), 1e-5), rounding to nearest even.
__device__ __forceinline__ float gamma_of_sum(double S, double numel) {
  return fmaxf(__double2float_rn(__ddiv_rn(S, numel)), 1e-5f);
}

// ---------------------------------------------------------------- codes
// Code rule: code = clamp(rint_half_even(fp32(w / gamma)), -1, 1) is nonzero
// exactly when fp32(|w| / gamma) > 0.5, i.e. when the exact quotient exceeds
// 0.5 + 2^-25 (the midpoint between 0.5 and the next float, which rounds to
// the even 0.5). With T = gamma * (0.5 + 2^-25) computed exactly in fp64 and
// thr the largest float <= T, that is |w| > thr: one compare, no division.
//
// 8 bf16 of one vector -> 16 bits of codes (element i at bits 2i, 2i + 1;
// field 00 = 0, 01 = +1, 11 = -1). For a 15-bit magnitude b and thr > 0,
// |w| > thr <=> b > bits(thr) >> 16, so both halves of a word are compared by
// one subtraction: 0x8000 + tb - b keeps bit 15 clear exactly when b > tb (no
// borrow crosses the halves, b <= 0x7FFF). The low elements' fields collect at
// bits 4j, 4j + 1 and the high elements' at 16 + 4j, 17 + 4j of one word, then
// one fold moves the high ones to 4j + 2, 4j + 3 (about four operations per
// element).
__device__ __forceinline__ uint32_t codes8_bf16(const uint4& v, uint32_t bias) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t acc = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t nz = ~(bias - (w[j] & 0x7FFF7FFFu)) & 0x80008000u;  // bits 15, 31: nonzero code
    const uint32_t nn = nz & w[j];                                     // and negative
    acc |= (nz >> (15 - 4 * j)) | (nn >> (14 - 4 * j));
  }
  return (acc & 0x3333u) | ((acc >> 14) & 0xCCCCu);
}

// 4 fp32 of one vector -> 8 bits of codes.
__device__ __forceinline__ uint32_t codes4_f32(const uint4& v, float thr) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t r = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t nz = fabsf(__uint_as_float(w[j])) > thr ? 1u : 0u;
    r |= (nz | ((nz & (w[j] >> 31)) << 1)) << (2 * j);
  }
  return r;
}

// Code bits of one 16-byte vector (16 bits for bf16, 8 for fp32). `key` is
// the bf16 compare bias or the fp32 threshold's bit pattern.
template <bool kF32>
__device__ __forceinline__ uint32_t vec_codes(const uint4& v, uint32_t key) {
  if constexpr (kF32) return codes4_f32(v, __uint_as_float(key));
  else return codes8_bf16(v, key);
}

// The vectors of a warp's 32 consecutive 16-byte vectors, one per lane, are
// V = 2 (bf16) or 4 (fp32) per group: the lanes of a group OR their code bits
// together and its first lane writes the group's 32-bit word.
template <bool kF32>
__device__ __forceinline__ uint32_t gather_group_word(uint32_t bits, int lane) {
  constexpr int V = kF32 ? 4 : 2;
  constexpr int kBits = 32 / V;
  uint32_t word = bits << (kBits * (lane & (V - 1)));
#pragma unroll
  for (int off = 1; off < V; off <<= 1) word |= __shfl_down_sync(0xffffffffu, word, off);
  return word;
}

// ---------------------------------------------------------------- grid barrier
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One thread per CTA: arrive on `ctr` and wait until all `expected` CTAs have
// (the caller's stores before this call are released to the other CTAs, and
// theirs acquired). Gives up after the pipeline wait bound and records a
// timeout. Returns false on timeout.
__device__ __forceinline__ bool grid_arrive_wait(uint32_t* ctr, uint32_t expected, int* err) {
  __threadfence();
  atomicAdd(ctr, 1u);
  if (ld_acquire_u32(ctr) >= expected) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (ld_acquire_u32(ctr) >= expected) return true;
    if ((i & 15) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
      record_error(err, kDevTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- S2
// One warp per token. The row stays in registers between the absmax and the
// quantisation: VPL = ceil(K / 256) 16-byte vectors per lane.
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

// Rows longer than 8192 elements: absmax pass, then a second read (from L2).
__global__ void __launch_bounds__(32 * kActRowsPerBlock) act_quant_long_kernel(const uint4* __restrict__ x,
                                                                               int64_t M, int nv,
                                                                               int8_t* __restrict__ xq,
                                                                               float* __restrict__ sx) {
  pdl_wait_primary();
  pdl_launch_dependents();
  act_rows_two_pass(x, M, nv, xq, sx, static_cast<int64_t>(blockIdx.x) * kActRowsPerBlock + (threadIdx.x >> 5),
                    static_cast<int64_t>(gridDim.x) * kActRowsPerBlock);
}

// ---------------------------------------------------------------- S1 (+ S2): the launches
// Launch 1: clears the workspace's counters, flag and exact-sum bins. It
// waits for the kernel before it in the stream (whose work may still use
// them), and only then lets the quantisation launch start; so the
// quantisation may read W and x and write its outputs from its first
// instruction, and waits for this launch itself only before its first use of
// the workspace.
__global__ void __launch_bounds__(256) quant_reset_kernel(uint8_t* __restrict__ ws) {
  pdl_wait_primary();
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    reinterpret_cast<uint32_t*>(ws + kWsArrive)[0] = 0u;
    reinterpret_cast<uint32_t*>(ws + kWsArrive)[1] = 0u;
    reinterpret_cast<uint32_t*>(ws + kWsFlag)[0] = 0u;
    reinterpret_cast<uint32_t*>(ws + kWsRows)[0] = 0u;
  }
  reinterpret_cast<unsigned long long*>(ws + kWsBins)[threadIdx.x] = 0ull;
}

struct QuantArgs {
  const uint4* W;       // [N, K] as 16-byte vectors
  int64_t ngroups;      // N K / 16: a group's 16 codes are one 32-bit word
  int64_t per;          // groups per CTA slice (the last slices may be shorter or empty)
  int onchip_cap;       // groups of a slice held in shared memory
  double numel;
  double enc_lo, enc_hi;  // S lies in [fp64 sum * enc_lo, fp64 sum * enc_hi]
  uint32_t* packed;
  float* gamma_out;
  uint8_t* ws;
  int* err;
  const uint4* x;       // S2: x [M, K] as 16-byte vectors (M = 0: no tokens)
  int64_t M;
  int nv;               // K / 8
  int8_t* xq;
  float* sx;
};

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Lane 0 claims `n` consecutive items of a counter, the warp gets the first.
__device__ __forceinline__ uint32_t warp_claim(uint32_t* ctr, uint32_t n) {
  uint32_t m = 0;
  if ((threadIdx.x & 31) == 0) m = atomicAdd(ctr, n);
  return __shfl_sync(0xffffffffu, m, 0);
}

// Token rows m0, m0 + 1 (those below M): both rows' loads are issued before
// either is quantised. Rows longer than 2560 elements (VPL = 0) are read twice
// (absmax, then quantisation from L1/L2).
template <int VPL>
__device__ __forceinline__ void token_pair(const QuantArgs& a, int64_t m0) {
  const int lane = threadIdx.x & 31;
  if constexpr (VPL > 0) {
    uint4 v0[VPL], v1[VPL];
    load_row<VPL>(a.x + m0 * a.nv, a.nv, lane, v0);
    const bool two = m0 + 1 < a.M;
    if (two) load_row<VPL>(a.x + (m0 + 1) * a.nv, a.nv, lane, v1);
    quant_row<VPL>(v0, a.nv, lane, m0, a.xq, a.sx);
    if (two) quant_row<VPL>(v1, a.nv, lane, m0 + 1, a.xq, a.sx);
  } else {
    act_rows_two_pass(a.x, m0 + 2 < a.M ? m0 + 2 : a.M, a.nv, a.xq, a.sx, m0, 1);
  }
}

// Codes of 128 consecutive 16-byte vectors of W from shared memory (kShared)
// or global memory: lane l takes vectors l, l + 32, l + 64, l + 96 (all loads
// first, conflict-free shared loads); a group's V lanes combine their bits and
// its first lane stores the group's word.
template <bool kF32, bool kShared>
__device__ __forceinline__ void code_round(const uint4* src, int64_t base, int64_t nvec, uint32_t* out, uint32_t key,
                                           int lane) {
  constexpr int V = kF32 ? 4 : 2;
  uint4 v[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = base + lane + 32 * u;
    v[u] = make_uint4(0u, 0u, 0u, 0u);
    if (i < nvec) v[u] = kShared ? src[i] : __ldg(src + i);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = base + lane + 32 * u;
    const uint32_t word = gather_group_word<kF32>(vec_codes<kF32>(v[u], key), lane);
    if (i < nvec && (lane & (V - 1)) == 0) out[i / V] = word;
  }
}

// Launch 2, 512 threads. Every warp first sums |W| of the CTA's slice as its
// bulk copies land (W, which gates every code, is read before any token);
// thread 0 then publishes the CTA's partial sum and arrives. Warp 0 becomes the
// control warp: the last CTA to arrive forms gamma from all partial sums (in
// one fixed order) and publishes it; the others wait for it. Meanwhile the
// other warps quantise token rows claimed from a counter shared by the grid;
// once gamma is known every warp takes rounds of 128 code vectors from a
// counter of the CTA, and then token rows again until none is left. If the
// enclosure of S straddles a rounding boundary of gamma (rare), every warp
// first bins its share of the slice for the exact sum.
template <bool kF32, int VPL>
__global__ void __launch_bounds__(kQThreads, 1) quant_fused_kernel(const __grid_constant__ QuantArgs a) {
  constexpr int V = kF32 ? 4 : 2;  // 16-byte vectors per group
  constexpr int kGroupBytes = 16 * V;
  constexpr int kChunkGroups = kChunkBytes / kGroupBytes;
  constexpr int kTailRegs = 2;
  extern __shared__ __align__(128) uint4 s_w[];
  __shared__ __align__(8) uint64_t s_bar[kMaxChunks];
  __shared__ unsigned long long s_bins[256];
  __shared__ double s_red[kQWarps];
  __shared__ float s_gamma;
  __shared__ uint32_t s_key;
  __shared__ int s_state;   // 0: gamma not known, 1: known, 2: bin for the exact sum, -1: abort
  __shared__ int s_round;   // next code round of this CTA
  __shared__ int s_binned;  // warps done binning
  __shared__ int s_abort;   // a wait of this CTA gave up

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, t = threadIdx.x;
  const int64_t b = blockIdx.x;
  const uint32_t G = gridDim.x;
  const int64_t g0 = b * a.per;
  const int64_t rest = a.ngroups - g0;
  const int64_t len = rest <= 0 ? 0 : (rest < a.per ? rest : a.per);
  const int on = static_cast<int>(len < a.onchip_cap ? len : a.onchip_cap);
  const int nch = (on + kChunkGroups - 1) / kChunkGroups;
  const int64_t onv = static_cast<int64_t>(on) * V;
  const int64_t tail_v0 = (g0 + on) * V, tail_v1 = (g0 + len) * V;
  uint32_t* arrive = reinterpret_cast<uint32_t*>(a.ws + kWsArrive);  // [0] partial sums, [1] exact sum
  uint32_t* flag = reinterpret_cast<uint32_t*>(a.ws + kWsFlag);      // [0] 1 gamma / 2 exact, [1] gamma bits
  uint32_t* rows = reinterpret_cast<uint32_t*>(a.ws + kWsRows);
  double* partials = reinterpret_cast<double*>(a.ws + kWsPartials);
  unsigned long long* gbins = reinterpret_cast<unsigned long long*>(a.ws + kWsBins);

  if (t == 0) {
    s_abort = 0;
    s_state = 0;
    s_round = 0;
    s_binned = 0;
    for (int c = 0; c < nch; ++c) mbar_init(&s_bar[c], 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    // the whole on-chip slice in flight at once
    for (int c = 0; c < nch; ++c) {
      const int cg0 = c * kChunkGroups;
      const int cgn = min(kChunkGroups, on - cg0);
      mbar_arrive_expect_tx(&s_bar[c], static_cast<uint32_t>(cgn * kGroupBytes));
      bulk_copy_g2s(s_w + static_cast<int64_t>(cg0) * V, a.W + (g0 + cg0) * V, static_cast<uint32_t>(cgn * kGroupBytes),
                    &s_bar[c]);
    }
  }
  __syncthreads();

  // -------------------------------------------------- |W| of the slice, all warps
  // thread t takes vectors t, t + 512, ... of each chunk, then of the tail
  uint4 tr[kTailRegs];
#pragma unroll
  for (int u = 0; u < kTailRegs; ++u) {
    const int64_t i = tail_v0 + t + static_cast<int64_t>(u) * kQThreads;
    tr[u] = i < tail_v1 ? __ldg(a.W + i) : make_uint4(0u, 0u, 0u, 0u);
  }
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int c = 0; c < nch; ++c) {
    if (!mbar_wait(&s_bar[c], 0, &s_abort, a.err)) {
      s_abort = 1;
      break;
    }
    const int v1 = min((c + 1) * kChunkGroups, on) * V;
    int i = c * kChunkGroups * V + t;
    for (; i + 3 * kQThreads < v1; i += 4 * kQThreads) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = s_w[i + u * kQThreads];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = add_abs<kF32>(acc[u], v[u]);
    }
    if (i < v1) acc[0] = add_abs<kF32>(acc[0], s_w[i]);
    if (i + kQThreads < v1) acc[1] = add_abs<kF32>(acc[1], s_w[i + kQThreads]);
    if (i + 2 * kQThreads < v1) acc[2] = add_abs<kF32>(acc[2], s_w[i + 2 * kQThreads]);
  }
#pragma unroll
  for (int u = 0; u < kTailRegs; ++u)
    if (tail_v0 + t + static_cast<int64_t>(u) * kQThreads < tail_v1) acc[u] = add_abs<kF32>(acc[u], tr[u]);
  for (int64_t i = tail_v0 + t + static_cast<int64_t>(kTailRegs) * kQThreads; i < tail_v1; i += 4 * kQThreads) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = i + u * kQThreads < tail_v1 ? __ldg(a.W + i + u * kQThreads) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (i + u * kQThreads < tail_v1) acc[u] = add_abs<kF32>(acc[u], v[u]);
  }
  double ts = __dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ts = __dadd_rn(ts, __shfl_xor_sync(0xffffffffu, ts, off));
  if (lane == 0) s_red[warp] = ts;
  __syncthreads();
  // the next launch may be scheduled once every CTA of this grid has come
  // this far (so all of them are resident)
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------ control warp: gamma
    uint32_t last = 0;
    if (lane == 0) {
      double part = 0.0;
      for (int w = 0; w < kQWarps; ++w) part = __dadd_rn(part, s_red[w]);
      partials[b] = part;
      pdl_wait_primary();  // launch 1 has cleared the workspace
      __threadfence();
      last = atomicAdd(&arrive[0], 1u) == G - 1;
      __threadfence();  // with the atomic: acquires the other CTAs' partial sums
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    int mode = 0;
    float gamma = 0.0f;
    if (last) {
      // the partial sums in one fixed order: lane l adds l, l + 32, ..., then a
      // fixed shuffle tree (the same sum whichever CTA forms it)
      double s = 0.0;
      for (uint32_t j = lane; j < G; j += 32) s = __dadd_rn(s, __ldcg(partials + j));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
      const float glo = gamma_of_sum(__dmul_rd(s, a.enc_lo), a.numel);
      const float ghi = gamma_of_sum(__dmul_ru(s, a.enc_hi), a.numel);
      mode = __float_as_uint(glo) == __float_as_uint(ghi) ? 1 : 2;
      gamma = glo;
      if (lane == 0) {
        flag[1] = __float_as_uint(glo);
        st_release_u32(&flag[0], static_cast<uint32_t>(mode));
      }
    } else {
      if (lane == 0) {
        // wait for the last CTA's gamma (bounded; polled every ~0.1 us)
        uint32_t f = ld_acquire_u32(&flag[0]);
        const unsigned long long t0 = globaltimer_ns();
        while (f == 0) {
          __nanosleep(100);
          f = ld_acquire_u32(&flag[0]);
          if (f == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(a.err, kDevTimeout);
            break;
          }
        }
        mode = static_cast<int>(f);
        gamma = __uint_as_float(__ldcg(&flag[1]));
      }
      mode = __shfl_sync(0xffffffffu, mode, 0);
      gamma = __shfl_sync(0xffffffffu, gamma, 0);
    }
    if (mode == 0 || s_abort) {
      if (lane == 0) s_state = -1;
    } else {
      if (mode == 2) {
        // exact sum: every warp bins its share of the slice (the work loop
        // below); then one arrival per CTA and the exact gamma
        for (int e = lane; e < 256; e += 32) s_bins[e] = 0ull;
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          s_state = 2;
        }
        bool ok = true;
        if (lane == 0) {
          const unsigned long long t0 = globaltimer_ns();
          while (*reinterpret_cast<volatile int*>(&s_binned) < kQWarps - 1) {
            __nanosleep(100);
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
              record_error(a.err, kDevTimeout);
              ok = false;
              break;
            }
          }
        }
        // warp 0's own share
        for (int64_t i = lane; i < onv; i += 32 * kQWarps) bin_abs<kF32>(s_bins, s_w[i]);
        for (int64_t i = tail_v0 + lane; i < tail_v1; i += 32 * kQWarps) bin_abs<kF32>(s_bins, __ldg(a.W + i));
        __syncwarp();
        __threadfence_block();
        for (int e = lane; e < 256; e += 32)
          if (s_bins[e]) atomicAdd(gbins + e, s_bins[e]);
        __syncwarp();  // every lane's bins are added before lane 0 arrives
        if (lane == 0 && ok) {
          ok = grid_arrive_wait(&arrive[1], G, a.err);
          if (ok) gamma = gamma_of_sum(exact_sum_from_bins(gbins, kF32 ? 23 : 7), a.numel);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        gamma = __shfl_sync(0xffffffffu, gamma, 0);
        if (!ok) mode = 0;
      }
      if (lane == 0) {
        if (mode == 0) {
          s_state = -1;
        } else {
          if (b == 0) *a.gamma_out = gamma;
          const float thr = __double2float_rd(__dmul_rn(static_cast<double>(gamma), 0.5 + 0x1p-25));
          uint32_t key;
          if constexpr (kF32) {
            key = __float_as_uint(thr);
          } else {
            const uint32_t tb = __float_as_uint(thr) >> 16;
            key = (tb | (tb << 16)) + 0x80008000u;
          }
          s_key = key;
          s_gamma = gamma;
          __threadfence_block();
          s_state = 1;
        }
      }
    }
    __syncwarp();
  }

  // -------------------------------------------------- work loop, all warps
  const int64_t on_rounds = (onv + 127) / 128;
  const int64_t n_rounds = on_rounds + (tail_v1 - tail_v0 + 127) / 128;
  bool rows_left = a.M > 0;
  bool binned = warp == 0;  // warp 0 bins inside the control block
  if (rows_left) pdl_wait_primary();  // launch 1 has cleared the row counter
  volatile int* state = &s_state;
  const unsigned long long t_idle = globaltimer_ns();
  for (;;) {
    const int st = *state;
    if (st < 0) break;
    if (st == 2 && !binned) {
      for (int64_t i = lane + 32 * warp; i < onv; i += 32 * kQWarps) bin_abs<kF32>(s_bins, s_w[i]);
      for (int64_t i = tail_v0 + lane + 32 * warp; i < tail_v1; i += 32 * kQWarps) bin_abs<kF32>(s_bins, __ldg(a.W + i));
      __syncwarp();
      __threadfence_block();
      if (lane == 0) atomicAdd(&s_binned, 1);
      binned = true;
      continue;
    }
    if (st == 1) {
      uint32_t r = 0;
      if (lane == 0) r = static_cast<uint32_t>(atomicAdd(&s_round, 1));
      r = __shfl_sync(0xffffffffu, r, 0);
      if (r < n_rounds) {
        const uint32_t key = s_key;
        if (r < on_rounds)
          code_round<kF32, true>(s_w, 128 * static_cast<int64_t>(r), onv, a.packed + g0, key, lane);
        else
          code_round<kF32, false>(a.W + tail_v0, 128 * (r - on_rounds), tail_v1 - tail_v0, a.packed + g0 + on, key,
                                  lane);
        continue;
      }
    }
    if (rows_left) {
      const int64_t m0 = warp_claim(rows, 2u);
      if (m0 < a.M) {
        token_pair<VPL>(a, m0);
        continue;
      }
      rows_left = false;
    }
    if (st == 1) break;  // codes all claimed, no rows left
    __nanosleep(200);    // waiting for gamma
    if (globaltimer_ns() - t_idle > 2 * kWaitLimitNs) break;  // the control warp gave up
  }
}

}  // namespace

// Fixed device scratch for bl_quantize_weight_noalloc: the workspace of one
// call (arrival counters, one fp64 partial sum per CTA, exact-sum bins),
// 10752 bytes. Every GPU that loads the library holds this array until the
// process exits.
static __device__ __align__(256) uint8_t g_noalloc_ws[kWsBytes];

size_t quantize_workspace_bytes() { return kWsBytes; }

namespace {

// Geometry of one S1 (+ S2) launch.
struct QuantGeometry {
  unsigned ctas;
  size_t smem;
};

template <bool kF32>
QuantGeometry quant_geometry(int64_t ngroups, int64_t M, QuantArgs& a) {
  constexpr int V = kF32 ? 4 : 2;
  constexpr int kGroupBytes = 16 * V;
  constexpr int kChunkGroups = kChunkBytes / kGroupBytes;
  constexpr int kElems = kF32 ? 4 : 8;  // elements per 16-byte vector
  // enough CTAs to spread the slice (>= 256 groups each) and the tokens (>= 16
  // rows each), at most one per SM so that all of them are resident together
  const int64_t want = std::max<int64_t>((ngroups + 255) / 256, (M + 15) / 16);
  const int64_t cap = std::min<int64_t>(device_sm_count(), kMaxQuantCtas);
  const int64_t G = std::max<int64_t>(1, std::min(want, cap));
  a.ngroups = ngroups;
  a.per = (ngroups + G - 1) / G;
  a.onchip_cap = kMaxOnchipBytes / kGroupBytes;
  const int64_t on_max = std::min<int64_t>(a.per, a.onchip_cap);
  // Enclosure of S around the fp64 tree sum: every leaf passes through at most
  // d roundings (its accumulator's sequential adds, the four accumulators, the
  // warp shuffle tree, the sequential warp sums, the lane sums of the
  // partials, their shuffle tree), each off by at most 2^-53 of a partial sum
  // that is at most S (1 + 2^-30) with all terms >= 0, so |fp64 sum - S| <=
  // d 2^-53 (1 + 2^-30) S; e = d 2^-52 covers S on both sides.
  const int64_t nch_max = (on_max + kChunkGroups - 1) / kChunkGroups;
  const double per_acc = static_cast<double>(a.per) * V / (4.0 * kQThreads) + static_cast<double>(nch_max) + 3.0;
  const double d = kElems * per_acc + 2 + 5 + kQWarps + std::ceil(static_cast<double>(G) / 32.0) + 5 + 8;
  const double e = std::ldexp(d, -52);
  a.enc_lo = 1.0 - e;
  a.enc_hi = 1.0 + e;
  return {static_cast<unsigned>(G), static_cast<size_t>(on_max) * kGroupBytes};
}

template <bool kF32, int VPL>
cudaError_t launch_fused(QuantArgs& a, cudaStream_t s) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(quant_fused_kernel<kF32, VPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kMaxOnchipBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const QuantGeometry geo = quant_geometry<kF32>(a.ngroups, a.M, a);
  cudaError_t e = launch_pdl(quant_reset_kernel, dim3(1), dim3(256), 0, s, a.ws);
  if (e != cudaSuccess) return e;
  return launch_pdl(quant_fused_kernel<kF32, VPL>, dim3(geo.ctas), dim3(kQThreads), geo.smem, s, a);
}

template <int VPL>
cudaError_t launch_fused_dtype(bool f32, QuantArgs& a, cudaStream_t s) {
  return f32 ? launch_fused<true, VPL>(a, s) : launch_fused<false, VPL>(a, s);
}

template <int VPL>
void launch_act(const uint4* xv, int64_t M, int nv, int8_t* xq, float* sx, cudaStream_t s) {
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

}  // namespace

cudaError_t launch_quantize(const void* W, int w_is_f32, int64_t N, int64_t K, const void* x, int64_t M,
                            uint8_t* packed, float* gamma, void* workspace, int8_t* xq, float* sx, int* err,
                            cudaStream_t s) {
  QuantArgs a{};
  a.W = static_cast<const uint4*>(W);
  a.ngroups = N * K / 16;  // K % 32 == 0
  a.numel = static_cast<double>(N * K);
  a.packed = reinterpret_cast<uint32_t*>(packed);
  a.gamma_out = gamma;
  a.ws = static_cast<uint8_t*>(workspace);
  a.err = err;
  a.x = static_cast<const uint4*>(x);
  a.M = M;
  a.nv = static_cast<int>(K / 8);
  a.xq = xq;
  a.sx = sx;
  const int per_lane = (a.nv + 31) / 32;
  const bool f32 = w_is_f32 != 0;
  cudaError_t e = cudaSuccess;
  switch (M > 0 && per_lane <= 10 ? per_lane : 0) {
#define BL_Q_CASE(n)                          \
  case n:                                     \
    e = launch_fused_dtype<n>(f32, a, s);     \
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

cudaError_t launch_quantize_weight(const void* W, int w_is_f32, int64_t N, int64_t K, uint8_t* packed,
                                   float* gamma, void* workspace, int* err, cudaStream_t s) {
  return launch_quantize(W, w_is_f32, N, K, nullptr, 0, packed, gamma, workspace, nullptr, nullptr, err, s);
}

// Device address of g_noalloc_ws on the current device. Host code only holds
// a stand-in for the array's name, so the address is looked up with the
// device current, on every call: a cached address would go stale if the
// caller reset the device and the module were loaded again elsewhere. The
// first lookup on a device loads the module there (so it belongs before any
// stream capture); later ones are host-side table lookups.
cudaError_t launch_quantize_weight_noalloc(const void* W, int w_is_f32, int64_t N, int64_t K, uint8_t* packed,
                                           float* gamma, int* err, cudaStream_t s) {
  void* scratch = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&scratch, g_noalloc_ws);
  if (e != cudaSuccess) return e;
  return launch_quantize_weight(W, w_is_f32, N, K, packed, gamma, scratch, err, s);
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

}  // namespace bl
