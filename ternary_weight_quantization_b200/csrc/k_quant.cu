// S1 and S2 of the BitLinear hot path on sm_100a: absmean ternarisation with
// 2-bit packing, and per-token absmax INT8 activation quantisation.
//
// S1 needs the mean |W| of the whole tensor before any code can be written,
// and S2 is independent of it. bl_quantize is two launches:
//
//   sum launch   every CTA sums |W| of its contiguous slice of W in fp64 and
//                stores the partial sum in its own workspace slot (no atomics,
//                no waits); the same warps quantise token rows (S2). This is
//                the pass that streams W and x from HBM.
//   code launch  (a programmatic dependent: its CTAs wait for the sum launch
//                to complete) every CTA reduces the partial sums in one fixed
//                order, forms gamma and writes the codes of its share of W,
//                which it reads again (the sum launch has just left W in L2;
//                its own loads are issued before gamma is known).
//
// gamma = max(fp32(fp64(fp64(S) / numel)), 1e-5) with S = sum |W| (exactly
// rounded to fp64, "1BitTraining.md" weight_quant / "bitlinear.py"
// ternary_quantize with the fp64 accumulation the reading fixes). The fp64
// tree sum carries a bounded rounding error, so gamma is formed at both ends
// of an enclosure of S; as the chain of roundings is monotone, when the two
// agree that value is the exact gamma (all but about one tensor in 10^5).
// Otherwise the code launch computes S exactly -- integer sums of the
// significands per exponent field, combined as one wide integer and rounded
// once -- behind a grid-wide barrier with a bounded wait, so gamma never
// depends on the reduction order or on the GPU's SM count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "bl_abs_sum.cuh"
#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

// ---------------------------------------------------------------- S1 geometry
constexpr int kSumThreads = 1024; // sum launch: 32 warps per CTA
constexpr int kSumWarps = kSumThreads / 32;
constexpr int kSumUnroll = 8;     // 16-byte loads in flight per thread
constexpr bool kSumInterleave = false;  // W in blocks dealt to the CTAs in turn (else contiguous slices)
constexpr int kCodeThreads = 512; // code launch: 16 warps per CTA
constexpr int kCodeWarps = kCodeThreads / 32;
constexpr int kCodeRowsPerCta = 10;// token rows a code-launch CTA quantises (< kCodeWarps)


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
// field 00 = 0, 01 = +1, 11 = -1). For a bf16 w and thr > 0, |w| > thr <=>
// w > tb or w < -tb with tb = thr truncated to bf16 (the largest bf16 <= thr),
// so two bf16x2 compares per word (on the multiply-add pipe) give both the
// nonzero and the sign information: each half of a result is 1.0 (0x3F80)
// where the compare holds, else 0. One byte permutation per word pair
// gathers the low bytes of the halves (0x80 or 0) of four elements; a high
// multiply by S = 2^25 + 2^19 + 2^13 + 2^7 moves bits 7, 15, 23, 31 to bits
// 0, 2, 4, 6 of its high word (+1 fields), one by 3 S to bits 0-1, 2-3, 4-5,
// 6-7 (-1 fields); every partial product lands on bits of its own, so nothing
// carries into the low byte, and the two (exclusive) results are added by the
// second multiply. Bits 16..31 of the result are not zero.
__device__ __forceinline__ uint32_t bf16x2_gt(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.gt.bf16x2.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_lt(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.lt.bf16x2.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// thr2: tb in both halves.
__device__ __forceinline__ uint32_t codes8_bf16(const uint4& v, uint32_t thr2) {
  constexpr uint32_t kSpread = (1u << 25) | (1u << 19) | (1u << 13) | (1u << 7);
  const uint32_t nthr2 = thr2 | 0x80008000u;
  const uint32_t pl = __byte_perm(bf16x2_gt(v.x, thr2), bf16x2_gt(v.y, thr2), 0x6420);  // +1, elements 0..3
  const uint32_t ph = __byte_perm(bf16x2_gt(v.z, thr2), bf16x2_gt(v.w, thr2), 0x6420);  // +1, elements 4..7
  const uint32_t nl = __byte_perm(bf16x2_lt(v.x, nthr2), bf16x2_lt(v.y, nthr2), 0x6420);  // -1
  const uint32_t nh = __byte_perm(bf16x2_lt(v.z, nthr2), bf16x2_lt(v.w, nthr2), 0x6420);
  const uint32_t lo = __umulhi(nl, 3u * kSpread) + __umulhi(pl, kSpread);
  const uint32_t hi = __umulhi(nh, 3u * kSpread) + __umulhi(ph, kSpread);
  return __byte_perm(lo, hi, 0x0040);
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
// the bf16 threshold in both halves or the fp32 threshold's bit pattern.
template <bool kF32>
__device__ __forceinline__ uint32_t vec_codes(const uint4& v, uint32_t key) {
  if constexpr (kF32) return codes4_f32(v, __uint_as_float(key));
  else return codes8_bf16(v, key);
}

// The vectors of a warp's 32 consecutive 16-byte vectors, one per lane, are
// V = 2 (bf16) or 4 (fp32) per group: the lanes of a group combine their code
// bits and its first lane gets the group's 32-bit word (bf16: the low halves
// of the two lanes' results; fp32: the four 8-bit results).
template <bool kF32>
__device__ __forceinline__ uint32_t gather_group_word(uint32_t bits, int lane) {
  if constexpr (kF32) {
    uint32_t word = bits << (8 * (lane & 3));
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) word |= __shfl_down_sync(0xffffffffu, word, off);
    return word;
  } else {
    return __byte_perm(bits, __shfl_down_sync(0xffffffffu, bits, 1), 0x5410);
  }
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
struct SumArgs {
  const uint4* W;  // [N, K] as 16-byte vectors
  int64_t nvec;    // vectors of W
  int64_t per;     // vectors per CTA slice (the last slices may be shorter or empty)
  double* parts;   // one partial sum per CTA
  uint8_t* ws;     // exact-sum counter and bins, cleared here for the code launch
  const uint4* x;  // S2: x [M, K] as 16-byte vectors (M = 0: no tokens)
  int64_t M;
  int nv;          // K / 8
  int8_t* xq;
  float* sx;
};

// Sum launch, kSumThreads threads per CTA. Nothing in it waits on another
// CTA. CTA b first quantises token rows [b M / G, (b + 1) M / G) (warp w:
// rows w, w + kSumWarps, ... of them), then sums |W| over its share, so that
// W is the most recent data in L2 when the code launch reads it again. Thread
// t adds its vectors (the j-th at a fixed index: in the CTA's contiguous
// slice, or in the j-th block of kSumThreads vectors dealt to the CTA) into
// accumulator j mod 4, in order, the elements of a vector in order; the CTA's
// partial sum is the four accumulators added pairwise, then a butterfly over
// the warp's lanes (the same value in every lane), then the warps' sums in
// warp order. Every step is a fixed sequence of fp64 additions, so the
// partial sums do not depend on scheduling.
template <bool kF32, int VPL>
__global__ void __launch_bounds__(kSumThreads, 1024 / kSumThreads) quant_sum_kernel(const __grid_constant__ SumArgs a) {
  __shared__ double s_red[kSumWarps];
  pdl_wait_primary();  // W and x may be written by earlier work of the stream
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, t = threadIdx.x;
  const int64_t b = blockIdx.x, G = gridDim.x;
  if (b == 0) {
    unsigned long long* bins = reinterpret_cast<unsigned long long*>(a.ws + kWsBins);
    for (int e = t; e < 256; e += kSumThreads) bins[e] = 0ull;
    if (t == 0) *reinterpret_cast<uint32_t*>(a.ws + kWsArrive) = 0u;
  }
  if (a.M > 0) {
    const int64_t r0 = b * a.M / G, r1 = (b + 1) * a.M / G;
    if constexpr (VPL > 0) act_rows<VPL, false>(a.x, r1, a.nv, a.xq, a.sx, r0 + warp, kSumWarps);
    else act_rows_two_pass(a.x, r1, a.nv, a.xq, a.sx, r0 + warp, kSumWarps);
  }
  // the thread's j-th vector of W: in its CTA's contiguous slice, or in
  // blocks of kSumThreads vectors dealt to the CTAs in turn
  const int64_t v0 = b * a.per;
  const int64_t vend = kSumInterleave ? a.nvec : (v0 + a.per < a.nvec ? v0 + a.per : a.nvec);
  auto vec_index = [&](int64_t j) -> int64_t {
    if constexpr (kSumInterleave) return (b + G * j) * kSumThreads + t;
    else return v0 + t + kSumThreads * j;
  };
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  int64_t j = 0;
  for (; vec_index(j + kSumUnroll - 1) < vend; j += kSumUnroll) {
    uint4 v[kSumUnroll];
#pragma unroll
    for (int u = 0; u < kSumUnroll; ++u) v[u] = __ldg(a.W + vec_index(j + u));
#pragma unroll
    for (int u = 0; u < kSumUnroll; ++u) acc[u & 3] = add_abs<kF32>(acc[u & 3], v[u]);
  }
  if (vec_index(j) < vend) {  // fewer than kSumUnroll vectors left for this thread
    uint4 v[kSumUnroll];
#pragma unroll
    for (int u = 0; u < kSumUnroll; ++u)
      v[u] = vec_index(j + u) < vend ? __ldg(a.W + vec_index(j + u)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kSumUnroll; ++u)
      if (vec_index(j + u) < vend) acc[u & 3] = add_abs<kF32>(acc[u & 3], v[u]);
  }
  double ts = __dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ts = __dadd_rn(ts, __shfl_xor_sync(0xffffffffu, ts, off));
  if (lane == 0) s_red[warp] = ts;
  __syncthreads();
  if (t == 0) {
    double p = 0.0;
#pragma unroll
    for (int w = 0; w < kSumWarps; ++w) p = __dadd_rn(p, s_red[w]);
    a.parts[b] = p;
  }
}

struct CodeArgs {
  const uint4* W;
  int64_t nvec;
  const double* parts;  // the sum launch's partial sums
  int nparts;
  double numel;
  double enc_lo, enc_hi;  // S lies in [fp64 sum * enc_lo, fp64 sum * enc_hi]
  uint32_t* packed;
  float* gamma_out;
  uint8_t* ws;
  int* err;
  const uint4* x;   // S2 rows [m_begin, m_begin + M2) of x (M2 = 0: none)
  int64_t m_begin, M2;
  int nv;           // K / 8
  int8_t* xq;
  float* sx;
};

// Round q of W: 128 consecutive 16-byte vectors, lane l holding vectors
// 128 q + l + 32 u (u = 0..3); vectors past W (or q >= q_end) are zero.
// Rounds below q_full (all 128 vectors inside W) take one address.
__device__ __forceinline__ void load_round(const uint4* W, int64_t q, int64_t q_end, int64_t q_full, int64_t nvec,
                                           int lane, uint4 (&v)[4]) {
  if (q < q_full) {
    const uint4* p = W + 128 * q + lane;
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(p + 32 * u);
    return;
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = 128 * q + lane + 32 * u;
    v[u] = (q < q_end && i < nvec) ? __ldg(W + i) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Codes of round q (as load_round holds it): a group's V lanes combine their
// bits and its first lane stores the group's word.
template <bool kF32>
__device__ __forceinline__ void store_round(const uint4 (&v)[4], int64_t q, int64_t q_full, int64_t nvec,
                                            uint32_t* out, uint32_t key, int lane) {
  constexpr int V = kF32 ? 4 : 2;
  uint32_t word[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) word[u] = gather_group_word<kF32>(vec_codes<kF32>(v[u], key), lane);
  if ((lane & (V - 1)) != 0) return;
  if (q < q_full) {
    uint32_t* p = out + (128 * q + lane) / V;
#pragma unroll
    for (int u = 0; u < 4; ++u) p[32 / V * u] = word[u];
    return;
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = 128 * q + lane + 32 * u;
    if (i < nvec) out[i / V] = word[u];
  }
}

// The compare key of the code rule for gamma: the fp32 threshold's bit
// pattern, or for bf16 the threshold truncated to bf16 in both halves.
template <bool kF32>
__device__ __forceinline__ uint32_t code_key(float gamma) {
  const float thr = __double2float_rd(__dmul_rn(static_cast<double>(gamma), 0.5 + 0x1p-25));
  if constexpr (kF32) return __float_as_uint(thr);
  const uint32_t tb = __float_as_uint(thr) >> 16;
  return tb | (tb << 16);
}

// Waits (bounded) until `mode` is set; -1 after the wait limit.
__device__ __forceinline__ int wait_mode(const volatile int* mode, int* err) {
  int m = *mode;
  if (m) return m;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    m = *mode;
    if (m) return m;
    if ((i & 255) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
      record_error(err, kDevTimeout);
      return -1;
    }
  }
}

// Code launch, kCodeThreads threads per CTA, all CTAs resident together (the
// exact-sum path meets at a grid-wide barrier). CTA b codes the rounds
// [b R / G, (b + 1) R / G) of the R rounds of 128 vectors: warp w first takes
// round w of the range, then claims the next unclaimed one from a counter of
// the CTA, loading each round while it codes the one before. Warps 1..r of
// the CTA also quantise the CTA's r token rows (S2 rows the sum launch left),
// their loads issued first, while warp 0 adds the partial sums (lane l:
// partial sums l, l + 32, ... in order, then a butterfly, so every CTA forms
// the same gamma) and the other warps load their first round. If the
// enclosure of S straddles a rounding boundary of gamma (rare), every warp
// bins rounds w, w + 16, ... of the CTA's range for the exact sum, the CTAs
// add their bins to the grid's and meet at the barrier, and every CTA forms
// the exact gamma.
template <bool kF32, int VPL>
__global__ void __launch_bounds__(kCodeThreads, 2) quant_code_kernel(const __grid_constant__ CodeArgs a) {
  __shared__ unsigned long long s_bins[256];
  __shared__ float s_gamma;
  __shared__ int s_mode;        // 0: not known yet, 1: gamma known, 2: exact sum needed, -1: gave up
  __shared__ uint32_t s_next;   // next round of the CTA's range to claim (offset from its first)
  pdl_wait_primary();           // the sum launch has completed
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = blockIdx.x, G = gridDim.x;
  const int64_t nrounds = (a.nvec + 127) / 128;
  const int64_t q0 = b * nrounds / G, q1 = (b + 1) * nrounds / G;
  const int64_t q_full = a.nvec / 128 < q1 ? a.nvec / 128 : q1;  // rounds wholly inside W
  const int64_t row = a.m_begin + b * a.M2 / G + warp - 1;
  const bool has_row = warp >= 1 && row < a.m_begin + (b + 1) * a.M2 / G;
  int64_t r = q0 + warp;
  // Warp 0's first loads of partial sums go out before any load of W or x
  // (which would queue ahead of them); lane l adds partial sums l, l + 32,
  // ... in order, 8 loads at a time.
  constexpr int kPartBatch = 8;
  double pv[kPartBatch];
  if (warp == 0) {
#pragma unroll
    for (int u = 0; u < kPartBatch; ++u) {
      const int p = 32 * u + lane;
      pv[u] = p < a.nparts ? __ldcg(a.parts + p) : 0.0;
    }
  }
  if (threadIdx.x == 0) s_mode = 0;
  __syncthreads();
  // one register array serves the token row (VPL vectors) and then the round
  // being coded (the first 4)
  uint4 buf[VPL > 4 ? VPL : 4];
  uint4(&v)[4] = *reinterpret_cast<uint4(*)[4]>(buf);
  if (has_row) {
    if constexpr (VPL > 0) load_row<VPL>(a.x + row * a.nv, a.nv, lane, *reinterpret_cast<uint4(*)[VPL > 0 ? VPL : 1]>(buf));
  } else {
    load_round(a.W, r, q1, q_full, a.nvec, lane, v);
  }
  if (warp == 0) {
    double s = 0.0;
    for (int k0 = 0; k0 < a.nparts; k0 += 32 * kPartBatch) {
      if (k0 > 0) {
#pragma unroll
        for (int u = 0; u < kPartBatch; ++u) {
          const int p = k0 + 32 * u + lane;
          pv[u] = p < a.nparts ? __ldcg(a.parts + p) : 0.0;
        }
      }
#pragma unroll
      for (int u = 0; u < kPartBatch; ++u)
        if (k0 + 32 * u + lane < a.nparts) s = __dadd_rn(s, pv[u]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
    for (int e = lane; e < 256; e += 32) s_bins[e] = 0ull;
    __syncwarp();
    if (lane == 0) {
      const float glo = gamma_of_sum(__dmul_rd(s, a.enc_lo), a.numel);
      const float ghi = gamma_of_sum(__dmul_ru(s, a.enc_hi), a.numel);
      s_gamma = glo;
      s_next = kCodeWarps;
      __threadfence_block();
      *reinterpret_cast<volatile int*>(&s_mode) = __float_as_uint(glo) == __float_as_uint(ghi) ? 1 : 2;
    }
  }
  if (has_row) {
    if constexpr (VPL > 0) quant_row<VPL>(*reinterpret_cast<uint4(*)[VPL > 0 ? VPL : 1]>(buf), a.nv, lane, row, a.xq, a.sx);
    else act_rows_two_pass(a.x, row + 1, a.nv, a.xq, a.sx, row, 1);
  }
  int mode = wait_mode(&s_mode, a.err);
  if (mode == 2) {
    for (int64_t q = q0 + warp; q < q1; q += kCodeWarps) {
      uint4 w[4];
      load_round(a.W, q, q1, q_full, a.nvec, lane, w);
#pragma unroll
      for (int u = 0; u < 4; ++u) bin_abs<kF32>(s_bins, w[u]);
    }
    __syncthreads();
    if (warp == 0) {
      unsigned long long* gbins = reinterpret_cast<unsigned long long*>(a.ws + kWsBins);
      for (int e = lane; e < 256; e += 32)
        if (s_bins[e]) atomicAdd(gbins + e, s_bins[e]);
      __syncwarp();  // every lane's bins are added before lane 0 arrives
      if (lane == 0) {
        if (grid_arrive_wait(reinterpret_cast<uint32_t*>(a.ws + kWsArrive), gridDim.x, a.err)) {
          s_gamma = gamma_of_sum(exact_sum_from_bins(gbins, kF32 ? 23 : 7), a.numel);
          s_mode = 1;
        } else {
          s_mode = -1;
        }
      }
    }
    __syncthreads();
    mode = s_mode;
  }
  if (mode < 0) return;
  const float gamma = *reinterpret_cast<const volatile float*>(&s_gamma);
  if (b == 0 && threadIdx.x == 0) *a.gamma_out = gamma;
  const uint32_t key = code_key<kF32>(gamma);
  if (has_row) load_round(a.W, r, q1, q_full, a.nvec, lane, v);
  while (r < q1) {
    uint32_t c = 0;
    if (lane == 0) c = atomicAdd(&s_next, 1u);
    const int64_t rn = q0 + __shfl_sync(0xffffffffu, c, 0);
    uint4 nx[4];
    load_round(a.W, rn, q1, q_full, a.nvec, lane, nx);
    store_round<kF32>(v, r, q_full, a.nvec, a.packed, key, lane);
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = nx[u];
    r = rn;
  }
}

}  // namespace

// Fixed device scratch for bl_quantize_weight_noalloc: the workspace of one
// call (the exact-sum arrival counter and bins, and one fp64 partial sum per
// CTA of the sum launch). Every GPU that loads the library holds this array
// until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_ws[kWsBytes];

size_t quantize_workspace_bytes() { return kWsBytes; }

namespace {

// Resident CTAs per SM of `kernel` at `threads` threads (cached per device in
// the caller's table).
template <typename Kernel>
int blocks_per_sm(Kernel kernel, int threads, int (&cache)[64]) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, 0) != cudaSuccess || occ < 1) occ = 1;
  cudaGetLastError();
  if (dev >= 0 && dev < 64) cache[dev] = occ;
  return occ;
}

// Blocks of the code launch for W of `nvec` vectors: no more CTAs than can
// be resident at once (the exact-sum barrier), and no more warps than rounds
// of 128 vectors.
template <bool kF32, int VPL>
int64_t code_grid(int64_t nvec) {
  static int occ_code[64] = {};
  const int64_t nrounds = (nvec + 127) / 128;
  const int64_t cap = device_sm_count() * blocks_per_sm(quant_code_kernel<kF32, VPL>, kCodeThreads, occ_code);
  return std::max<int64_t>(1, std::min<int64_t>(cap, (nrounds + kCodeWarps - 1) / kCodeWarps));
}

// The code launch's arguments for W (`nvec` vectors, `numel` elements) whose
// `nparts` partial sums are in the workspace, every term having passed
// through at most `part_roundings` roundings inside its partial sum. No
// token rows (the caller sets them).
//
// Enclosure of S around the fp64 sum: on top of those roundings the code
// launch adds the ceil(nparts / 32) sequential partial sums of a lane and 5
// butterfly levels. Each rounding is off by at most 2^-53 of a partial sum,
// and with all terms >= 0 every partial sum is at most S (1 + 2^-30), so
// |fp64 sum - S| <= d 2^-53 (1 + 2^-30) S; e = d 2^-52 (8 roundings to
// spare) covers S on both sides.
CodeArgs code_args(const void* W, int64_t nvec, int64_t numel, int nparts, double part_roundings, uint8_t* packed,
                   float* gamma, uint8_t* ws, int* err) {
  CodeArgs ca{};
  ca.W = static_cast<const uint4*>(W);
  ca.nvec = nvec;
  ca.parts = reinterpret_cast<const double*>(ws + kWsParts);
  ca.nparts = nparts;
  ca.numel = static_cast<double>(numel);
  ca.packed = reinterpret_cast<uint32_t*>(packed);
  ca.gamma_out = gamma;
  ca.ws = ws;
  ca.err = err;
  const double d = part_roundings + static_cast<double>((nparts + 31) / 32) + 5 + 8;
  const double e = std::ldexp(d, -52);
  ca.enc_lo = 1.0 - e;
  ca.enc_hi = 1.0 + e;
  return ca;
}

// The two launches of S1 (+ S2 when M > 0).
template <bool kF32, int VPL>
cudaError_t launch_s1(const void* W, int64_t N, int64_t K, const void* x, int64_t M, uint8_t* packed, float* gamma,
                      uint8_t* ws, int8_t* xq, float* sx, int* err, cudaStream_t s) {
  constexpr int kElems = kF32 ? 4 : 8;  // elements per 16-byte vector
  static int occ_sum[64] = {};
  const int64_t sms = device_sm_count();
  const int64_t nvec = N * K / kElems;
  // the code launch takes up to kCodeRowsPerCta token rows per CTA (the rest
  // go to the sum launch)
  const int64_t G2 = code_grid<kF32, VPL>(nvec);
  const int64_t M2 = std::min<int64_t>(M, G2 * kCodeRowsPerCta), M1 = M - M2;

  SumArgs sa{};
  sa.W = static_cast<const uint4*>(W);
  sa.nvec = nvec;
  sa.ws = ws;
  sa.parts = reinterpret_cast<double*>(ws + kWsParts);
  sa.x = static_cast<const uint4*>(x);
  sa.M = M1;
  sa.nv = static_cast<int>(K / 8);
  sa.xq = xq;
  sa.sx = sx;
  // sum launch: every SM filled (at most kMaxQuantCtas partial sums), fewer
  // CTAs only when W has fewer than 2048 vectors per CTA and its tokens fewer
  // than one row per warp
  const int64_t cap1 =
      std::min<int64_t>(sms * blocks_per_sm(quant_sum_kernel<kF32, VPL>, kSumThreads, occ_sum), kMaxQuantCtas);
  const int64_t want1 = std::max<int64_t>((nvec + kSumThreads * kSumUnroll - 1) / (kSumThreads * kSumUnroll),
                                          (M1 + kSumWarps - 1) / kSumWarps);
  const int64_t G1 = std::max<int64_t>(1, std::min(want1, cap1));
  sa.per = (nvec + G1 - 1) / G1;

  // Roundings of a term inside its partial sum: its accumulator's sequential
  // adds (kElems per vector, at most ceil(nj / 4) vectors of the thread's nj),
  // the two levels joining the four accumulators, the 5 butterfly levels and
  // the kSumWarps sequential warp sums.
  const int64_t nj = kSumInterleave ? ((nvec + kSumThreads - 1) / kSumThreads + G1 - 1) / G1
                                    : (sa.per + kSumThreads - 1) / kSumThreads;  // vectors per thread
  const double part_roundings = static_cast<double>(kElems) * static_cast<double>((nj + 3) / 4) + 2 + 5 + kSumWarps;
  CodeArgs ca = code_args(W, nvec, N * K, static_cast<int>(G1), part_roundings, packed, gamma, ws, err);
  ca.x = sa.x;
  ca.m_begin = M1;
  ca.M2 = M2;
  ca.nv = sa.nv;
  ca.xq = xq;
  ca.sx = sx;

  cudaError_t st = launch_pdl(quant_sum_kernel<kF32, VPL>, dim3(static_cast<unsigned>(G1)), dim3(kSumThreads), 0, s, sa);
  if (st != cudaSuccess) return st;
  return launch_pdl(quant_code_kernel<kF32, VPL>, dim3(static_cast<unsigned>(G2)), dim3(kCodeThreads), 0, s, ca);
}

template <int VPL>
void launch_act(const uint4* xv, int64_t M, int nv, int8_t* xq, float* sx, cudaStream_t s) {
  constexpr bool kPrefetch = VPL <= 12;
  static int per_sm[64] = {};
  const int occ = blocks_per_sm(act_quant_kernel<VPL, kPrefetch>, 32 * kActRowsPerBlock, per_sm);
  const int64_t want = (M + kActRowsPerBlock - 1) / kActRowsPerBlock;
  const int64_t cap = static_cast<int64_t>(occ) * device_sm_count();
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  launch_pdl(act_quant_kernel<VPL, kPrefetch>, dim3(grid), dim3(32 * kActRowsPerBlock), 0, s, xv, M, nv, xq, sx);
}

}  // namespace

cudaError_t launch_quantize(const void* W, int w_is_f32, int64_t N, int64_t K, const void* x, int64_t M,
                            uint8_t* packed, float* gamma, void* workspace, int8_t* xq, float* sx, int* err,
                            cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int per_lane = (static_cast<int>(K / 8) + 31) / 32;
  const bool f32 = w_is_f32 != 0;
  cudaError_t e = cudaSuccess;
  switch (M > 0 && per_lane <= 10 ? per_lane : 0) {
#define BL_Q_CASE(n)                                                                     \
  case n:                                                                                \
    e = f32 ? launch_s1<true, n>(W, N, K, x, M, packed, gamma, ws, xq, sx, err, s)      \
            : launch_s1<false, n>(W, N, K, x, M, packed, gamma, ws, xq, sx, err, s);    \
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

cudaError_t launch_quantize_codes(const void* W, int w_is_f32, int64_t N, int64_t K, int nparts,
                                  double part_roundings, uint8_t* packed, float* gamma, void* workspace, int* err,
                                  cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t nvec = N * K / (w_is_f32 ? 4 : 8);
  const CodeArgs ca = code_args(W, nvec, N * K, nparts, part_roundings, packed, gamma, ws, err);
  const dim3 block(kCodeThreads);
  cudaError_t e = w_is_f32
                      ? launch_pdl(quant_code_kernel<true, 0>, dim3(static_cast<unsigned>(code_grid<true, 0>(nvec))),
                                   block, 0, s, ca)
                      : launch_pdl(quant_code_kernel<false, 0>, dim3(static_cast<unsigned>(code_grid<false, 0>(nvec))),
                                   block, 0, s, ca);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
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
