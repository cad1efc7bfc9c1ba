// The master-free sign-gradient update on sm_100a ("1BitTraining.md", "Why
// this always holds", closing paragraph: the straight-through gradient and
// the gradient of the quantised weight share their sign, so a sign-based
// optimiser needs only the 2-bit weights on the device and one bit of
// gradient per weight, sent to one place that accumulates them).
//
//   G1 sign words   dW -> one sign bit per weight, 32 to a word
//   G2 vote         R ranks' sign words -> majority direction, 2-bit packed
//   G3 update       W <- dtype_rn(fp32(W) - lr * direction) where W is held
//   G2 + G3 + S1    the holder's vote and update in one sweep that also forms
//                   S1's |W| partial sums, followed by S1's code launch
//
// The three separate passes are HBM-bound streams with 16-byte vector loads.
// Each thread takes U items spaced one grid apart (so every load instruction
// of a warp stays contiguous) and issues all of their loads before it
// computes: with the grid sized to the work, the whole tensor is in flight in
// about one round trip instead of several dependent ones. The fused sweep
// works in warp rounds of 32 word positions (see signsgd_apply_kernel).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "bl_abs_sum.cuh"
#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kThreads = 256;

// ---------------------------------------------------------------- G1
// Sign bits of four bf16 values (two per word): bytes 1 and 3 of each word
// carry the sign bits at bit 7. One byte permutation gathers the four bytes,
// and the product by 2^21 + 2^14 + 2^7 + 1 moves bit 7 + 8i to bit 28 + i
// (the other partial products land below bit 28 at distinct positions, so
// nothing carries into the top nibble).
__device__ __forceinline__ uint32_t sign_nibble_bf16(uint32_t a, uint32_t b) {
  const uint32_t g = __byte_perm(a, b, 0x7531);
  return ((g & 0x80808080u) * 0x00204081u) >> 28;
}

// Word w covers elements 32 w .. 32 w + 31 of the flattened [N, K] tensor;
// element 32 w + j -> bit j.
template <bool kF32>
__device__ __forceinline__ uint32_t sign_word(const uint4 (&v)[kF32 ? 8 : 4]) {
  uint32_t s = 0;
  if constexpr (!kF32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s |= sign_nibble_bf16(v[i].x, v[i].y) << (8 * i);
      s |= sign_nibble_bf16(v[i].z, v[i].w) << (8 * i + 4);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      s |= ((v[i].x >> 31) | ((v[i].y >> 31) << 1) | ((v[i].z >> 31) << 2) | ((v[i].w >> 31) << 3)) << (4 * i);
  }
  return s;
}

constexpr int kPackU = 4;  // sign words per thread

template <bool kF32>
__global__ void __launch_bounds__(kThreads) sign_pack_kernel(const uint4* __restrict__ dw, int64_t nwords,
                                                             uint32_t* __restrict__ out) {
  pdl_wait_primary();
  pdl_launch_dependents();
  constexpr int kVecs = kF32 ? 8 : 4;  // 16-byte vectors per word
  const int64_t T = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t w0 = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; w0 < nwords; w0 += kPackU * T) {
    uint4 v[kPackU][kVecs];
#pragma unroll
    for (int u = 0; u < kPackU; ++u) {
      const int64_t w = w0 + u * T;
      if (w < nwords) {
#pragma unroll
        for (int i = 0; i < kVecs; ++i) v[u][i] = __ldg(dw + w * kVecs + i);
      }
    }
#pragma unroll
    for (int u = 0; u < kPackU; ++u) {
      const int64_t w = w0 + u * T;
      if (w < nwords) out[w] = sign_word<kF32>(v[u]);
    }
  }
}

// ---------------------------------------------------------------- G2
// 16 bits -> even bits of a 32-bit word.
__device__ __forceinline__ uint32_t spread_even16(uint32_t x) {
  x &= 0xFFFFu;
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  x = (x | (x << 2)) & 0x33333333u;
  x = (x | (x << 1)) & 0x55555555u;
  return x;
}

constexpr int kVotePlanes = 7;  // counts up to 127 ranks

// Per word position: the 32 counts of negative votes are kept bit-sliced
// (plane b holds bit b of every count; adding a rank's word is a ripple of
// and/xor through the planes), then compared with R / 2 from the top plane
// down. Direction per weight: +1 where the positive votes outnumber the
// negative ones, -1 where the negative ones do, 0 on a tie; written as the
// 2-bit ternary field (bit 2j = nonzero, bit 2j+1 = negative).
constexpr int kVoteU = 4;  // word positions per thread

__device__ __forceinline__ uint2 vote_fields(const uint32_t (&plane)[kVotePlanes], int ranks, uint32_t half) {
  uint32_t gt = 0u, eq = 0xFFFFFFFFu;  // count > half, count == half
#pragma unroll
  for (int b = kVotePlanes - 1; b >= 0; --b) {
    if ((half >> b) & 1u) {
      eq &= plane[b];
    } else {
      gt |= eq & plane[b];
      eq &= ~plane[b];
    }
  }
  // R odd: count > half <=> more negatives, otherwise more positives.
  // R even: count == half is a tie.
  const uint32_t neg = gt;
  const uint32_t nz = (ranks & 1) ? 0xFFFFFFFFu : ~eq;
  return make_uint2(spread_even16(nz) | (spread_even16(neg) << 1),
                    spread_even16(nz >> 16) | (spread_even16(neg >> 16) << 1));
}

__global__ void __launch_bounds__(kThreads) sign_vote_kernel(const uint32_t* __restrict__ words, int ranks,
                                                             int64_t nwords, uint2* __restrict__ dir) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const uint32_t half = static_cast<uint32_t>(ranks) >> 1;
  const int64_t T = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t w0 = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; w0 < nwords; w0 += kVoteU * T) {
    uint32_t plane[kVoteU][kVotePlanes];
#pragma unroll
    for (int u = 0; u < kVoteU; ++u)
#pragma unroll
      for (int b = 0; b < kVotePlanes; ++b) plane[u][b] = 0u;
    for (int r = 0; r < ranks; ++r) {
      const uint32_t* src = words + static_cast<int64_t>(r) * nwords;
      uint32_t x[kVoteU];
#pragma unroll
      for (int u = 0; u < kVoteU; ++u) x[u] = (w0 + u * T < nwords) ? __ldg(src + w0 + u * T) : 0u;
#pragma unroll
      for (int u = 0; u < kVoteU; ++u) {
        uint32_t carry = x[u];
#pragma unroll
        for (int b = 0; b < kVotePlanes; ++b) {
          const uint32_t t = plane[u][b] & carry;
          plane[u][b] ^= carry;
          carry = t;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kVoteU; ++u)
      if (w0 + u * T < nwords) dir[w0 + u * T] = vote_fields(plane[u], ranks, half);
  }
}

// ---------------------------------------------------------------- G3
// A group of 16 weights shares one 32-bit word of 2-bit direction fields.
// step = +lr (field 01), -lr (11), +0 (00; the unused 10 also moves nothing);
// W' = dtype_rn(fp32(W) - step), the subtraction rounded once in fp32.
__device__ __forceinline__ float step_of(uint32_t field, float lr) {
  return field == 1u ? lr : (field == 3u ? -lr : 0.0f);
}

constexpr int kUpdateU = 4;  // 16-weight groups per thread

// One 16-byte vector of W: 8 bf16 weights (fields in bits 0..15 of d) or 4
// fp32 weights (bits 0..7), element e taking field e.
template <bool kF32>
__device__ __forceinline__ void update_vec(uint4& v, uint32_t d, float lr) {
  if constexpr (!kF32) {
    uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __fsub_rn(__uint_as_float(u[j] << 16), step_of((d >> (4 * j)) & 3u, lr));
      const float hi = __fsub_rn(__uint_as_float(u[j] & 0xFFFF0000u), step_of((d >> (4 * j + 2)) & 3u, lr));
      const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
      u[j] = *reinterpret_cast<const uint32_t*>(&r);
    }
  } else {
    float* f = reinterpret_cast<float*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) f[j] = __fsub_rn(f[j], step_of((d >> (2 * j)) & 3u, lr));
  }
}

template <bool kF32>
__device__ __forceinline__ void update_group(uint4 (&v)[kF32 ? 4 : 2], uint32_t d, float lr) {
  constexpr int kBits = kF32 ? 8 : 16;  // direction bits per vector
#pragma unroll
  for (int i = 0; i < (kF32 ? 4 : 2); ++i) update_vec<kF32>(v[i], d >> (kBits * i), lr);
}

template <bool kF32>
__global__ void __launch_bounds__(kThreads) signsgd_update_kernel(uint4* __restrict__ W,
                                                                  const uint32_t* __restrict__ dir,
                                                                  int64_t ngroups, float lr) {
  pdl_wait_primary();
  pdl_launch_dependents();
  constexpr int kVecs = kF32 ? 4 : 2;  // 16-byte vectors per group
  const int64_t T = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t g0 = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; g0 < ngroups; g0 += kUpdateU * T) {
    uint4 v[kUpdateU][kVecs];
    uint32_t d[kUpdateU];
#pragma unroll
    for (int u = 0; u < kUpdateU; ++u) {
      const int64_t g = g0 + u * T;
      if (g < ngroups) {
        d[u] = __ldg(dir + g);
#pragma unroll
        for (int i = 0; i < kVecs; ++i) v[u][i] = W[g * kVecs + i];
      }
    }
#pragma unroll
    for (int u = 0; u < kUpdateU; ++u) {
      const int64_t g = g0 + u * T;
      if (g < ngroups) {
        update_group<kF32>(v[u], d[u], lr);
#pragma unroll
        for (int i = 0; i < kVecs; ++i) W[g * kVecs + i] = v[u][i];
      }
    }
  }
}

// ---------------------------------------------------------------- G2 + G3 + the sums of S1
// The holder's step in one sweep over W. A round is 32 consecutive word
// positions (32 x 32 weights); warp w of CTA b takes rounds w, w + kWarps, ...
// of the CTA's slice of positions. Lane l votes the R ranks' words of
// position l of the round, loads vectors l, l + 32, ... of the round's
// weights (each load and store of the warp one contiguous 512-byte block),
// takes each vector's direction bits from the lane that voted its position
// (a shuffle), updates the vector in place and adds |W'| as written into
// fp64 accumulator i mod 4 for its i-th vector. The CTA's partial sum is
// then formed as in S1's sum launch (the four accumulators pairwise, a
// butterfly over the lanes, the warps in order), so S1's code launch follows
// directly: gamma of W' needs sum |W'|, which this pass has in hand, and W'
// is the most recent data in L2. CTA 0 also clears the exact-sum counter
// and bins of the code launch.
//
// One CTA per SM with 64 KB of W in flight: 1024 threads for bf16 (4
// vectors a lane), 512 for f32 (8 vectors; the register budget of a thread
// doubles).
template <bool kF32>
constexpr int kApplyThreads = kF32 ? 512 : 1024;

struct ApplyArgs {
  const uint32_t* words;  // rank r's sign words at words + r * nwords
  int ranks;
  int64_t nwords;         // N * K / 32 word positions
  int64_t per;            // word positions per CTA slice (the last slices may be shorter or empty)
  uint4* W;               // [N, K] as 16-byte vectors, 32 weights per word position
  float lr;
  uint8_t* ws;            // S1 workspace
};

template <bool kF32>
__global__ void __launch_bounds__(kApplyThreads<kF32>, 1) signsgd_apply_kernel(const __grid_constant__ ApplyArgs a) {
  constexpr int kVecs = kF32 ? 8 : 4;  // 16-byte vectors per word position
  constexpr int T = kApplyThreads<kF32>;
  constexpr int kWarps = T / 32;
  __shared__ double s_red[kWarps];
  pdl_wait_primary();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, t = threadIdx.x;
  const int64_t b = blockIdx.x;
  if (b == 0) {
    unsigned long long* bins = reinterpret_cast<unsigned long long*>(a.ws + kWsBins);
    for (int e = t; e < 256; e += T) bins[e] = 0ull;
    if (t == 0) *reinterpret_cast<uint32_t*>(a.ws + kWsArrive) = 0u;
  }
  const uint32_t half = static_cast<uint32_t>(a.ranks) >> 1;
  const int64_t w0 = b * a.per;
  const int64_t wend = w0 + a.per < a.nwords ? w0 + a.per : a.nwords;
  const int64_t vend = wend * kVecs;
  const int part = lane % kVecs;  // which kVecs-th of a position's weights lane's vectors hold
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int64_t base = w0 + 32 * warp; base < wend; base += T) {
    // the round's 32 positions are 32 kVecs consecutive vectors; lane l
    // holds vectors l + 32 i (one 512-byte block of the warp per i)
    const int64_t vbase = base * kVecs;
    uint4 v[kVecs];
#pragma unroll
    for (int i = 0; i < kVecs; ++i) {
      const int64_t j = vbase + lane + 32 * i;
      v[i] = j < vend ? a.W[j] : make_uint4(0u, 0u, 0u, 0u);
    }
    // lane l votes position base + l
    uint32_t plane[kVotePlanes];
#pragma unroll
    for (int p = 0; p < kVotePlanes; ++p) plane[p] = 0u;
    const bool votes = base + lane < wend;
    for (int r = 0; r < a.ranks; ++r) {
      uint32_t carry = votes ? __ldg(a.words + static_cast<int64_t>(r) * a.nwords + base + lane) : 0u;
#pragma unroll
      for (int p = 0; p < kVotePlanes; ++p) {
        const uint32_t c = plane[p] & carry;
        plane[p] ^= carry;
        carry = c;
      }
    }
    const uint2 d = vote_fields(plane, a.ranks, half);
#pragma unroll
    for (int i = 0; i < kVecs; ++i) {
      // vector l + 32 i of the round belongs to position (l + 32 i) / kVecs
      const int src = (lane + 32 * i) / kVecs;
      const uint32_t dx = __shfl_sync(0xffffffffu, d.x, src);
      const uint32_t dy = __shfl_sync(0xffffffffu, d.y, src);
      const uint32_t f = part < kVecs / 2 ? dx : dy;
      update_vec<kF32>(v[i], f >> ((64 / kVecs) * (part % (kVecs / 2))), a.lr);
      const int64_t j = vbase + lane + 32 * i;
      if (j < vend) {
        acc[i & 3] = add_abs<kF32>(acc[i & 3], v[i]);
        a.W[j] = v[i];
      }
    }
  }
  double ts = __dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ts = __dadd_rn(ts, __shfl_xor_sync(0xffffffffu, ts, off));
  if (lane == 0) s_red[warp] = ts;
  __syncthreads();
  if (t == 0) {
    double p = 0.0;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) p = __dadd_rn(p, s_red[i]);
    reinterpret_cast<double*>(a.ws + kWsParts)[b] = p;
  }
}

// Blocks for `items` work items taken `per_thread` to a thread, at most eight
// 256-thread blocks per SM (one wave).
unsigned stream_blocks(int64_t items, int per_thread) {
  const int64_t threads = (items + per_thread - 1) / per_thread;
  const int64_t want = (threads + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(8) * device_sm_count();
  return static_cast<unsigned>(want < cap ? want : cap);
}

}  // namespace

cudaError_t launch_sign_pack(const void* dW, int dw_is_f32, int64_t N, int64_t K, uint32_t* out, cudaStream_t s) {
  const int64_t nwords = N * K / 32;
  const uint4* p = static_cast<const uint4*>(dW);
  const dim3 grid(stream_blocks(nwords, kPackU));
  cudaError_t e = dw_is_f32 ? launch_pdl(sign_pack_kernel<true>, grid, dim3(kThreads), 0, s, p, nwords, out)
                            : launch_pdl(sign_pack_kernel<false>, grid, dim3(kThreads), 0, s, p, nwords, out);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_sign_vote(const uint32_t* words, int ranks, int64_t N, int64_t K, uint8_t* direction,
                             cudaStream_t s) {
  const int64_t nwords = N * K / 32;
  cudaError_t e = launch_pdl(sign_vote_kernel, dim3(stream_blocks(nwords, kVoteU)), dim3(kThreads), 0, s, words,
                             ranks, nwords, reinterpret_cast<uint2*>(direction));
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_signsgd_update(void* W, int w_is_f32, int64_t N, int64_t K, const uint8_t* direction, float lr,
                                  cudaStream_t s) {
  const int64_t ngroups = N * K / 16;
  uint4* p = static_cast<uint4*>(W);
  const uint32_t* d = reinterpret_cast<const uint32_t*>(direction);
  const dim3 grid(stream_blocks(ngroups, kUpdateU));
  cudaError_t e = w_is_f32 ? launch_pdl(signsgd_update_kernel<true>, grid, dim3(kThreads), 0, s, p, d, ngroups, lr)
                           : launch_pdl(signsgd_update_kernel<false>, grid, dim3(kThreads), 0, s, p, d, ngroups, lr);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_signsgd_apply(const uint32_t* words, int ranks, void* W, int w_is_f32, int64_t N, int64_t K,
                                 float lr, uint8_t* packed, float* gamma, void* workspace, int* err, cudaStream_t s) {
  const int64_t nwords = N * K / 32;
  const int T = w_is_f32 ? kApplyThreads<true> : kApplyThreads<false>;
  // one CTA per SM (at most kMaxQuantCtas partial sums), fewer when W has
  // fewer word positions than that many threads
  const int64_t cap = std::min<int64_t>(device_sm_count(), kMaxQuantCtas);
  const int64_t want = (nwords + T - 1) / T;
  const int64_t G = std::max<int64_t>(1, std::min(cap, want));
  ApplyArgs aa{};
  aa.words = words;
  aa.ranks = ranks;
  aa.nwords = nwords;
  aa.per = ((nwords + G - 1) / G + 31) / 32 * 32;  // whole rounds of 32 positions
  aa.W = static_cast<uint4*>(W);
  aa.lr = lr;
  aa.ws = static_cast<uint8_t*>(workspace);
  // Roundings of a term inside its partial sum: 8 adds into its accumulator
  // per round of the lane's warp (ceil(per / T) of them), the two levels
  // joining the four accumulators, the 5 butterfly levels and the T / 32
  // sequential warp sums.
  const int64_t nj = (aa.per + T - 1) / T;
  const double part_roundings = 8.0 * static_cast<double>(nj) + 2 + 5 + T / 32;
  cudaError_t e = w_is_f32 ? launch_pdl(signsgd_apply_kernel<true>, dim3(static_cast<unsigned>(G)), dim3(T), 0, s, aa)
                           : launch_pdl(signsgd_apply_kernel<false>, dim3(static_cast<unsigned>(G)), dim3(T), 0, s, aa);
  if (e != cudaSuccess) return e;
  return launch_quantize_codes(W, w_is_f32, N, K, static_cast<int>(G), part_roundings, packed, gamma, workspace, err,
                               s);
}

}  // namespace bl
