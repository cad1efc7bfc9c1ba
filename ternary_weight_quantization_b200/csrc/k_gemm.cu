// S3 and S4 of the BitLinear hot path on sm_100a: the INT32-exact forward GEMM
// and the two straight-through backward GEMMs ("bitnet-qat-train", Semantics:
// y = quant(x) . ternarize(W)^T . s_x . gamma; dX = dY . W_hat;
// dW = dY^T . x_hat, with W_hat and x_hat rebuilt from the saved 2-bit and
// INT8 state).
//
// One persistent, warp-specialised CTA-pair kernel template serves all three:
//
//   D[i][j] = sum_r A[i][r] * B[j][r]        (tcgen05.mma cta_group::2, TMEM accumulators)
//   out[j][i] = epilogue(D[i][j])            (i contiguous in the output)
//
//   op   A (REBUILT in smem)                    B (TMA)                       r
//   Fwd  codes[n][k] int8, K-major              xq[m][k] int8, K-major        k
//   Dx   2 codes^T[k][n] bf16 {-2,0,2}, MN-major dY[m][n] bf16, K-major        n
//   Dw   x_hat^T[k][m] bf16, MN-major           dY^T[n][m] bf16, MN-major     m
//
// A pair tile is 256 A rows x BN B rows. Each CTA of the pair rebuilds its own
// 128 A rows from the staged 2-bit / INT8 source (never written to HBM) and
// TMA-loads its own BN/2 B rows; the leader CTA issues one M=256 MMA that
// reads both CTAs' shared memory and accumulates 128 rows into each CTA's
// TMEM. No TMA multicast is used. Forward tiles wider than one MMA (BN = 320,
// for shapes with a few more tiles than pairs) issue two MMAs of BN/2 columns
// per step on the same A -- columns 0..BN/2-1 and BN/2..BN-1 -- into one
// accumulator of BN columns (the two-buffer overlap of epilogue and MMAs
// needs BN <= 256).
//
// The forward family runs one GEMM per launch. The backward family runs dX
// and dW in ONE launch: the two GEMMs' tiles (different lengths: N/64 and M/64
// k-blocks) are spread over the CTA pairs by a longest-processing-time
// schedule computed on the host and passed in the kernel parameters, so the
// pairs finish together instead of idling through a partly filled last wave.
// Given a workspace and N >= 2048, a launch before it writes x_hat once
// (xhat_kernel) and dW's stages load their A operand from there by TMA
// instead of rebuilding it (every dW tile would rebuild its x_hat slab).
//
// Warp w runs on SM sub-partition w % 4. Roles (512 threads per CTA):
//   warp 0      loads: TMA for B, for Dw's q / s_x and for the packed codes
//               (cp.async for the codes when K % 64 != 0: their rows are then
//               not 16-byte aligned, which a tensor map requires)
//   warp 1      TMEM allocation (512 columns, pair-wide); in the leader
//               CTA one lane issues the tcgen05.mma
//   warps 2-4, 6-8, 10-11  rebuild A from the staged source, in two groups
//               of four taking alternate stages
//   warps 5, 9  idle (keeps sub-partition 1 to the MMA warp: rebuild warps
//               there would compete with it for issue slots)
//   warps 12-15 epilogue: TMEM -> registers -> bf16/f32 box in smem -> TMA store
// Barriers: src_full (per CTA: staged source landed), full (leader: both
// CTAs' B bytes landed and both CTAs' A rebuilt -- one wait per stage for the
// MMA lane), empty and tmem_full (both CTAs, completed by multicast
// tcgen05.commit), tmem_empty (leader: both CTAs' epilogues drained a TMEM
// buffer). The MMA lane's loop is kept minimal because the tensor core's
// instruction queue is shallow: the next stage's MMAs must be issued while
// the current stage's last MMA still executes. Every wait is bounded: on
// expiry a CTA records a timeout in the device error word, tells its peer,
// drains what it has in flight, frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdarg>
#include <cstddef>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "bl_device.cuh"
#include "bl_internal.h"

namespace bl {
namespace {

constexpr int kThreads = 512;
constexpr int kWarpLoad = 0;
constexpr int kWarpMma = 1;
constexpr int kNumRebuildWarps = 8;  // warps 2, 3, 4, 6, 7, 8, 10, 11
// The rebuild warps form two groups of four that take alternate pipeline
// stages, so one group's fixed per-stage latency (shared loads, proxy fence,
// barrier arrival) overlaps the other's work.
constexpr int kRebuildGroups = 2;
constexpr int kRebuildThreads = 32 * kNumRebuildWarps / kRebuildGroups;  // threads per stage
constexpr int kWarpEpi0 = 12;        // warps 12..15 (TMEM lane quadrants 0..3)
constexpr int kNumEpiWarps = 4;

// Rebuild slot of warp w (0..7), or -1 (warps 0, 1, 5, 9 and 12..15).
__device__ __forceinline__ int rebuild_slot(int w) {
  if (w < 2 || w >= kWarpEpi0 || (w & 3) == 1) return -1;
  return w - 2 - (w >= 6) - (w >= 10);
}

constexpr int BM = 128;              // A rows per CTA; a pair covers 2 * BM
constexpr uint32_t kTmemCols = 512;  // two accumulators at columns 0 and 256 (one of BN for BN > 256)
constexpr int kSmemLimit = 232448;           // per-CTA dynamic shared memory on sm_100
constexpr int kMaxPairs = 128;
constexpr int kMaxSchedTiles = 2048;

enum class Op { Fwd, Dx, Dw };
enum class Family { Fwd, Bwd };

// TMEM accumulators a pair cycles through: two of 256 columns, or one of BN
// columns for the wide forward tiles.
template <int BN>
constexpr int kAccBufs = BN > 256 ? 1 : 2;
// Wide forward tiles: this CTA's B rows 0..BN/4-1 hold tokens
// bp + (BN/4) r + ... (the first MMA's half for rank r) and rows BN/4..BN/2-1
// hold tokens bp + BN/2 + (BN/4) r + ... (the second MMA's), so accumulator
// column c is token bp + c; each half arrives in one box of BN/4 rows.
template <int BN>
constexpr int kWideBox = BN > 256 ? BN / 4 : BN / 2;

// Stage geometry of a family. Every op issues four MMAs per stage.
template <Family F, int BN>
struct Geo;

// Epilogue staging per warp: kEpiSlots boxes of 32 x 32 bf16 (2 KB each);
// an f32 box takes two slots.
// Forward: reduction over k in blocks of 128 bytes; kind::i8 consumes 32 k per MMA.
template <int BN>
struct Geo<Family::Fwd, BN> {
  // 320-column tiles: two staging slots per epilogue warp leave room for a
  // fifth pipeline stage (four with four slots); measured on B200 at the
  // down-projection 35.5 -> 33.7 us
  static constexpr int kEpiSlots = BN > 256 ? 2 : 4;
  static constexpr int kEpiScaleBytes = (BN > 256 ? BN : 256) * 4;  // s_x[m] * gamma of the tile's columns
  static constexpr int kBlockR = 128;
  static constexpr int kABytes = BM * 128;         // 128 rows x 128 int8
  static constexpr int kBBytes = (BN / 2) * 128;   // BN/2 rows x 128 int8
  static constexpr int kSrcBytes = BM * 32;        // packed: 128 rows x 32 bytes
  static constexpr int kSxBytes = 0;
};

// Backward: reduction blocks of 64 (n for dX, m for dW); kind::f16 consumes
// 16 per MMA. The source slot fits dW's q tile (64 x 128 int8, swizzled) and
// dX's packed tile (64 rows x 32 bytes). dW's B is MN-major: BN/2 must be a
// multiple of 64 (whole 128-byte swizzle atoms).
template <int BN>
struct Geo<Family::Bwd, BN> {
  static_assert((BN / 2) % 64 == 0, "MN-major B needs whole 64-element chunks");
  static constexpr int kEpiSlots = 2;
  static constexpr int kEpiScaleBytes = 0;
  static constexpr int kBlockR = 64;
  static constexpr int kABytes = BM * 64 * 2;      // 128 x 64 bf16
  static constexpr int kBBytes = (BN / 2) * 128;   // BN/2 x 64 bf16
  static constexpr int kSrcBytes = 64 * 128;
  static constexpr int kSxBytes = 64 * 4;
};

// Per-op MMA operand formats: instruction descriptor, descriptor leading byte
// offsets and the per-MMA step of each operand's start address (16-byte units).
template <Op op, int BN>
struct MmaCfg;
template <int BN>
struct MmaCfg<Op::Fwd, BN> {
  // BN > 256: two MMAs of N = BN/2, on B rows 0..BN/4-1 and BN/4..BN/2-1 of
  // each CTA (columns 0.. and BN/2.. of the accumulator). Measured on B200
  // against one of N = 256 and one of N = BN - 256: down-projection forward
  // 37.3 -> 35.9 us (y bit-identical).
  static constexpr uint32_t kIdesc = make_idesc(2 /*s32*/, 1 /*s8*/, 0, 0, 2 * BM, BN > 256 ? BN / 2 : BN);
  static constexpr uint32_t kIdesc2 = make_idesc(2, 1, 0, 0, 2 * BM, BN > 256 ? BN / 2 : 16);
  static constexpr uint32_t kLboA = 16, kLboB = 16;
  static constexpr uint64_t kStepA = 2, kStepB = 2;  // 32 bytes of K (K-major)
};
template <int BN>
struct MmaCfg<Op::Dx, BN> {
  static constexpr uint32_t kIdesc = make_idesc(1 /*f32*/, 1 /*bf16*/, 1 /*A MN*/, 0, 2 * BM, BN);
  static constexpr uint32_t kLboA = 8192, kLboB = 16;
  static constexpr uint64_t kStepA = 128, kStepB = 2;  // 16 rows (MN-major) / 32 bytes (K-major)
};
template <int BN>
struct MmaCfg<Op::Dw, BN> {
  static constexpr uint32_t kIdesc = make_idesc(1, 1, 1 /*A MN*/, 1 /*B MN*/, 2 * BM, BN);
  static constexpr uint32_t kLboA = 8192, kLboB = 8192;
  static constexpr uint64_t kStepA = 128, kStepB = 128;
};

template <Family F, int BN>
struct Layout {
  using G = Geo<F, BN>;
  static constexpr int kStageBytes = G::kABytes + G::kBBytes + G::kSrcBytes + G::kSxBytes;
  static constexpr int kEpiStageBytes = G::kEpiSlots * 2048 + G::kEpiScaleBytes;  // per epilogue warp
  static constexpr int kReserve = 1024 /*base alignment*/ + kNumEpiWarps * kEpiStageBytes + 512;
  static constexpr int kS0 = (kSmemLimit - kReserve) / kStageBytes;
  static constexpr int kS = kS0 > 8 ? 8 : kS0;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kS * G::kABytes;
  static constexpr int kOffSrc = kOffB + kS * G::kBBytes;
  static constexpr int kOffSx = kOffSrc + kS * G::kSrcBytes;
  static constexpr int kOffEpi = kOffSx + kS * G::kSxBytes;
  static constexpr int kOffBar = kOffEpi + kNumEpiWarps * kEpiStageBytes;
  // src_full[S], full[S], empty[S], tmem_full[2], tmem_empty[2], done
  static constexpr int kNumBars = 3 * kS + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  static constexpr int kDynBytes = kBytes + 1024;
  static_assert(kS >= 2, "at least two pipeline stages");
  static_assert(12 * kEpiStageBytes <= kOffEpi, "warps 0..11 stage the last tile's epilogue in the operand stages");
  static_assert(kDynBytes <= kSmemLimit, "shared memory budget");
  static_assert(G::kABytes % 1024 == 0 && G::kBBytes % 1024 == 0 && G::kSrcBytes % 1024 == 0, "alignment");
};

// One GEMM of a launch.
struct OpParams {
  int rows_a;     // extent of the A-row index i (N for Fwd, K for Dx/Dw)
  int rows_b;     // extent of the B-row index j (M for Fwd/Dx, N for Dw)
  int red;        // reduction length (K, N, M)
  int tiles_a, num_kb, ntiles;
  void* out;      // [rows_b][ldo]
  int64_t ldo;
  int out_f32;    // Dw
  int accumulate; // Dw
  int src_tma;    // Fwd/Dx: packed codes by TMA (K % 64 == 0) instead of cp.async
  int tma_store;  // output through the TMA store map of this op
  int sign_words; // Dw: out receives the sign bits of dW (32 per word along K) instead of dW
  int xhat_tma;   // Dw: A = x_hat^T loaded by TMA from a bf16 [M][K] copy made before the launch
                  // (the source map), instead of rebuilt from q and s_x in every tile
};

struct GemmParams {
  OpParams op[2];         // Fwd: op[0]; Bwd: op[0] = dX, op[1] = dW (either may have 0 tiles)
  int ntiles;             // op[0].ntiles + op[1].ntiles
  int64_t K;              // in_features (row length of packed codes / q)
  const uint8_t* packed;  // Fwd, Dx
  const float* sx;        // Fwd epilogue
  const float* gamma;     // Fwd, Dx epilogue
  int32_t* debug_acc;     // Fwd, optional
  int* err;
  int use_sched;          // 1: pair p runs sched_tile[sched_start[p] .. sched_start[p+1])
                          // 0: pair p runs tiles p, p + npairs, ...
  uint16_t sched_start[kMaxPairs + 1];
  uint16_t sched_tile[kMaxSchedTiles];
};

struct TileInfo {
  int opi;  // index into GemmParams::op
  int a0;   // first A row of this CTA
  int bp;   // first B row of the pair tile
};

__device__ __forceinline__ bool next_tile(const GemmParams& p, int pair, int npairs, int i, int& tile) {
  if (p.use_sched) {
    const int idx = p.sched_start[pair] + i;
    if (idx >= p.sched_start[pair + 1]) return false;
    tile = p.sched_tile[idx];
  } else {
    tile = pair + i * npairs;
    if (tile >= p.ntiles) return false;
  }
  return true;
}

template <int BN>
__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, int tile, uint32_t rank) {
  TileInfo t;
  t.opi = tile >= p.op[0].ntiles ? 1 : 0;
  const int u = tile - (t.opi ? p.op[0].ntiles : 0);
  const OpParams& P = p.op[t.opi];
  t.a0 = (u % P.tiles_a) * (2 * BM) + static_cast<int>(rank) * BM;
  t.bp = (u / P.tiles_a) * BN;
  return t;
}

// ---------------------------------------------------------------- rebuild helpers

// Two bytes of four 2-bit fields each, already placed in bytes 0 and 2 of x
// -> nibble i holds field i.
__device__ __forceinline__ uint32_t spread_fields8(uint32_t x) {
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  x = (x | (x << 2)) & 0x33333333u;
  return x;
}

// 16 packed codes (one 32-bit word) -> 16 int8 codes. One byte permutation
// places each byte pair of w in bytes 0 and 2 (the first spreading step),
// two shift/mask steps spread the fields to nibbles, and a byte permutation
// per four codes looks each nibble up in a 4-entry table. The rebuild of the
// forward operand is ALU-bound on its SM sub-partitions, so every step counts.
__device__ __forceinline__ uint4 codes16_to_s8(uint32_t w) {
  constexpr uint32_t kTable = 0xFFFE0100u;  // field 0 -> 0, 1 -> +1, 2 -> -2 (unused), 3 -> -1
  const uint32_t lo = spread_fields8(__byte_perm(w, 0u, 0x4140));  // bytes 0, 1 of w
  const uint32_t hi = spread_fields8(__byte_perm(w, 0u, 0x4342));  // bytes 2, 3 of w
  uint4 r;
  r.x = __byte_perm(kTable, 0u, lo & 0xFFFFu);
  r.y = __byte_perm(kTable, 0u, lo >> 16);
  r.z = __byte_perm(kTable, 0u, hi & 0xFFFFu);
  r.w = __byte_perm(kTable, 0u, hi >> 16);
  return r;
}

// 8 packed codes (16 bits) -> 8 bf16 values 2 * code in {-2, 0, +2}. With
// the factor 2 the map is linear in the 2-bit field: bf16 2.0 is 0x4000 and
// -2.0 is 0xC000, i.e. field f in {0, 1, 3} -> f * 0x4000, so each field only
// moves to bits 14-15 of its half (one shift and one mask per two codes). The
// dX epilogue scales by gamma / 2 (exact), and (2 acc) * (gamma / 2) is
// acc * gamma exactly, so dX is unchanged: every product and partial sum of
// the doubled operand is exactly twice the plain one.
__device__ __forceinline__ uint4 codes8_to_bf16x2(uint32_t h) {
  h &= 0xFFFFu;
  // field 2w at bits 4w, 4w+1; field 2w+1 at bits 4w+16, 4w+17 (bits 14-15
  // hold two fields at once but are never selected)
  const uint32_t s = h | (h << 14);
  return make_uint4((s << 14) & 0xC000C000u, (s << 10) & 0xC000C000u, (s << 6) & 0xC000C000u,
                    (s << 2) & 0xC000C000u);
}

// 16 int8 (x_hat source) * s -> 16 bf16, each bf16_rn(fp32(q) * s).
// fp32(q) uses the 2^23 shifter: bits 0x4B0000uu are 2^23 + u with
// u = q + 128, so subtracting 2^23 + 128 is exact. The subtraction and the
// product by s run on pairs (packed fp32x2, each lane rounded like the scalar
// instruction).
__device__ __forceinline__ uint64_t f32x2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint32_t f32x2_to_bf16x2(uint64_t v) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "r"(static_cast<uint32_t>(v >> 32)), "r"(static_cast<uint32_t>(v)));
  return r;
}

__device__ __forceinline__ void s8x16_to_bf16(const uint4& v, float s, uint4& o0, uint4& o1) {
  const uint32_t w[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u, v.w ^ 0x80808080u};
  constexpr uint64_t kShift2 = 0x4B0000804B000080ull;  // {2^23 + 128, 2^23 + 128}
  const uint64_t s2 = (static_cast<uint64_t>(__float_as_uint(s)) << 32) | __float_as_uint(s);
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int b = 0; b < 4; b += 2) {
      const uint32_t lo = __byte_perm(w[i], 0x4B000000u, 0x7440u | b);
      const uint32_t hi = __byte_perm(w[i], 0x4B000000u, 0x7440u | (b + 1));
      const uint64_t q2 = f32x2_sub((static_cast<uint64_t>(hi) << 32) | lo, kShift2);
      out[i * 2 + b / 2] = f32x2_to_bf16x2(f32x2_mul(q2, s2));
    }
  }
  o0 = make_uint4(out[0], out[1], out[2], out[3]);
  o1 = make_uint4(out[4], out[5], out[6], out[7]);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// ---------------------------------------------------------------- per-op stage work

struct Maps {
  const CUtensorMap* b;
  const CUtensorMap* src;
  const CUtensorMap* sx;
};

// Load warp, one stage: this CTA's B rows (pair TMA, counted on the leader's
// `full`), and the source of its A rows (counted on the local `src_full`,
// which expects one arrival).
template <Op op, Family F, int BN, bool kLean>
__device__ __forceinline__ void load_stage(const GemmParams& p, const OpParams& P, const Maps& m, bool leader,
                                           int lane, int a0, int bp, int bh, int kb, uint64_t* full, uint32_t full_lead,
                                           uint64_t* src_full, uint8_t* sA, uint8_t* sB, uint8_t* sSrc, uint8_t* sSx) {
  using G = Geo<F, BN>;
  const int r0 = kb * G::kBlockR;
  const int kq = static_cast<int>(p.K / 4);
  if (lane == 0) {
    if (leader) mbar_arrive_expect_tx(full, 2 * G::kBBytes);
    if constexpr (op == Op::Dw) {
#pragma unroll
      for (int j = 0; j < (BN / 2) / 64; ++j) tma_load_2d_pair(m.b, full_lead, sB + j * 8192, bh + 64 * j, r0);
      if (kLean || P.xhat_tma) {
        // A itself: two 64 (k) x 64 (m) bf16 boxes of x_hat, 128-byte
        // swizzled exactly as the rebuild writes them
        mbar_arrive_expect_tx(src_full, 2 * 64 * 128);
        tma_load_2d(m.src, src_full, sA, a0, r0);
        tma_load_2d(m.src, src_full, sA + 8192, a0 + 64, r0);
      } else {
        mbar_arrive_expect_tx(src_full, 64 * 128 + 64 * 4);
        tma_load_2d(m.src, src_full, sSrc, a0, r0);
        tma_load_2d(m.sx, src_full, sSx, r0, 0);
      }
    } else {
      if constexpr (op == Op::Fwd && BN > 256) {
        static_assert(2 * kWideBox<BN> == BN / 2 && (kWideBox<BN> * 128) % 1024 == 0,
                      "each MMA's rows come in one box, at a whole swizzle atom");
        const int r = (bh - bp) / (BN / 2);  // rank of this CTA
        tma_load_2d_pair(m.b, full_lead, sB, r0, bp + kWideBox<BN> * r);
        tma_load_2d_pair(m.b, full_lead, sB + kWideBox<BN> * 128, r0, bp + BN / 2 + kWideBox<BN> * r);
      } else {
        tma_load_2d_pair(m.b, full_lead, sB, r0, bh);
      }
      if (kLean || P.src_tma) {
        // packed codes as one TMA box: Fwd rows a0..a0+127 x bytes [kb*32, +32);
        // Dx rows (n) r0..r0+63 x bytes [a0/4, +32)
        if constexpr (op == Op::Fwd) {
          mbar_arrive_expect_tx(src_full, BM * 32);
          tma_load_2d(m.src, src_full, sSrc, kb * 32, a0);
        } else {
          mbar_arrive_expect_tx(src_full, 64 * 32);
          tma_load_2d(m.src, src_full, sSrc, a0 / 4, r0);
        }
      }
    }
  }
  if constexpr (op != Op::Dw && !kLean) {
    if (!P.src_tma) {
      // packed codes by 8-byte cp.async (rows not 16-byte aligned), placed in
      // the 32-byte-swizzled layout the TMA path produces; every lane's copies
      // hold the phase open until they land, lane 0 gives the one arrival
      constexpr int kChunks = (op == Op::Fwd) ? 16 : 8;  // per lane
#pragma unroll
      for (int it = 0; it < kChunks; ++it) {
        const int c = lane + 32 * it;
        const int row = c >> 2, part = c & 3;
        bool valid;
        const uint8_t* src;
        if constexpr (op == Op::Fwd) {
          // packed rows a0..a0+127, bytes [kb*32, kb*32+32)
          valid = (a0 + row < P.rows_a) && (r0 + part * 32 < P.red);
          src = p.packed + static_cast<int64_t>(a0 + row) * kq + kb * 32 + part * 8;
        } else {
          // packed rows (n) r0..r0+63, bytes covering k in [a0, a0+128)
          valid = (r0 + row < P.red) && (a0 + part * 32 < P.rows_a);
          src = p.packed + static_cast<int64_t>(r0 + row) * kq + a0 / 4 + part * 8;
        }
        const int dst = row * 32 + ((((part >> 1) ^ (row >> 2)) & 1) << 4) + ((part & 1) << 3);
        cp_async_8(sSrc + dst, valid ? src : p.packed, valid ? 8u : 0u);
      }
      cp_async_mbar_arrive(src_full);
      __syncwarp();
      if (lane == 0) mbar_arrive(src_full);
    }
  }
}

// Rebuild group (128 threads), one stage: A rows of this CTA from the staged source.
template <Op op, Family F, int BN>
__device__ __forceinline__ void rebuild_stage(int rt, uint32_t sA, uint32_t sSrc, const float* sSx) {
  if constexpr (op == Op::Fwd) {
    // row rt: 32 packed bytes -> 128 int8 codes, K-major with 128-byte swizzle.
    // The staged rows are 32-byte swizzled (16-byte half c of row r at c ^ bit
    // 2 of r), so lanes 0..3 and 4..7 of each group of 8 read different banks.
    const uint32_t h = (rt >> 2) & 1;
    const uint4 w0 = ld_shared_v4(sSrc + rt * 32 + h * 16);        // codes 0..63
    const uint4 w1 = ld_shared_v4(sSrc + rt * 32 + (h ^ 1) * 16);  // codes 64..127
    const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const uint32_t row_base = sA + rt * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) st_shared_v4(row_base + ((c ^ (rt & 7)) << 4), codes16_to_s8(words[c]));
  } else if constexpr (op == Op::Dx) {
    // reduction row n = rt % 64, output k half = rt / 64 (64 k values); the
    // staged rows are 32-byte swizzled like the forward's
    const int n = rt & 63, half = rt >> 6;
    const uint4 w = ld_shared_v4(sSrc + n * 32 + ((half ^ ((n >> 2) & 1)) << 4));
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    const uint32_t base = sA + half * 8192 + n * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t hw = words[j >> 1] >> ((j & 1) * 16);
      st_shared_v4(base + ((j ^ (n & 7)) << 4), codes8_to_bf16x2(hw));
    }
  } else {
    // token m = rt % 64, k half = rt / 64; q staging is 128-byte swizzled
    const int m = rt & 63, half = rt >> 6;
    const float s = sSx[m];
    const uint32_t base = sA + half * 8192 + m * 128;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = half * 4 + i;  // logical 16-byte chunk (16 k values)
      const uint4 v = ld_shared_v4(sSrc + m * 128 + ((c ^ (m & 7)) << 4));
      uint4 o0, o1;
      s8x16_to_bf16(v, s, o0, o1);
      const int j0 = 2 * i, j1 = 2 * i + 1;  // 8-k units within this half
      st_shared_v4(base + ((j0 ^ (m & 7)) << 4), o0);
      st_shared_v4(base + ((j1 ^ (m & 7)) << 4), o1);
    }
  }
}

// MMA lane, one stage: four pair MMAs (eight for the wide forward tiles).
template <Op op, int BN>
__device__ __forceinline__ void mma_stage(uint32_t d_tmem, uint32_t sa, uint32_t sb, int kb) {
  using M = MmaCfg<op, BN>;
  const uint64_t ad = smem_desc_sw128(sa, M::kLboA, 1024);
  const uint64_t bd = smem_desc_sw128(sb, M::kLboB, 1024);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint32_t acc = (kb | kk) != 0;
    if constexpr (op == Op::Fwd) {
      mma_i8_pair(d_tmem, ad + kk * M::kStepA, bd + kk * M::kStepB, M::kIdesc, acc);
      if constexpr (BN > 256) {
        const uint64_t bd2 = smem_desc_sw128(sb + kWideBox<BN> * 128, M::kLboB, 1024);
        mma_i8_pair(d_tmem + BN / 2, ad + kk * M::kStepA, bd2 + kk * M::kStepB, M::kIdesc2, acc);
      }
    } else
      mma_f16_pair(d_tmem, ad + kk * M::kStepA, bd + kk * M::kStepB, M::kIdesc, acc);
  }
}

// Epilogue value of accumulator word `a`: the forward scales the exact INT32
// sum by s_x[m] * gamma, dX by gamma / 2 (its sum is over 2 * code); dW is
// the fp32 sum.
template <Op op>
__device__ __forceinline__ float epi_value(uint32_t a, float scale) {
  if constexpr (op == Op::Fwd) return __fmul_rn(static_cast<float>(static_cast<int32_t>(a)), scale);
  else if constexpr (op == Op::Dx) return __fmul_rn(__uint_as_float(a), scale);
  else return __uint_as_float(a);
}

// Largest K for which every forward accumulator (|acc| <= 127 K) is below
// 2^22, the range of the exact 1.5 * 2^23 int -> float shifter.
constexpr int kShifterMaxK = 33024;

// {hi, lo} -> bf16x2 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t cvt_bf16x2(float hi, float lo) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void st_shared_b16(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(static_cast<unsigned short>(v)) : "memory");
}

__device__ __forceinline__ uint64_t pair_u64(uint32_t lo, uint32_t hi) {
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Epilogue paths taken for f32 output, accumulation, the debug output and
// row pitches a tensor map cannot take: kept out of line so that the common
// bf16 path stays small in the instruction caches.
// f32 box through the warp's whole 4 KB staging slot.
template <Op op>
__device__ __noinline__ void epilogue_chunk_f32(const CUtensorMap* out_map, const uint32_t* r, uint32_t stg, int lane,
                                                int i0, int j0) {
  if (lane == 0) bulk_wait_group_read<0>();  // the previous box has been read
  __syncwarp();
  for (int jj = 0; jj < 32; ++jj) st_shared_b32(stg + jj * 128 + lane * 4, __float_as_uint(epi_value<op>(r[jj], 0.0f)));
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(out_map, stg, i0, j0);
    bulk_commit_group();
  }
}

// Direct stores: lane i writes column i of each row j (the warp's 32 lanes
// write contiguous elements of one row).
template <Op op>
__device__ __noinline__ void epilogue_chunk_direct(const GemmParams& p, const OpParams& P, const uint32_t* r, int lane,
                                                   int i0, int j0, float col_scale, float gamma) {
  const int i = i0 + lane;
  for (int jj = 0; jj < 32; ++jj) {
    float scale = 0.0f;
    if constexpr (op == Op::Fwd) scale = __shfl_sync(0xffffffffu, col_scale, jj);
    else if constexpr (op == Op::Dx) scale = gamma;
    const int j = j0 + jj;
    if (i >= P.rows_a || j >= P.rows_b) continue;
    const int64_t off = static_cast<int64_t>(j) * P.ldo + i;
    float v = epi_value<op>(r[jj], scale);
    if constexpr (op == Op::Fwd) {
      if (p.debug_acc) p.debug_acc[off] = static_cast<int32_t>(r[jj]);
    }
    if (P.out_f32) {
      float* o = static_cast<float*>(P.out) + off;
      if (P.accumulate) v = __fadd_rn(v, *o);
      *o = v;
    } else {
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(P.out) + off;
      if (P.accumulate) v = __fadd_rn(v, __bfloat162float(*o));
      *o = __float2bfloat16_rn(v);
    }
  }
}

// Sign bits of dW instead of dW: lane = k (i0 + lane), r[jj] = the fp32 sum
// of dW[j0 + jj][k]. Rounding to bf16 or fp32 keeps the sign (-0 included),
// so the sign bit of the sum is the sign bit of dW; one ballot per row gives
// the row's 32 bits for k = i0 .. i0 + 31 (bit l = k i0 + l), which is word
// (j K + i0) / 32 of the flattened [N, K] sign words. Lane jj writes row
// j0 + jj's word.
__device__ __forceinline__ void epilogue_chunk_signs(const OpParams& P, const uint32_t (&r)[32], int lane, int i0,
                                                     int j0) {
  uint32_t mine = 0;
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) {
    const uint32_t w = __ballot_sync(0xffffffffu, (r[jj] >> 31) != 0u);
    mine = lane == jj ? w : mine;
  }
  const int j = j0 + lane;
  if (j < P.rows_b) static_cast<uint32_t*>(P.out)[static_cast<int64_t>(j) * (P.ldo / 32) + i0 / 32] = mine;
}

// Epilogue, one 32 x 32 chunk in registers: lane = output column i (A row),
// r[jj] = output row j0 + jj. The common case is a bf16 box converted into
// one of the warp's kSlots 2 KB staging slots (used in turn) and written by
// one TMA store. `seq` counts the warp's bf16 boxes.
template <Op op, int kSlots, bool kLean>
__device__ __forceinline__ void epilogue_chunk(const GemmParams& p, const OpParams& P, const CUtensorMap* out_map,
                                               uint32_t (&r)[32], uint32_t stg, uint32_t scales, int lane, int i0,
                                               int j0, int c, float col_scale, float gamma, uint32_t& seq) {
  if (i0 >= P.rows_a || j0 >= P.rows_b) return;
  if constexpr (op == Op::Dw && !kLean) {
    if (P.sign_words) {
      epilogue_chunk_signs(P, r, lane, i0, j0);
      return;
    }
  }
  if (!kLean && (!P.tma_store || P.out_f32)) {
    // the out-of-line paths take a copy, so that r itself stays in registers
    uint32_t t[32];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) t[jj] = r[jj];
    if (!P.tma_store)
      epilogue_chunk_direct<op>(p, P, t, lane, i0, j0, col_scale, gamma);
    else
      epilogue_chunk_f32<op>(out_map, t, stg, lane, i0, j0);
    return;
  }
  const uint32_t slot = stg + (seq % kSlots) * 2048u;
  if (lane == 0) bulk_wait_group_read<kSlots - 1>();  // the box last stored from this slot has been read
  __syncwarp();
  // This lane's column for the chunk's 32 rows: rows 2 pr and 2 pr + 1 are
  // converted together (packed fp32x2 arithmetic, each half rounded like the
  // scalar instruction, then one bf16x2 conversion) and written to their two
  // rows of the staging box by two 16-bit stores.
  const uint32_t col = slot + static_cast<uint32_t>(lane) * 2;
  if constexpr (op == Op::Fwd) {
    // exact int32 -> fp32 through the 1.5 * 2^23 shifter (|acc| <= 127 K < 2^22)
    // when K allows (always in the lean instance), else the conversion
    // instruction; then one rounding by the row's scale, read from the warp's
    // table (broadcast loads)
    const bool shifter = kLean || P.red <= kShifterMaxK;
    constexpr uint64_t kMagic2 = 0x4B4000004B400000ull;  // {1.5 * 2^23, 1.5 * 2^23}
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 sc = ld_shared_f4(scales + (c * 32 + 4 * u) * 4);
      const float sv[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 4 * u + 2 * h;
        uint64_t f2;
        if (shifter) {
          f2 = f32x2_sub(pair_u64(r[j] + 0x4B400000u, r[j + 1] + 0x4B400000u), kMagic2);
        } else {
          f2 = pair_u64(__float_as_uint(static_cast<float>(static_cast<int32_t>(r[j]))),
                        __float_as_uint(static_cast<float>(static_cast<int32_t>(r[j + 1]))));
        }
        const uint32_t b2 =
            f32x2_to_bf16x2(f32x2_mul(f2, pair_u64(__float_as_uint(sv[2 * h]), __float_as_uint(sv[2 * h + 1]))));
        st_shared_b16(col + j * 64, b2);
        st_shared_b16(col + (j + 1) * 64, b2 >> 16);
      }
    }
  } else {
#pragma unroll
    for (int pr = 0; pr < 16; ++pr) {
      const int j = 2 * pr;
      uint32_t b2;
      if constexpr (op == Op::Dx)
        b2 = f32x2_to_bf16x2(f32x2_mul(pair_u64(r[j], r[j + 1]),
                                       pair_u64(__float_as_uint(gamma), __float_as_uint(gamma))));
      else
        b2 = f32x2_to_bf16x2(pair_u64(r[j], r[j + 1]));
      st_shared_b16(col + j * 64, b2);
      st_shared_b16(col + (j + 1) * 64, b2 >> 16);
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(out_map, slot, i0, j0);
    bulk_commit_group();
  }
  ++seq;
}

// Epilogue, one tile: drain the TMEM accumulator two 32-column chunks per
// (rolled) iteration; each chunk's TMEM load overlaps the previous chunk's
// conversion and store. The warp takes the chunk pairs pb, pb + ps, ... of
// its lane quadrant (all of them for a tile whose buffer is handed back
// afterwards; for a pair's last tile all 16 warps share the pairs). With
// `release`, the buffer is handed back once the last load has landed.
template <Op op, int BN, int kSlots, bool kLean>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, const OpParams& P, const CUtensorMap* out_map,
                                              uint32_t tmem_base, int buf, uint32_t stg, int lane, int q, int a0,
                                              int bp, float gamma, int pb, int ps, bool release,
                                              uint32_t tmem_empty_lead, uint32_t& seq) {
  static_assert(BN % 64 == 0, "chunks are drained in pairs");
  constexpr int kPairs = BN / 64;
  if (pb >= kPairs) return;
  const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * 256;
  const int i0 = a0 + q * 32;
  // forward: the warp's table of the tile's column scales s_x[m] * gamma
  const uint32_t scales = stg + kSlots * 2048u;
  if constexpr (op == Op::Fwd) {
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
      const int j = bp + c * 32 + lane;
      st_shared_b32(scales + (c * 32 + lane) * 4, __float_as_uint(j < P.rows_b ? __fmul_rn(__ldg(p.sx + j), gamma)
                                                                               : 0.0f));
    }
    __syncwarp();
  }
  uint32_t ra[32], rb[32];
  tmem_ld_32x32b_x32(tbase + 64 * pb, ra);
  tmem_ld_wait();
#pragma unroll 1
  for (int pr = pb; pr < kPairs; pr += ps) {
    const int c = 2 * pr;
    const bool more = pr + ps < kPairs;
    // forward: s_x[m] * gamma of the two chunks' columns (lane l: column 32c + l)
    float s0 = 0.0f, s1 = 0.0f;
    if constexpr (op == Op::Fwd) {
      const int j = bp + c * 32 + lane;
      s0 = j < P.rows_b ? __fmul_rn(__ldg(p.sx + j), gamma) : 0.0f;
      s1 = j + 32 < P.rows_b ? __fmul_rn(__ldg(p.sx + j + 32), gamma) : 0.0f;
    }
    tmem_ld_32x32b_x32(tbase + 32 * (c + 1), rb);
    epilogue_chunk<op, kSlots, kLean>(p, P, out_map, ra, stg, scales, lane, i0, bp + c * 32, c, s0, gamma, seq);
    tmem_ld_wait();
    if (more) {
      tmem_ld_32x32b_x32(tbase + 64 * (pr + ps), ra);
    } else if (release) {
      // every TMEM load of this buffer has landed: hand it back
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty_lead);
    }
    epilogue_chunk<op, kSlots, kLean>(p, P, out_map, rb, stg, scales, lane, i0, bp + (c + 1) * 32, c + 1, s1, gamma, seq);
    if (more) tmem_ld_wait();
  }
}

// ---------------------------------------------------------------- the kernel

template <Family F, int BN, bool kLean>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap map_b0, const __grid_constant__ CUtensorMap map_src0,
                     const __grid_constant__ CUtensorMap map_out0, const __grid_constant__ CUtensorMap map_b1,
                     const __grid_constant__ CUtensorMap map_src1, const __grid_constant__ CUtensorMap map_out1,
                     const __grid_constant__ CUtensorMap map_sx, const __grid_constant__ GemmParams p) {
  using G = Geo<F, BN>;
  using L = Layout<F, BN>;
  constexpr int S = L::kS;
  constexpr Op kOp0 = (F == Family::Fwd) ? Op::Fwd : Op::Dx;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* src_full = bars;
  uint64_t* full = bars + S;
  uint64_t* empty = bars + 2 * S;
  uint64_t* tmem_full = bars + 3 * S;
  uint64_t* tmem_empty = bars + 3 * S + 2;
  uint64_t* done_bar = bars + 3 * S + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  int* issued_parity = reinterpret_cast<int*>(smem + L::kOffMisc + 8);  // [S]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&src_full[s], 1);
      mbar_init(&full[s], 1 + 2 * (kNumRebuildWarps / kRebuildGroups));  // expect_tx + both CTAs' rebuilding warps
      mbar_init(&empty[s], 1);
      issued_parity[s] = -1;
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], 2 * kNumEpiWarps);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // inputs come from earlier kernels in the stream: the set-up above overlaps
  // their tail, the first read waits for them
  pdl_wait_primary();
  pdl_launch_dependents();

  // A failed wait also stops the peer CTA's waits.
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_wait(bar, parity, abort_flag, p.err)) return true;
    st_cluster_u32(map_to_rank(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u), 1u);
    return false;
  };
  auto lead = [&](uint64_t* bar) -> uint32_t { return map_to_rank(smem_u32(bar), 0); };
  const Maps maps0{&map_b0, &map_src0, &map_sx};
  const Maps maps1{&map_b1, &map_src1, &map_sx};

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      if (p.op[0].ntiles) {
        prefetch_tensormap(&map_b0);
        if (p.op[0].src_tma) prefetch_tensormap(&map_src0);
      }
      if (F == Family::Bwd && p.op[1].ntiles) {
        prefetch_tensormap(&map_b1);
        prefetch_tensormap(&map_src1);
        if (!p.op[1].xhat_tma) prefetch_tensormap(&map_sx);
      }
    }
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int tile;
    for (int i = 0; ok && next_tile(p, pair, npairs, i, tile); ++i) {
      const TileInfo t = decode_tile<BN>(p, tile, rank);
      const OpParams& P = p.op[t.opi];
      const int bh = t.bp + static_cast<int>(rank) * (BN / 2);  // this CTA's B rows
      for (int kb = 0; kb < P.num_kb; ++kb) {
        if (!wait(&empty[stage], phase ^ 1)) {
          ok = false;
          break;
        }
        if (lane == 0) issued_parity[stage] = static_cast<int>(phase);
        uint8_t* sA = smem + L::kOffA + stage * G::kABytes;
        uint8_t* sB = smem + L::kOffB + stage * G::kBBytes;
        uint8_t* sSrc = smem + L::kOffSrc + stage * G::kSrcBytes;
        uint8_t* sSx = smem + L::kOffSx + stage * G::kSxBytes;
        if (t.opi == 0)
          load_stage<kOp0, F, BN, kLean>(p, P, maps0, leader, lane, t.a0, t.bp, bh, kb, &full[stage], lead(&full[stage]),
                                  &src_full[stage], sA, sB, sSrc, sSx);
        else if constexpr (F == Family::Bwd)
          load_stage<Op::Dw, F, BN, kLean>(p, P, maps1, leader, lane, t.a0, t.bp, bh, kb, &full[stage], lead(&full[stage]),
                                    &src_full[stage], sA, sB, sSrc, sSx);
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    __syncwarp();
    if (!ok && lane == 0) {
      // let every copy already issued land before the CTA exits (one time
      // bound for all of them; `full` also counts rebuild arrivals that may
      // never come on this path)
      const unsigned long long deadline = globaltimer_ns() + kWaitLimitNs;
      for (int s = 0; s < S; ++s) {
        if (issued_parity[s] < 0) continue;
        mbar_drain_until(&src_full[s], static_cast<uint32_t>(issued_parity[s]), deadline);
        if (leader) mbar_drain_until(&full[s], static_cast<uint32_t>(issued_parity[s]), deadline);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issue (leader CTA, one lane)
    if (leader && lane == 0) {
      const uint32_t sa0 = smem_u32(smem + L::kOffA), sb0 = smem_u32(smem + L::kOffB);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t buf_phase = 0;
      bool ok = true;
      int tile;
      for (int i = 0; ok && next_tile(p, pair, npairs, i, tile); ++i) {
        const int opi = tile >= p.op[0].ntiles ? 1 : 0;
        const int num_kb = p.op[opi].num_kb;
        if (!wait(&tmem_empty[buf], buf_phase ^ 1)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * 256);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sa0 + stage * G::kABytes, sb = sb0 + stage * G::kBBytes;
          if (opi == 0)
            mma_stage<kOp0, BN>(d_tmem, sa, sb, kb);
          else if constexpr (F == Family::Bwd)
            mma_stage<Op::Dw, BN>(d_tmem, sa, sb, kb);
          mma_commit_pair(&empty[stage], 0x3);
          if (kb == num_kb - 1) mma_commit_pair(&tmem_full[buf], 0x3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (++buf == kAccBufs<BN>) {
          buf = 0;
          buf_phase ^= 1;
        }
      }
      // done_bar completes in both CTAs once every MMA issued so far has finished
      mma_commit_pair(done_bar, 0x3);
    }
    if (lane == 0) mbar_drain(done_bar, 0);
    __syncwarp();
  } else if (rebuild_slot(warp) >= 0) {
    // ------------------------------------------------------------ rebuild A (both CTAs)
    static_assert(kRebuildThreads == 128, "rebuild mappings assume 128 threads per stage");
    const int slot = rebuild_slot(warp);
    const int group = slot >> 2;                    // 0 or 1: even or odd stage sequence numbers
    const int rt = (slot & 3) * 32 + lane;          // 0..127 within the group
    int stage = 0;
    uint32_t phase = 0;
    int seq = 0;                                    // stage sequence number across tiles
    bool ok = true;
    int tile;
    for (int i = 0; ok && next_tile(p, pair, npairs, i, tile); ++i) {
      const int opi = tile >= p.op[0].ntiles ? 1 : 0;
      const int num_kb = p.op[opi].num_kb;
      for (int kb = 0; kb < num_kb; ++kb, ++seq) {
        if ((seq & 1) == group) {
          if (!wait(&src_full[stage], phase)) {
            ok = false;
            break;
          }
          const uint32_t sA = smem_u32(smem + L::kOffA + stage * G::kABytes);
          const uint32_t sSrc = smem_u32(smem + L::kOffSrc + stage * G::kSrcBytes);
          const float* sSx = reinterpret_cast<const float*>(smem + L::kOffSx + stage * G::kSxBytes);
          if (opi == 0)
            rebuild_stage<kOp0, F, BN>(rt, sA, sSrc, sSx);
          else if constexpr (F == Family::Bwd) {
            if (!kLean && !p.op[1].xhat_tma) rebuild_stage<Op::Dw, F, BN>(rt, sA, sSrc, sSx);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead(&full[stage]));
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  }

  {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Warps 12..15 drain every tile's accumulator, waiting on tmem_full tile
    // by tile (they hand each buffer back, so they are never two phases
    // behind it). A pair's last tile is shared by all 16 warps: warps 0..11
    // join after their own loops, once done_bar (committed after the pair's
    // last MMA, used once, so its phase cannot be mistaken) shows that every
    // MMA has completed; no operand stage is then read or loaded any more, so
    // they stage their output boxes in the operand stage area. Warp w takes
    // chunk pairs w / 4, + 4, ... of lane quadrant w % 4.
    const bool epi_warp = warp >= kWarpEpi0;
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const uint32_t stg = epi_warp ? smem_u32(smem + L::kOffEpi + (warp - kWarpEpi0) * L::kEpiStageBytes)
                                  : smem_u32(smem + L::kOffA + warp * L::kEpiStageBytes);
    // dX's operand holds 2 * code (codes8_to_bf16x2): its epilogue takes gamma / 2
    const float gamma = p.gamma ? (F == Family::Bwd ? 0.5f : 1.0f) * __ldg(p.gamma) : 1.0f;
    int n = 0, tile = 0;
    while (next_tile(p, pair, npairs, n, tile)) ++n;
    bool ready = epi_warp || (n > 0 && wait(done_bar, 0));
    if (ready && !epi_warp) tc_fence_after();
    int buf = 0;
    uint32_t buf_phase = 0;
    uint32_t seq = 0;
    for (int i = 0; ready && i < n; ++i) {
      next_tile(p, pair, npairs, i, tile);
      const bool last = i == n - 1;
      if (epi_warp || last) {
        const TileInfo t = decode_tile<BN>(p, tile, rank);
        const OpParams& P = p.op[t.opi];
        if (epi_warp) {
          if (!wait(&tmem_full[buf], buf_phase)) break;
          tc_fence_after();
        }
        const int pb = last ? warp >> 2 : 0, ps = last ? 4 : 1;
        if (t.opi == 0)
          epilogue_tile<kOp0, BN, G::kEpiSlots, kLean>(p, P, &map_out0, tmem_base, buf, stg, lane, q, t.a0, t.bp, gamma,
                                                pb, ps, !last, lead(&tmem_empty[buf]), seq);
        else if constexpr (F == Family::Bwd)
          epilogue_tile<Op::Dw, BN, G::kEpiSlots, kLean>(p, P, &map_out1, tmem_base, buf, stg, lane, q, t.a0, t.bp, gamma,
                                                  pb, ps, !last, lead(&tmem_empty[buf]), seq);
      }
      if (++buf == kAccBufs<BN>) {
        buf = 0;
        buf_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_group_all();  // output writes complete before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- forward for few tokens
// With up to 16 tokens the forward is bound by reading the packed codes once
// (N K / 4 bytes), not by arithmetic, and the tensor-core tiles would leave
// most SMs idle. K % 64 == 0 takes the warp-MMA kernel further down; the
// kernel here covers K % 64 != 0, where rows of packed codes are 8-byte but
// not 16-byte aligned. Warp w takes rows_per_warp consecutive output features
// n (rows of the packed codes); for each row its lanes read consecutive
// 8-byte chunks (32 codes), so every load instruction of the warp covers
// contiguous bytes, and each lane forms the INT32 partial dot products of its
// chunks with all kM tokens (codes expanded to int8 as in the GEMM rebuild,
// __dp4a). The tokens' INT8 rows sit in shared memory with a 16-byte pad
// after every chunk's 32 bytes, so the lanes' 16-byte loads fall in distinct
// banks; kRows rows are taken at a time so that each token chunk read from
// shared memory serves several rows. A row's kM sums are reduced over the
// warp by recursive halving (each step exchanges half of the remaining sums,
// so every lane ends with the total of one token) -- integer adds, exact in
// any order -- and y = bf16_rn(fp32(acc) * fp32(s_x[m] * gamma)) as in the
// GEMM epilogue.
constexpr int kFewWarps = 8;
constexpr int kFewMaxM = 16;
constexpr int kFewWarpsPerSm = 16;  // target resident warps per SM when N allows

__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Sums v[0..kM) over the warp: on return lane l holds the total of token
// few_token_of<kM>(l) (every lane of a group of 32 / kM lanes the same).
template <int kM>
__device__ __forceinline__ int32_t few_reduce(int32_t (&v)[kM], int lane) {
  int off = 16;
#pragma unroll
  for (int w = kM / 2; w >= 1; w /= 2, off /= 2) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const int32_t send = up ? v[i] : v[i + w];
      const int32_t keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  int32_t s = v[0];
#pragma unroll
  for (int o = off; o >= 1; o /= 2) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

template <int kM>
__device__ __forceinline__ int few_token_of(int lane) {
  int m = 0, off = 16;
#pragma unroll
  for (int w = kM / 2; w >= 1; w /= 2, off /= 2) m += (lane & off) ? w : 0;
  return m;
}

// Lanes whose bits below the last halving step are zero write the results.
template <int kM>
__device__ __forceinline__ bool few_writer(int lane) {
  constexpr int kLow = 32 / kM;  // lanes holding one token's total
  return (lane & (kLow - 1)) == 0;
}

template <int kM>
__global__ void __launch_bounds__(32 * kFewWarps) few_forward_kernel(
    const int8_t* __restrict__ xq, const float* __restrict__ sx, const uint8_t* __restrict__ packed,
    const float* __restrict__ gamma_ptr, int M, int N, int K, int rows_per_warp, __nv_bfloat16* __restrict__ y,
    int32_t* __restrict__ debug_acc) {
  constexpr int kChunk = 8;           // bytes of packed codes per lane chunk (32 codes)
  extern __shared__ __align__(16) uint8_t s_x[];  // [kM][cpr] chunks of 32 token bytes, each + 16 pad
  constexpr int kPitch = 4 * kChunk + 16;
  constexpr int kWords = kChunk / 4;  // 32-bit code words per chunk (16 codes each)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row_bytes = K / 4, cpr = row_bytes / kChunk;
  const int64_t n0 = (static_cast<int64_t>(blockIdx.x) * kFewWarps + warp) * rows_per_warp;
  const int nrows = n0 < N ? static_cast<int>(N - n0 < rows_per_warp ? N - n0 : rows_per_warp) : 0;
  pdl_wait_primary();
  pdl_launch_dependents();
  // the tokens' rows into shared memory (rows M .. kM-1 zero)
  const int pieces = K / 16;  // 16-byte pieces per token row
  for (int i = threadIdx.x; i < kM * pieces; i += blockDim.x) {
    const int m = i / pieces, q = i - m * pieces;
    const int c = q / kWords, t = q - c * kWords;
    const uint4 v = m < M ? __ldg(reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(m) * K) + q)
                          : make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(s_x + (m * cpr + c) * kPitch + 16 * t) = v;
  }
  __syncthreads();
  if (nrows == 0) return;
  const float gamma = __ldg(gamma_ptr);
  const uint32_t sbase = smem_u32(s_x);
  const int me = few_token_of<kM>(lane);
  const bool writer = few_writer<kM>(lane) && me < M;
  const float scale = writer ? __fmul_rn(__ldg(sx + me), gamma) : 0.0f;
  // kRows rows at a time, so that every token chunk read from shared memory
  // serves kRows rows; kSlots chunks per row and lane in flight
  constexpr int kRows = kM >= 16 ? 2 : 4;
  constexpr int kSlots = 8 / kRows;
  for (int g = 0; g < nrows; g += kRows) {
    int32_t acc[kRows][kM];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int m = 0; m < kM; ++m) acc[r][m] = 0;
    for (int c0 = 0; c0 < cpr; c0 += 32 * kSlots) {
      uint32_t words[kRows][kSlots][kWords];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const uint8_t* row = packed + (n0 + g + r) * row_bytes;
#pragma unroll
        for (int u = 0; u < kSlots; ++u) {
          const int c = c0 + 32 * u + lane;
          const bool ok = g + r < nrows && c < cpr;
          const uint2 w = ok ? __ldg(reinterpret_cast<const uint2*>(row) + c) : make_uint2(0u, 0u);
          words[r][u][0] = w.x;
          words[r][u][1] = w.y;
        }
      }
#pragma unroll
      for (int u = 0; u < kSlots; ++u) {
        if (c0 + 32 * u >= cpr) break;  // no lane of the warp has chunk slot u
        const int c = c0 + 32 * u + lane;
        if (c < cpr) {
#pragma unroll
          for (int t = 0; t < kWords; ++t) {
            uint4 q[kRows];
#pragma unroll
            for (int r = 0; r < kRows; ++r) q[r] = codes16_to_s8(words[r][u][t]);
            const uint32_t xa = sbase + c * kPitch + 16 * t;
#pragma unroll
            for (int m = 0; m < kM; ++m) {
              const uint4 xv = ld_shared_v4(xa + m * cpr * kPitch);
#pragma unroll
              for (int r = 0; r < kRows; ++r) {
                int32_t a = __dp4a(static_cast<int32_t>(q[r].x), static_cast<int32_t>(xv.x), acc[r][m]);
                a = __dp4a(static_cast<int32_t>(q[r].y), static_cast<int32_t>(xv.y), a);
                a = __dp4a(static_cast<int32_t>(q[r].z), static_cast<int32_t>(xv.z), a);
                acc[r][m] = __dp4a(static_cast<int32_t>(q[r].w), static_cast<int32_t>(xv.w), a);
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int32_t total = few_reduce<kM>(acc[r], lane);
      if (writer && g + r < nrows) {
        const int64_t off = static_cast<int64_t>(me) * N + n0 + g + r;
        y[off] = __float2bfloat16_rn(__fmul_rn(static_cast<float>(total), scale));
        if (debug_acc) debug_acc[off] = total;
      }
    }
  }
}

template <int kM>
cudaError_t launch_few(const int8_t* xq, const float* sx, const uint8_t* packed, const float* gamma, int M, int N,
                       int K, void* y, int32_t* debug_acc, cudaStream_t s) {
  const int cpr = K / 4 / 8;
  const size_t smem = static_cast<size_t>(kM) * cpr * (4 * 8 + 16);
  static int configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(few_forward_kernel<kM>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  // enough warps to fill every SM when N allows, each with whole rows
  constexpr int kRows = kM >= 16 ? 2 : 4;  // rows a warp takes at a time
  const int64_t target = static_cast<int64_t>(device_sm_count()) * kFewWarpsPerSm;
  int rpw = static_cast<int>(std::max<int64_t>(1, (N + target - 1) / target));
  rpw = (rpw + kRows - 1) / kRows * kRows;
  const int64_t warps = (N + rpw - 1) / rpw;
  const unsigned grid = static_cast<unsigned>((warps + kFewWarps - 1) / kFewWarps);
  cudaError_t e = launch_pdl(few_forward_kernel<kM>, dim3(grid), dim3(32 * kFewWarps), smem, s, xq, sx, packed, gamma,
                             M, N, K, rpw, static_cast<__nv_bfloat16*>(y), debug_acc);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Smallest power-of-two token count >= M whose token rows fit the SIMT
// few-token kernel's shared memory at this K, else 0.
int few_slots(int64_t M, int64_t K) {
  if (M > kFewMaxM) return 0;
  int slots = 1;
  while (slots < M) slots *= 2;
  const size_t smem = static_cast<size_t>(slots) * (K / 4 / 8) * (4 * 8 + 16);
  return smem <= static_cast<size_t>(kSmemLimit) ? slots : 0;
}

cudaError_t launch_few_slots(int slots, const int8_t* xq, const float* sx, const uint8_t* packed, const float* gamma,
                             int M, int N, int K, void* y, int32_t* debug_acc, cudaStream_t s) {
  switch (slots) {
    case 1: return launch_few<1>(xq, sx, packed, gamma, M, N, K, y, debug_acc, s);
    case 2: return launch_few<2>(xq, sx, packed, gamma, M, N, K, y, debug_acc, s);
    case 4: return launch_few<4>(xq, sx, packed, gamma, M, N, K, y, debug_acc, s);
    case 8: return launch_few<8>(xq, sx, packed, gamma, M, N, K, y, debug_acc, s);
    default: return launch_few<16>(xq, sx, packed, gamma, M, N, K, y, debug_acc, s);
  }
}

// Few tokens with K % 64 == 0: the same products on the tensor cores' warp
// MMA (m16n8k32, s8 x s8 -> s32), so that a code is expanded to int8 once
// for all the tokens instead of once per token and lane. A warp takes a tile
// of 16 output features (rows of the packed codes) and a slice of K in blocks
// of 256 codes; lane (g, t) (g = lane / 4, t = lane % 4) reads the 16 bytes
// [16 t, 16 t + 16) of a block of rows g and g + 8 and the 64 matching INT8
// values of tokens g (and g + 8). The MMA's k index 4 t + j (16 + 4 t + j)
// stands for the block's code 64 t + 16 w + j (64 t + 16 w + 4 + j) in its
// step 2 w and 64 t + 16 w + 8 + j (... + 12 + j) in step 2 w + 1: the
// mapping depends on t and j only, so A and B agree on it and the sum over k
// is the dot product (INT32 sums are exact in any order). The CTA's warps
// take consecutive K slices of one tile and their sums are added in shared
// memory. Tensor cores of this form (not tcgen05) suit a launch this small:
// no tensor memory to allocate, and the work per SM is a few hundred MMAs.
constexpr int kFewMmaMaxWarps = 8;

__device__ __forceinline__ void mma_s8_16832(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int kNT>  // tiles of 8 tokens: 1 (M <= 8) or 2 (M <= 16)
__global__ void __launch_bounds__(32 * kFewMmaMaxWarps) few_mma_forward_kernel(
    const int8_t* __restrict__ xq, const float* __restrict__ sx, const uint8_t* __restrict__ packed,
    const float* __restrict__ gamma_ptr, int M, int N, int K, __nv_bfloat16* __restrict__ y,
    int32_t* __restrict__ debug_acc) {
  __shared__ int32_t s_red[kFewMmaMaxWarps - 1][4 * kNT][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, S = blockDim.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int row_bytes = K / 4;
  const int nblocks = (K + 255) / 256;
  const int b0 = warp * nblocks / S, b1 = (warp + 1) * nblocks / S;  // this warp's blocks
  const int64_t n_base = static_cast<int64_t>(blockIdx.x) * 16;
  // L2 prefetch of the slice of the tile's rows (safe before the wait)
  if (lane < 16 && n_base + lane < N && b1 > b0) {
    const int lo = b0 * 64, hi = b1 * 64 < row_bytes ? b1 * 64 : row_bytes;
    prefetch_l2_bulk(packed + (n_base + lane) * row_bytes + lo, static_cast<uint32_t>(hi - lo));
  }
  pdl_wait_primary();
  pdl_launch_dependents();
  const bool r0ok = n_base + g < N, r1ok = n_base + g + 8 < N;
  const uint8_t* row0 = packed + (n_base + g) * row_bytes;
  const uint8_t* row1 = packed + (n_base + g + 8) * row_bytes;
  // the epilogue's scales, fetched now (warp 0 writes: tokens 8 j + 2 t + {0, 1})
  float scale[kNT][2];
  if (warp == 0) {
    const float gamma = __ldg(gamma_ptr);
#pragma unroll
    for (int j = 0; j < kNT; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = 8 * j + 2 * t + h;
        scale[j][h] = m < M ? __fmul_rn(__ldg(sx + m), gamma) : 0.0f;
      }
  }
  int32_t acc[kNT][4];
#pragma unroll
  for (int j = 0; j < kNT; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = 0;
  // block b's operands of this lane: codes of rows g and g + 8, tokens' INT8
  struct Operands {
    uint4 c0, c1, x[kNT][4];
  };
  auto load_block = [&](int b, Operands& o) {
    const int off = b * 64 + 16 * t;  // this lane's 16 bytes of the block (64 codes)
    const bool in = b < b1 && off < row_bytes;
    o.c0 = (in && r0ok) ? __ldg(reinterpret_cast<const uint4*>(row0 + off)) : make_uint4(0u, 0u, 0u, 0u);
    o.c1 = (in && r1ok) ? __ldg(reinterpret_cast<const uint4*>(row1 + off)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int j = 0; j < kNT; ++j) {
      const int m = 8 * j + g;
      const uint4* xr = reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(m) * K + 4 * off);
#pragma unroll
      for (int u = 0; u < 4; ++u) o.x[j][u] = (in && m < M) ? __ldg(xr + u) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  // one token tile: the next block's loads are in flight while this one is
  // multiplied; two tiles: loaded one block at a time (registers)
  Operands cur, nxt;
  load_block(b0, cur);
  for (int b = b0; b < b1; ++b) {
    if constexpr (kNT == 1) load_block(b + 1, nxt);
    const uint32_t w0[4] = {cur.c0.x, cur.c0.y, cur.c0.z, cur.c0.w}, w1[4] = {cur.c1.x, cur.c1.y, cur.c1.z, cur.c1.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint4 qa = codes16_to_s8(w0[w]), qb = codes16_to_s8(w1[w]);
#pragma unroll
      for (int j = 0; j < kNT; ++j) {
        mma_s8_16832(acc[j], qa.x, qb.x, qa.y, qb.y, cur.x[j][w].x, cur.x[j][w].y);
        mma_s8_16832(acc[j], qa.z, qb.z, qa.w, qb.w, cur.x[j][w].z, cur.x[j][w].w);
      }
    }
    if constexpr (kNT == 1) cur = nxt;
    else load_block(b + 1, cur);
  }
  // the warps' sums, added by warp 0
  if (warp > 0) {
#pragma unroll
    for (int j = 0; j < kNT; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) s_red[warp - 1][4 * j + i][lane] = acc[j][i];
  }
  __syncthreads();
  if (warp != 0) return;
  for (int w = 1; w < S; ++w)
#pragma unroll
    for (int j = 0; j < kNT; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[j][i] += s_red[w - 1][4 * j + i][lane];
  // acc[j][i]: feature n_base + g (+8 for i >= 2), token 8 j + 2 t + (i & 1)
#pragma unroll
  for (int j = 0; j < kNT; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = 8 * j + 2 * t + (i & 1);
      const int64_t n = n_base + g + (i >= 2 ? 8 : 0);
      if (m < M && n < N) {
        const int64_t o = static_cast<int64_t>(m) * N + n;
        y[o] = __float2bfloat16_rn(__fmul_rn(static_cast<float>(acc[j][i]), scale[j][i & 1]));
        if (debug_acc) debug_acc[o] = acc[j][i];
      }
    }
}

template <int kNT>
cudaError_t launch_few_mma(const int8_t* xq, const float* sx, const uint8_t* packed, const float* gamma, int M,
                           int N, int K, void* y, int32_t* debug_acc, cudaStream_t s) {
  // warps per tile (a power of two, at most one per block of 256 codes):
  // enough warps to fill every SM, while leaving room for the next launch's
  // CTAs (whose L2 prefetch then overlaps this launch)
  const int64_t tiles = (N + 15) / 16;
  const int nblocks = (K + 255) / 256;
  const int64_t target = static_cast<int64_t>(device_sm_count()) * kFewWarpsPerSm;
  // (one token tile: at most 4 warps measured faster, 4.0 against 4.3 us at
  // M = 1; two tiles: 8)
  constexpr int kMaxS = kNT == 1 ? 4 : kFewMmaMaxWarps;
  int S = 1;
  while (S < kMaxS && S < nblocks && tiles * S < target) S *= 2;
  cudaError_t e = launch_pdl(few_mma_forward_kernel<kNT>, dim3(static_cast<unsigned>(tiles)), dim3(32 * S), 0, s, xq,
                             sx, packed, gamma, M, N, K, static_cast<__nv_bfloat16*>(y), debug_acc);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Degenerate reduction (M == 0 in dW): the product is all zeros.
__global__ void zero_dw_kernel(void* out, int64_t n, int out_f32, int accumulate) {
  if (accumulate) return;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  if (out_f32)
    static_cast<float*>(out)[i] = 0.0f;
  else
    static_cast<uint16_t*>(out)[i] = 0;
}

// x_hat = bf16_rn(fp32(q) * s_x[m]) for all of xq [M][K] into a bf16 [M][K]
// workspace, converted exactly as the dW rebuild does (s8x16_to_bf16), so
// that dW tiles can load their A operand by TMA instead of rebuilding it in
// every tile (each x_hat element would otherwise be rebuilt once per
// 256-feature block of dW). A chunk is 8 values: an 8-byte load and one
// 16-byte store, so consecutive lanes read 256 and write 512 contiguous bytes
// per warp access (whole 32-byte sectors). Thread t takes kXhatU chunks
// spaced one grid apart, all loads issued first, in a grid of up to 16 CTAs
// per SM. Measured on B200 at 4096 x 2560 (CUDA graphs, one box): 6.5 us
// with 2 chunks per thread, 6.8 with 4, 7.4 with 8, 10.1 with 16; 9.2 us
// for 16-value chunks (16-byte loads, two 16-byte stores 32 bytes apart).
constexpr int kXhatU = 2;

__global__ void __launch_bounds__(256) xhat_kernel(const uint2* __restrict__ xq, const float* __restrict__ sx,
                                                   int64_t chunks, int chunks_per_row, uint4* __restrict__ out) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const int64_t T = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const bool narrow = chunks <= 0xFFFFFFFFll;  // the row index by 32-bit division
  for (int64_t c0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c0 < chunks; c0 += kXhatU * T) {
    uint2 v[kXhatU];
    float s[kXhatU];
#pragma unroll
    for (int u = 0; u < kXhatU; ++u) {
      const int64_t c = c0 + u * T;
      if (c < chunks) {
        v[u] = __ldg(xq + c);
        const int64_t row = narrow ? static_cast<int64_t>(static_cast<uint32_t>(c) / static_cast<uint32_t>(chunks_per_row))
                                   : c / chunks_per_row;
        s[u] = __ldg(sx + row);
      }
    }
#pragma unroll
    for (int u = 0; u < kXhatU; ++u) {
      const int64_t c = c0 + u * T;
      if (c < chunks) {
        uint4 o0, o1;  // o1 (values 8..15 of a 16-value chunk) is not needed
        s8x16_to_bf16(make_uint4(v[u].x, v[u].y, 0u, 0u), s[u], o0, o1);
        out[c] = o0;
      }
    }
  }
}

// ---------------------------------------------------------------- host side

thread_local char g_launch_detail[160] = "";

void set_launch_detail(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_launch_detail, sizeof(g_launch_detail), fmt, ap);
  va_end(ap);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw,
                 const char* what) {
  auto enc = get_encode_fn();
  if (!enc) {
    set_launch_detail("cuTensorMapEncodeTiled is unavailable (%s)", what);
    return false;
  }
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_launch_detail("tensor map for %s rejected (CUresult %d)", what, static_cast<int>(r));
    return false;
  }
  return true;
}

// Number of CTA pairs of this kernel that can be resident at once (GPCs with
// an odd number of SMs leave one SM out of pairing), capped at SMs / 2.
template <Family F, int BN>
int resident_pairs() {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  using L = Layout<F, BN>;
  int n = device_sm_count() / 2;
  if (cudaFuncSetAttribute(gemm_pair_kernel<F, BN, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynBytes) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * n);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::kDynBytes;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, gemm_pair_kernel<F, BN, false>, &cfg) == cudaSuccess && clusters > 0 &&
        clusters < n)
      n = clusters;
  }
  cudaGetLastError();
  if (n > kMaxPairs) n = kMaxPairs;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

void fill_op(OpParams& P, int rows_a, int rows_b, int red, int block_r, int bn) {
  P.rows_a = rows_a;
  P.rows_b = rows_b;
  P.red = red;
  P.tiles_a = (rows_a + 2 * BM - 1) / (2 * BM);
  P.num_kb = (red + block_r - 1) / block_r;
  P.ntiles = rows_a > 0 && rows_b > 0 ? P.tiles_a * ((rows_b + bn - 1) / bn) : 0;
}

// Longest-processing-time schedule of the launch's tiles over the pairs:
// tiles in decreasing cost (k-blocks plus a per-tile overhead), each to the
// least-loaded pair. Falls back to round robin beyond the parameter capacity.
// The last schedule is cached (thread-local) by its inputs.
void build_schedule(GemmParams& p, int npairs) {
  p.use_sched = 0;
  if (p.ntiles > kMaxSchedTiles || npairs > kMaxPairs || p.ntiles <= npairs) return;
  struct Key {
    int n0, n1, kb0, kb1, np;
  };
  thread_local Key key{-1, -1, -1, -1, -1};
  thread_local std::vector<uint16_t> start, tiles;
  const Key k{p.op[0].ntiles, p.op[1].ntiles, p.op[0].num_kb, p.op[1].num_kb, npairs};
  if (std::memcmp(&k, &key, sizeof(Key)) != 0) {
    constexpr int kTileOverhead = 4;  // k-block equivalents per tile (epilogue, pipeline ramp)
    const int cost[2] = {k.kb0 + kTileOverhead, k.kb1 + kTileOverhead};
    std::vector<int> order(p.ntiles);
    for (int t = 0; t < p.ntiles; ++t) order[t] = t;
    auto tcost = [&](int t) { return cost[t >= k.n0 ? 1 : 0]; };
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return tcost(a) > tcost(b); });
    std::vector<long long> load(npairs, 0);
    std::vector<std::vector<uint16_t>> lists(npairs);
    for (int t : order) {
      int best = 0;
      for (int q = 1; q < npairs; ++q)
        if (load[q] < load[best]) best = q;
      load[best] += tcost(t);
      lists[best].push_back(static_cast<uint16_t>(t));
    }
    start.assign(npairs + 1, 0);
    tiles.clear();
    for (int q = 0; q < npairs; ++q) {
      start[q] = static_cast<uint16_t>(tiles.size());
      tiles.insert(tiles.end(), lists[q].begin(), lists[q].end());
    }
    start[npairs] = static_cast<uint16_t>(tiles.size());
    key = k;
  }
  std::memcpy(p.sched_start, start.data(), start.size() * sizeof(uint16_t));
  std::memcpy(p.sched_tile, tiles.data(), tiles.size() * sizeof(uint16_t));
  p.use_sched = 1;
}

// Whether every op with tiles takes the common paths: operands and packed
// codes by TMA (x_hat from the workspace for dW), bf16 outputs by TMA store
// (no sign words, no accumulation, no debug output) and, for the forward,
// sums small enough for the shifter conversion. Such launches run the kernel
// instance compiled without the other paths (measured on B200: forward
// 59.1 -> 58.1 us, backward 205.2 -> 204.9 us at up_proj; the forward's
// conversion then fixed to the shifter: 58.7 -> 57.4 us; the outputs
// unchanged).
bool lean_params(const GemmParams& p, bool fwd) {
  const OpParams& a = p.op[0];
  const OpParams& b = p.op[1];
  const bool a_ok =
      a.ntiles == 0 || (a.src_tma && a.tma_store && !a.out_f32 && (!fwd || a.red <= kShifterMaxK));
  const bool b_ok = b.ntiles == 0 || (b.xhat_tma && b.tma_store && !b.out_f32 && !b.sign_words && !b.accumulate);
  return a_ok && b_ok && p.debug_acc == nullptr;
}

template <Family F, int BN>
cudaError_t launch_pair(const CUtensorMap* maps, GemmParams& p, int npairs, cudaStream_t s) {
  using L = Layout<F, BN>;
  static int configured[64] = {};  // attributes set once per process per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    for (auto k : {gemm_pair_kernel<F, BN, false>, gemm_pair_kernel<F, BN, true>}) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynBytes);
      if (e != cudaSuccess) return e;
    }
    configured[dev] = 1;
  }
  p.ntiles = p.op[0].ntiles + p.op[1].ntiles;
  if (p.ntiles == 0) return cudaSuccess;
  const int pairs = p.ntiles < npairs ? p.ntiles : npairs;
  build_schedule(p, pairs);
  static const bool log = std::getenv("BL_LOG") != nullptr;
  if (log)
    std::fprintf(stderr, "[bitlinear] gemm family=%d BN=%d stages=%d smem=%d tiles=%d+%d kb=%d/%d pairs=%d sched=%d\n",
                 static_cast<int>(F), BN, L::kS, L::kDynBytes, p.op[0].ntiles, p.op[1].ntiles, p.op[0].num_kb,
                 p.op[1].num_kb, pairs, p.use_sched);
  cudaError_t e = launch_pdl(lean_params(p, F == Family::Fwd) ? gemm_pair_kernel<F, BN, true>
                                                              : gemm_pair_kernel<F, BN, false>,
                             dim3(2 * pairs), dim3(kThreads), L::kDynBytes, s, maps[0], maps[1], maps[2], maps[3],
                             maps[4], maps[5], maps[6], p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Output tensor map for TMA stores: [rows][cols] of 2- or 4-byte elements,
// 32 x 32 boxes. TMA needs a 16-byte row pitch.
bool make_out_map(CUtensorMap* m, void* base, bool f32, int64_t rows, int64_t cols, const char* what) {
  return make_map_2d(m, base, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cols, rows,
                     cols * (f32 ? 4 : 2), 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE, what);
}

// B rows per pair tile for the forward: the candidate with the least
// estimated time, rounds x (k-blocks x stage time + tile overhead), where a
// round is one tile on every pair. The stage and tile times are per-BN
// weights measured on B200 (ns, CUDA graphs of the up- and down-projection
// forwards): up to 256 columns a stage takes ~0.42-0.45 us and the
// epilogue overlaps the next tile; the 320-column tile's two MMAs and
// single accumulator cost more per stage and expose its epilogue, so it wins
// only where it saves a round (the down-projection: 70 tiles in one round
// against 80 in two).
struct BnCost {
  int bn, stage_ns, tile_ns;
};
int choose_bn(int rows_a, int rows_b, int red, int npairs, const BnCost* cands, int ncands) {
  const long long tiles_a = (rows_a + 2 * BM - 1) / (2 * BM);
  const long long kb = (red + 127) / 128;
  int best = cands[0].bn;
  long long best_cost = -1;
  for (int i = 0; i < ncands; ++i) {
    const long long tiles = tiles_a * ((rows_b + cands[i].bn - 1) / cands[i].bn);
    const long long rounds = (tiles + npairs - 1) / npairs;
    const long long cost = rounds * (kb * cands[i].stage_ns + cands[i].tile_ns);
    if (best_cost < 0 || cost < best_cost) {
      best = cands[i].bn;
      best_cost = cost;
    }
  }
  return best;
}

}  // namespace

const char* launch_detail() { return g_launch_detail; }

void clear_launch_detail() { g_launch_detail[0] = 0; }

int device_sm_count() {
  static int cached[64];
  static bool init[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!init[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
    init[dev] = true;
  }
  return cached[dev];
}

cudaError_t launch_forward(const int8_t* xq, const float* sx, const uint8_t* w_packed, const float* gamma,
                           int64_t M, int64_t N, int64_t K, void* y, int32_t* debug_acc, int* err,
                           cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  // few tokens: the packed codes' bandwidth, not the tensor cores, bounds the
  // forward (the tokens' codes must fit in shared memory)
  if (M <= kFewMaxM && (K % 64) == 0) {
    const int m = static_cast<int>(M), nn = static_cast<int>(N), kk = static_cast<int>(K);
    return M <= 8 ? launch_few_mma<1>(xq, sx, w_packed, gamma, m, nn, kk, y, debug_acc, s)
                  : launch_few_mma<2>(xq, sx, w_packed, gamma, m, nn, kk, y, debug_acc, s);
  }
  if (const int slots = few_slots(M, K)) {
    const int m = static_cast<int>(M), nn = static_cast<int>(N), kk = static_cast<int>(K);
    return launch_few_slots(slots, xq, sx, w_packed, gamma, m, nn, kk, y, debug_acc, s);
  }
  static const BnCost kCands[4] = {{256, 450, 500}, {320, 680, 2800}, {192, 445, 500}, {128, 420, 500}};
  const int npairs = resident_pairs<Family::Fwd, 256>();
  const int bn = choose_bn(static_cast<int>(N), static_cast<int>(M), static_cast<int>(K), npairs, kCands, 4);
  CUtensorMap maps[7] = {};  // b0, src0, out0, b1, src1, out1, sx
  const int box_rows = bn > 256 ? bn / 4 : bn / 2;  // wide tiles load B in two boxes
  if (!make_map_2d(&maps[0], xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, box_rows, CU_TENSOR_MAP_SWIZZLE_128B,
                   "xq"))
    return cudaErrorInvalidValue;
  // y [M][N] bf16 by TMA stores when its rows are 16-byte multiples
  const bool tma_store = (N % 8) == 0 && debug_acc == nullptr;
  if (tma_store && !make_out_map(&maps[2], y, false, M, N, "y")) return cudaErrorInvalidValue;
  // packed codes [N][K/4] bytes: a TMA tensor needs a 16-byte row pitch (K % 64 == 0)
  const bool src_tma = (K % 64) == 0;
  if (src_tma && !make_map_2d(&maps[1], w_packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 4, N, K / 4, 32, BM,
                              CU_TENSOR_MAP_SWIZZLE_32B, "w_packed (fwd)"))
    return cudaErrorInvalidValue;
  static thread_local GemmParams p;
  std::memset(&p, 0, offsetof(GemmParams, sched_start));
  fill_op(p.op[0], static_cast<int>(N), static_cast<int>(M), static_cast<int>(K), 128, bn);
  p.op[0].out = y;
  p.op[0].ldo = N;
  p.op[0].src_tma = src_tma;
  p.op[0].tma_store = tma_store;
  p.K = K;
  p.packed = w_packed;
  p.sx = sx;
  p.gamma = gamma;
  p.debug_acc = debug_acc;
  p.err = err;
  if (bn == 320) return launch_pair<Family::Fwd, 320>(maps, p, npairs, s);
  if (bn == 256) return launch_pair<Family::Fwd, 256>(maps, p, npairs, s);
  if (bn == 192) return launch_pair<Family::Fwd, 192>(maps, p, npairs, s);
  return launch_pair<Family::Fwd, 128>(maps, p, npairs, s);
}

// x_hat is made in the workspace only where its rebuilds would cost more
// than the extra launch: every dW tile column block (256 features) rebuilds
// all of x_hat once, and the launch moves 3 bytes per element. Measured on
// B200 (CUDA graphs, rebuild against workspace, interleaved): 27 blocks
// (N 6912, K 2560) 213.8 -> 205.8 us with the first form of the launch;
// with the current one (6.5 us at 4096 x 2560) 10 blocks (N 2560, K 6912)
// 117.3 -> 115.0 us. The break-even is near 7 blocks.
bool backward_uses_xhat(int64_t N) { return N >= 8 * 256; }

// dX and/or dW in one launch (either output may be null).
cudaError_t launch_backward(const void* dY, const int8_t* xq, const float* sx, const uint8_t* w_packed,
                            const float* gamma, int64_t M, int64_t N, int64_t K, void* dX, void* dW, int dw_is_f32,
                            int accumulate, int dw_signs, void* xhat_ws, int* err, cudaStream_t s) {
  if (dW && M == 0) {
    // dW = 0: zeros, or sign words of +0 (all bits clear, 4-byte words)
    const int64_t n = dw_signs ? N * K / 32 : N * K;
    zero_dw_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(dW, n, dw_signs ? 1 : dw_is_f32,
                                                                           dw_signs ? 0 : accumulate);
    if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
  }
  if (M == 0) return cudaSuccess;
  constexpr int BN = 256;
  if (!backward_uses_xhat(N)) xhat_ws = nullptr;
  const int npairs = resident_pairs<Family::Bwd, BN>();
  CUtensorMap maps[7] = {};  // b0, src0, out0, b1, src1, out1, sx
  const bool src_tma = (K % 64) == 0;
  if (dX) {
    if (!make_out_map(&maps[2], dX, false, M, K, "dX")) return cudaErrorInvalidValue;
    if (!make_map_2d(&maps[0], dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, N * 2, 64, BN / 2,
                     CU_TENSOR_MAP_SWIZZLE_128B, "dY (dX)"))
      return cudaErrorInvalidValue;
    if (src_tma && !make_map_2d(&maps[1], w_packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 4, N, K / 4, 32, 64,
                                CU_TENSOR_MAP_SWIZZLE_32B, "w_packed (dX)"))
      return cudaErrorInvalidValue;
  }
  if (dW) {
    // s_x as a one-row 2D tensor: [1][M] floats, row pitch rounded up to 16 bytes
    const uint64_t sx_pitch = ((static_cast<uint64_t>(M) * 4 + 15) / 16) * 16;
    if (!make_map_2d(&maps[3], dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, N * 2, 64, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B, "dY (dW)"))
      return cudaErrorInvalidValue;
    if (xhat_ws) {
      // x_hat [M][K] bf16 in the workspace, loaded as dW's A in 64 x 64 boxes
      if (!make_map_2d(&maps[4], xhat_ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, K * 2, 64, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B, "x_hat (dW)"))
        return cudaErrorInvalidValue;
    } else if (!make_map_2d(&maps[4], xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B,
                            "xq (dW)") ||
               !make_map_2d(&maps[6], sx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, M, 1, sx_pitch, 64, 1,
                            CU_TENSOR_MAP_SWIZZLE_NONE, "sx (dW)")) {
      return cudaErrorInvalidValue;
    }
    if (!accumulate && !dw_signs && !make_out_map(&maps[5], dW, dw_is_f32 != 0, N, K, "dW"))
      return cudaErrorInvalidValue;
  }
  static thread_local GemmParams p;
  std::memset(&p, 0, offsetof(GemmParams, sched_start));
  if (dX) {
    fill_op(p.op[0], static_cast<int>(K), static_cast<int>(M), static_cast<int>(N), 64, BN);
    p.op[0].out = dX;
    p.op[0].ldo = K;
    p.op[0].src_tma = src_tma;
    p.op[0].tma_store = 1;
  }
  if (dW) {
    fill_op(p.op[1], static_cast<int>(K), static_cast<int>(N), static_cast<int>(M), 64, BN);
    p.op[1].out = dW;
    p.op[1].ldo = K;
    p.op[1].out_f32 = dw_signs ? 0 : dw_is_f32;
    p.op[1].accumulate = dw_signs ? 0 : accumulate;
    p.op[1].tma_store = !accumulate && !dw_signs;
    p.op[1].sign_words = dw_signs;
    p.op[1].xhat_tma = xhat_ws != nullptr;
  }
  p.K = K;
  p.packed = w_packed;
  p.sx = sx;
  p.gamma = dX ? gamma : nullptr;
  p.err = err;
  if (dW && xhat_ws) {
    const int64_t chunks = M * K / 8;
    const int64_t want = (chunks + 256 * kXhatU - 1) / (256 * kXhatU);
    const int64_t cap = static_cast<int64_t>(16) * device_sm_count();
    cudaError_t e = launch_pdl(xhat_kernel, dim3(static_cast<unsigned>(want < cap ? want : cap)), dim3(256), 0, s,
                               reinterpret_cast<const uint2*>(xq), sx, chunks, static_cast<int>(K / 8),
                               static_cast<uint4*>(xhat_ws));
    if (e != cudaSuccess) return e;
  }
  return launch_pair<Family::Bwd, BN>(maps, p, npairs, s);
}

}  // namespace bl
