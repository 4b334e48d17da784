// Per-group rotation + INT4 quantisation on the tensor cores (sm_100a): y = x R per row and
// 128-channel group, then scale = max|y| * scale_mult, codes = RNE(y * 7 / max|y|), nibble-packed.
//
// Givens (ParoQuant page §2.2/§2.3): K layers of disjoint Givens pairs per group, then the channel
// scale exp(-beta) (activations) or exp(+beta) (weights).  Every layer and the scale are linear
// and fixed by the plan, so per group they compose into one 128 x 128 matrix R_g (ParoQuant page
// §6.4: rotation on the tensor cores).  The plan stores R_g transposed (K-major for the MMA) as
// two bf16 terms R_hi + R_lo (R_lo carries the rounding residual of R_hi, so R_hi + R_lo is R to
// about 2^-17 relative).  x is exact in bf16 and every product is exact in the float32
// accumulator, so y carries only that residual and float32 summation error.
// Block Hadamard (Hadamard page §2.1/§6.1): R = H_128 unnormalised (+-1, exact in bf16, one
// term, the same for every group); the 1/sqrt(128) is folded into the stored scale.
//
// Group sizes (ParoQuant page §4.1: g = 64 for layers with many outliers; §6: g = 256 on
// mobile parts).  A tile always spans 128 channels for g <= 128: g = 64 puts two groups' matrices
// on the diagonal of the tile's 128 x 128 matrix and takes two maxima per row.  g = 256 (block
// Hadamard only) spans 256 channels: H_256 = [[H, H], [H, -H]] with H = H_128, so each output
// half is two accumulating K = 128 products against +H or -H (both resident), into a 256-column
// accumulator; the row's maximum is taken over both halves before it is quantised.
//
// One kernel per call, persistent, one CTA per SM.  Tiles are (128 rows, one group); each CTA
// takes a contiguous range of tiles in group-major order so the group's matrix stays resident.
//   warp 0      TMA producer: the X tile (128 rows x 128 channels bf16, two 128-byte swizzled
//               K-blocks) into a 4-stage ring; the matrix terms of a new group into their slots.
//   warp 1      TMEM allocator and MMA issuer: terms x 2 K-blocks x 4 tcgen05.mma kind::f16
//               (M128 N128 K16) per tile into a double-buffered float32 accumulator.
//   warps 2..9  two epilogue warpgroups taking alternate tiles (one accumulator buffer each); one
//               thread per row (TMEM lane): 128 values of y from tensor memory, absmax, quantise,
//               pack, store.
// Every mbarrier wait is bounded; a timeout sets the plan's status bit and the CTA drains.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "rows.cuh"

namespace pq {
namespace {

constexpr int RT_M = 128;                 // rows per tile (MMA M, TMEM lanes)
constexpr int RT_N = 128;                 // output channels (MMA N)
constexpr int RT_KB = 64;                 // bf16 per 128-byte swizzle row (one K-block)
constexpr int RT_STAGES = 4;              // X stages of two K-blocks (g <= 128)
constexpr int RT_THREADS = 320;           // warps 0-1 control, 2-5 and 6-9 two epilogue warpgroups
constexpr uint64_t kRtWaitNs = 2000000000ull;
constexpr uint32_t kKBlockBytes = RT_M * 128;          // one K-block of an X tile: 16 KB
constexpr uint32_t kRotBytes = 2 * RT_N * 128 * 2;     // two terms of one matrix: 64 KB

// Per group size: channels per tile, K-blocks per X stage, X stages, accumulator columns.
template <int GW> struct RtGeom {
  static constexpr int TW = GW > 128 ? GW : 128;
  static constexpr int KBS = TW / RT_KB;
  static constexpr int STAGES = RT_STAGES * 2 / KBS;
  static constexpr uint32_t BUF = (uint32_t)TW;               // TMEM columns per accumulator buffer
  static constexpr uint32_t TMEM_COLS = 2 * BUF;
  static constexpr uint32_t TILE_BYTES = (uint32_t)KBS * kKBlockBytes;
};
constexpr float kRoundMagicR = 12582912.0f;            // 1.5 * 2^23

struct __align__(1024) RotSmem {
  uint8_t x[RT_STAGES * 2][RT_M * 128];   // [stage * K-blocks per stage + K-block][128 rows x 128 bytes]
  uint8_t r[2][2][RT_N * 128];            // [term hi/lo][K-block][128 out channels x 128 bytes]
  uint64_t x_full[RT_STAGES];
  uint64_t x_empty[RT_STAGES];
  uint64_t r_full;
  uint64_t r_empty;
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_slot;
  int abort_flag;
};
constexpr size_t kRotSmemBytes = sizeof(RotSmem) + 1024;
static_assert(kRotSmemBytes <= 232448, "shared memory exceeds 227 KB");

// D format F32 (bits 4-5 = 1), A and B BF16 (bits 7-9, 10-12 = 1), both K-major, N/8, M/16.
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(RT_N >> 3) << 17) |
                                ((uint32_t)(RT_M >> 4) << 24);

__device__ __forceinline__ bool rt_wait(RotSmem& S, uint64_t* bar, uint32_t parity, unsigned int* status) {
  if (ptx::mbar_wait_bounded(bar, parity, &S.abort_flag, kRtWaitNs)) return true;
  S.abort_flag = 1;
  atomicOr(status, PQ_DEV_TIMEOUT);
  return false;
}

__device__ __forceinline__ bool rt_warp_wait(RotSmem& S, uint64_t* bar, uint32_t parity, unsigned int* status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = rt_wait(S, bar, parity, status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ void rt_drain(uint64_t* bar, uint32_t parity) {
  int never = 0;
  (void)ptx::mbar_wait_bounded(bar, parity, &never, kRtWaitNs);
}

// 8 values -> 8 nibbles: byte k = q[2k] | q[2k+1] << 4, q = RNE(v * inv) (|q| <= 7).
__device__ __forceinline__ uint32_t rt_pack8(const float* v, float inv) {
  uint32_t b[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) b[k] = __float_as_uint(fmaf(v[k], inv, kRoundMagicR));
  const uint32_t even = __byte_perm(__byte_perm(b[0], b[2], 0x0040), __byte_perm(b[4], b[6], 0x0040), 0x5410);
  const uint32_t odd = __byte_perm(__byte_perm(b[1], b[3], 0x0040), __byte_perm(b[5], b[7], 0x0040), 0x5410);
  return (even & 0x0F0F0F0Fu) | ((odd << 4) & 0xF0F0F0F0u);
}

// 8 values -> 8 high digits of 8-bit codes: with q = RNE(v * inv) (|q| <= 119), the high digit
// floor((q + 8) / 16) is bits 4..7 of q + 8, which the FMA with 1.5 * 2^23 + 8 leaves there (the
// low digit, q - 16 q_hi, has the nibble of q itself: rt_pack8).
__device__ __forceinline__ uint32_t rt_pack8_hi(const float* v, float inv) {
  uint32_t b[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) b[k] = __float_as_uint(fmaf(v[k], inv, kRoundMagicR + 8.0f)) >> 4;
  const uint32_t even = __byte_perm(__byte_perm(b[0], b[2], 0x0040), __byte_perm(b[4], b[6], 0x0040), 0x5410);
  const uint32_t odd = __byte_perm(__byte_perm(b[1], b[3], 0x0040), __byte_perm(b[5], b[7], 0x0040), 0x5410);
  return (even & 0x0F0F0F0Fu) | ((odd << 4) & 0xF0F0F0F0u);
}

// Tiles are numbered group-major: tile = gi * row_blocks + rb.  CTA c owns [begin, end).
// terms: 1 (R exact in bf16) or 2 (R_hi + R_lo).  r_groups: number of distinct matrices (G, or 1
// when every group uses the same one).  scale_mult: stored scale = max|y| * scale_mult.
// kColMax: instead of quantising, the per-channel maximum of |y| over all rows (RRS page, main
// equation: s_j = max |(X_rot)_j|).  The operands are swapped (D = R^T X^T: tensor-memory lanes
// are output channels, columns are rows), so each epilogue thread owns one channel and takes
// its maximum over the tile's 128 rows in registers; the result (times scale_mult) is merged
// into chan_max[channel] with an unsigned atomic maximum on the float's bits (all values are
// non-negative, for which the bit order is the numeric order).  Rows past the end read as zeros.
// GW: the group size (64, 128 or 256); G counts groups of GW channels; a tile spans
// RtGeom<GW>::TW channels (one group for 128 and 256, two for 64).
// Gx, slot8, scale_mult8, weights (g = 128): 8-bit outlier groups (ParoQuant page §4.1).  Rows
// of codes and scales hold Gx = G + 3 n8 groups; slot8[gi] >= 0 marks an 8-bit group j: its
// codes q = RNE(119 y / m) split into digits q = 16 q_hi + q_lo (both -8..7), written as four
// 4-bit groups with power-of-two scale factors so that the W4A4 GEMM forms the 8-bit product:
// activations (hi, hi, lo, lo) with (16 s, 16 s, s, s), weights (hi, lo, hi, lo) with
// (16 s, s, 16 s, s), at slots gi, G + 3j, G + 3j + 1, G + 3j + 2; s = m * scale_mult8.
template <bool kColMax, int GW>
__global__ void __launch_bounds__(RT_THREADS, 1) rotate_mma_kernel(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmR, int64_t rows, int G,
    int row_blocks, int64_t num_tiles, int terms, int r_groups, float scale_mult, uint8_t* __restrict__ codes,
    float* __restrict__ scales, unsigned int* __restrict__ chan_max, unsigned int* status, int Gx,
    const int16_t* __restrict__ slot8, float scale_mult8, int weights) {
  static_assert(!kColMax || GW == 128, "column maxima are taken on 128-channel groups");
  using Geo = RtGeom<GW>;
  constexpr int KBS = Geo::KBS, STAGES = Geo::STAGES;
  extern __shared__ unsigned char smem_raw[];
  RotSmem& S = *reinterpret_cast<RotSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A GEMM launched as this grid's programmatic dependent may start its prologue and weight
  // loads now; it waits for this grid's completion before it reads the codes.
  ptx::griddep_launch_dependents();
  const int64_t begin = num_tiles * blockIdx.x / gridDim.x;
  const int64_t end = num_tiles * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&S.x_full[s], 1);
      ptx::mbar_init(&S.x_empty[s], 1);
    }
    ptx::mbar_init(&S.r_full, 1);
    ptx::mbar_init(&S.r_empty, 1);
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.acc_full[b], 1);
      ptx::mbar_init(&S.acc_empty[b], 4);   // the 4 warps of the warpgroup that owns buffer b
    }
    ptx::mbar_init(&S.mma_done, 1);
    S.abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmR);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&S.tmem_slot, Geo::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = S.tmem_slot;

  if (warp == 0) {
    // --------------------------------------------------------------------- producer
    if (lane == 0) {
      int step = 0, loaded = 0;           // loaded: number of matrices loaded so far
      int cur_r = -1;
      bool ok = true;
      for (int64_t tile = begin; tile < end && ok; ++tile, ++step) {
        const int gi = (int)(tile / row_blocks);
        const int ri = r_groups > 1 ? gi : 0;
        const int64_t r0 = (tile - (int64_t)gi * row_blocks) * RT_M;
        if (ri != cur_r) {
          // The previous matrix is free once every MMA issued with it has completed.
          if (loaded > 0 && !rt_wait(S, &S.r_empty, (uint32_t)(loaded - 1) & 1u, status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&S.r_full, kRotBytes / 2 * terms);
          for (int term = 0; term < terms; ++term)
            for (int kb = 0; kb < 2; ++kb)
              ptx::tma_load_2d(S.r[term][kb], &tmR, &S.r_full, kb * RT_KB, (ri * terms + term) * RT_N);
          cur_r = ri;
          ++loaded;
        }
        const int s = step % STAGES;
        const uint32_t ph = (uint32_t)(step / STAGES) & 1u;
        if (!rt_wait(S, &S.x_empty[s], ph ^ 1u, status)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&S.x_full[s], Geo::TILE_BYTES);
        for (int kb = 0; kb < KBS; ++kb)
          ptx::tma_load_2d(S.x[s * KBS + kb], &tmX, &S.x_full[s], gi * Geo::TW + kb * RT_KB, (int)r0);
      }
      // Drain: every load issued lands before the CTA may exit.
      for (int j = (step > STAGES ? step - STAGES : 0); j < step; ++j)
        rt_drain(&S.x_full[j % STAGES], (uint32_t)(j / STAGES) & 1u);
      if (loaded > 0) rt_drain(&S.r_full, (uint32_t)(loaded - 1) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int step = 0, used = 0;             // used: matrices this thread has waited for
      int cur_r = -1;
      bool ok = true;
      for (int64_t tile = begin; tile < end && ok; ++tile, ++step) {
        const int gi = (int)(tile / row_blocks);
        const int ri = r_groups > 1 ? gi : 0;
        if (ri != cur_r) {
          if (used > 0) ptx::umma_commit(&S.r_empty);   // the old matrix is free after these MMAs
          if (!rt_wait(S, &S.r_full, (uint32_t)used & 1u, status)) { ok = false; break; }
          cur_r = ri;
          ++used;
        }
        const int s = step % STAGES;
        const uint32_t ph = (uint32_t)(step / STAGES) & 1u;
        const int b = step & 1;
        const uint32_t u = (uint32_t)(step >> 1);
        if (!rt_wait(S, &S.acc_empty[b], (u & 1u) ^ 1u, status)) { ok = false; break; }
        if (!rt_wait(S, &S.x_full[s], ph, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)b * Geo::BUF;
        if constexpr (GW == 256) {
          // Output half o = sum over input halves i of X_i (+-H): -H only for (i, o) = (1, 1).
#pragma unroll
          for (int o = 0; o < 2; ++o) {
            int n = 0;
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
              for (int kb = 0; kb < 2; ++kb) {
                const uint32_t a0 = ptx::smem_addr(S.x[s * KBS + 2 * i + kb]);
                const uint32_t b0 = ptx::smem_addr(S.r[o & i][kb]);
#pragma unroll
                for (int k = 0; k < 4; ++k, ++n)
                  ptx::umma_f16(d + (uint32_t)(o * RT_N), ptx::smem_desc_sw128(a0 + 32 * k),
                                ptx::smem_desc_sw128(b0 + 32 * k), kIdescBf16, n > 0 ? 1u : 0u);
              }
          }
        } else {
          int n = 0;
          for (int term = 0; term < terms; ++term)
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
              const uint32_t a0 = ptx::smem_addr(S.x[s * KBS + kb]);
              const uint32_t b0 = ptx::smem_addr(S.r[term][kb]);
#pragma unroll
              for (int k = 0; k < 4; ++k, ++n) {   // K16 per MMA = 32 bytes along the swizzled row
                const uint64_t da = ptx::smem_desc_sw128(a0 + 32 * k), db = ptx::smem_desc_sw128(b0 + 32 * k);
                if (kColMax) ptx::umma_f16(d, db, da, kIdescBf16, n > 0 ? 1u : 0u);   // D = R^T X^T
                else ptx::umma_f16(d, da, db, kIdescBf16, n > 0 ? 1u : 0u);           // D = X R
              }
            }
        }
        ptx::umma_commit(&S.x_empty[s]);
        ptx::umma_commit(&S.acc_full[b]);
      }
      ptx::umma_commit(&S.mma_done);
      rt_drain(&S.mma_done, 0);
    }
  } else {
    // -------------------------------------------------------------------- epilogue
    // Warpgroup wg takes the tiles of steps with step % 2 == wg, i.e. accumulator buffer wg.
    const int wg = (warp - 2) >> 2;
    const int quarter = warp & 3;         // TMEM lanes 32 quarter .. + 31
    const int rl = quarter * 32 + lane;   // row within the tile
    int step = wg;
    for (int64_t tile = begin + wg; tile < end; tile += 2, step += 2) {
      const int gi = (int)(tile / row_blocks);
      const int64_t t = (tile - (int64_t)gi * row_blocks) * RT_M + rl;
      const int b = step & 1;
      const uint32_t u = (uint32_t)(step >> 1);
      if (!rt_warp_wait(S, &S.acc_full[b], u & 1u, status)) break;
      ptx::tc_fence_after();
      const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)b * Geo::BUF;
      if constexpr (GW == 256) {
        // The row's 256 values: the maximum over both halves first, then a second read of the
        // accumulator to quantise (tcgen05.ld is warp-collective: every lane takes part).
        float m = 0.0f;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t r[32];
          ptx::tmem_ld32(ta + 32 * c, r);
          ptx::tmem_ld_wait();
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(r[j]);
          m = fmaxf(m, row_absmax<32>(f));
        }
        const float inv = m > 0.0f ? 7.0f * __frcp_rn(m) : 0.0f;
        uint4* dst = reinterpret_cast<uint4*>(codes + t * (int64_t)G * 128 + gi * 128);
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t r[32];
          ptx::tmem_ld32(ta + 32 * c, r);
          ptx::tmem_ld_wait();
          float y[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) y[j] = __uint_as_float(r[j]);
          if (t < rows) dst[c] = make_uint4(rt_pack8(y, inv), rt_pack8(y + 8, inv), rt_pack8(y + 16, inv),
                                            rt_pack8(y + 24, inv));
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.acc_empty[b]);
        if (t < rows) scales[t * G + gi] = m * scale_mult;
      } else {
      float y[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(ta + 32 * c, r);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) y[32 * c + j] = __uint_as_float(r[j]);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.acc_empty[b]);
      const float m = row_absmax<128>(y);
      if constexpr (kColMax) {
        // this thread's lane is output channel rl of group gi; its columns are the tile's rows
        atomicMax(chan_max + (int64_t)gi * 128 + rl, __float_as_uint(m * scale_mult));
        continue;
      }
      if constexpr (GW == 64) {
        // two groups per tile: channels 0..63 and 64..127 of the row, one maximum each
        const float mh[2] = {row_absmax<64>(y), row_absmax<64>(y + 64)};
        if (t < rows) {
          uint4* dst = reinterpret_cast<uint4*>(codes + t * (int64_t)G * 32 + gi * 64);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float inv = mh[k >> 1] > 0.0f ? 7.0f * __frcp_rn(mh[k >> 1]) : 0.0f;
            dst[k] = make_uint4(rt_pack8(y + 32 * k, inv), rt_pack8(y + 32 * k + 8, inv),
                                rt_pack8(y + 32 * k + 16, inv), rt_pack8(y + 32 * k + 24, inv));
          }
          scales[t * G + 2 * gi] = mh[0] * scale_mult;
          scales[t * G + 2 * gi + 1] = mh[1] * scale_mult;
        }
        continue;
      }
      const int j8 = slot8 != nullptr ? (int)__ldg(slot8 + gi) : -1;   // the same for the whole tile
      if (j8 >= 0) {
        if (t < rows) {
          const float inv8 = m > 0.0f ? 119.0f * __frcp_rn(m) : 0.0f;
          uint8_t* crow = codes + t * (int64_t)Gx * 64;
          uint4* hi_a = reinterpret_cast<uint4*>(crow + gi * 64);
          uint4* hi_b = reinterpret_cast<uint4*>(crow + (G + 3 * j8 + (weights ? 1 : 0)) * 64);
          uint4* lo_a = reinterpret_cast<uint4*>(crow + (G + 3 * j8 + (weights ? 0 : 1)) * 64);
          uint4* lo_b = reinterpret_cast<uint4*>(crow + (G + 3 * j8 + 2) * 64);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 hi = make_uint4(rt_pack8_hi(y + 32 * k, inv8), rt_pack8_hi(y + 32 * k + 8, inv8),
                                        rt_pack8_hi(y + 32 * k + 16, inv8), rt_pack8_hi(y + 32 * k + 24, inv8));
            const uint4 lo = make_uint4(rt_pack8(y + 32 * k, inv8), rt_pack8(y + 32 * k + 8, inv8),
                                        rt_pack8(y + 32 * k + 16, inv8), rt_pack8(y + 32 * k + 24, inv8));
            hi_a[k] = hi;
            hi_b[k] = hi;
            lo_a[k] = lo;
            lo_b[k] = lo;
          }
          const float s8 = m * scale_mult8;
          float* srow = scales + t * Gx;
          srow[gi] = 16.0f * s8;
          srow[G + 3 * j8] = weights ? s8 : 16.0f * s8;
          srow[G + 3 * j8 + 1] = weights ? 16.0f * s8 : s8;
          srow[G + 3 * j8 + 2] = s8;
        }
        continue;
      }
      const float inv = m > 0.0f ? 7.0f * __frcp_rn(m) : 0.0f;
      if (t < rows) {
        uint4* dst = reinterpret_cast<uint4*>(codes + t * (int64_t)Gx * 64 + gi * 64);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          dst[k] = make_uint4(rt_pack8(y + 32 * k, inv), rt_pack8(y + 32 * k + 8, inv),
                              rt_pack8(y + 32 * k + 16, inv), rt_pack8(y + 32 * k + 24, inv));
        scales[t * Gx + gi] = m * scale_mult;
      }
      }   // GW <= 128
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Geo::TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFnR)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFnR encode_fn_r() {
  static std::atomic<EncodeTiledFnR> cache{nullptr};
  EncodeTiledFnR fn = cache.load(std::memory_order_acquire);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFnR>(p);
      cache.store(fn, std::memory_order_release);
    }
  }
  return fn;
}

}  // namespace

// bf16 [rows][inner] (row stride ld elements) with a box of 64 x 128 and 128-byte swizzle.
cudaError_t make_bf16_tile_map(CUtensorMap* map, const void* base, int64_t rows, int64_t inner, int64_t ld) {
  EncodeTiledFnR enc = encode_fn_r();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)RT_KB, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// uint8 [rows][inner] (row stride = inner bytes) with a box of box_inner bytes x box_rows, zero
// fill outside; swizzle128: the 128-byte swizzle (box_inner must then be 128).
cudaError_t make_u8_tile_map(CUtensorMap* map, const void* base, int64_t rows, int64_t inner, int box_inner,
                             int box_rows, bool swizzle128) {
  EncodeTiledFnR enc = encode_fn_r();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)inner};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// bf16 rows [rows][D] (row stride ld elements) seen as [rows][D/64][64]: a box of box_rows whole
// rows lands as D/64 * box_rows lines of 128 bytes with the 128-byte swizzle (line L's 16-byte
// chunk c at L * 128 + ((c ^ (L mod 8)) * 16)); rows past the end read as zero.  D / 64 <= 256.
cudaError_t make_bf16_row_lines_map(CUtensorMap* map, const void* base, int64_t rows, int64_t D, int64_t ld,
                                    int box_rows) {
  EncodeTiledFnR enc = encode_fn_r();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {64, (cuuint64_t)(D / 64), (cuuint64_t)rows};
  cuuint64_t strides[2] = {128, (cuuint64_t)ld * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)(D / 64), (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

template <int GW>
cudaError_t launch_rotate_mma_g(const pq_plan* plan, const CUtensorMap& tmX, const CUtensorMap& tmR, int64_t rows,
                                int terms, int r_groups, float scale_mult, uint8_t* codes, float* scales,
                                cudaStream_t stream, float scale_mult8 = 0.0f, int weights = 0) {
  const int row_blocks = (int)((rows + RT_M - 1) / RT_M);
  const int64_t tiles = (int64_t)row_blocks * (plan->D / RtGeom<GW>::TW);
  const int sms = device_sm_count();
  const int grid = (int)(tiles < sms ? tiles : sms);
  static std::atomic<bool> attr_done[kMaxDevices];
  cudaError_t e = set_kernel_attributes(reinterpret_cast<const void*>(rotate_mma_kernel<false, GW>), (int)kRotSmemBytes,
                                        attr_done);
  if (e != cudaSuccess) return e;
  rotate_mma_kernel<false, GW><<<grid, RT_THREADS, kRotSmemBytes, stream>>>(
      tmX, tmR, rows, plan->G, row_blocks, tiles, terms, r_groups, scale_mult, codes, scales, nullptr, plan->d_status,
      plan->Gx, plan->n8 > 0 ? plan->d_slot8 : nullptr, scale_mult8, weights);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rotate_mma(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, int weights,
                              uint8_t* codes, float* scales, cudaStream_t stream, unsigned int* chan_max) {
  if (rows <= 0) return cudaSuccess;
  const bool givens = plan->kind == PQ_GIVENS;
  const int g = plan->g;
  // Operand matrices: Givens, one per 128-channel tile (two groups' matrices on the diagonal at
  // g = 64), two bf16 terms; Hadamard, one exact term (H_128, or diag(H_64, H_64)), or at
  // g = 256 the two matrices +H_128 and -H_128.
  const int terms = givens || g == 256 ? 2 : 1;
  const int r_groups = givens ? plan->D / 128 : 1;
  CUtensorMap tmX, tmR;
  cudaError_t e = make_bf16_tile_map(&tmX, X, rows, plan->D, ldx);
  if (e != cudaSuccess) return e;
  const uint16_t* R = plan->d_rot + (size_t)(weights && givens ? 1 : 0) * r_groups * terms * RT_N * 128;
  e = make_bf16_tile_map(&tmR, R, (int64_t)r_groups * terms * RT_N, 128, 128);
  if (e != cudaSuccess) return e;
  if (chan_max) {
    // column maxima of the normalised rotation: max |x R| (Hadamard: R unnormalised, so / sqrt(128))
    const int row_blocks = (int)((rows + RT_M - 1) / RT_M);
    const int64_t tiles = (int64_t)row_blocks * plan->G;
    const int sms = device_sm_count();
    const int grid = (int)(tiles < sms ? tiles : sms);
    static std::atomic<bool> attr_cm[kMaxDevices];
    e = set_kernel_attributes(reinterpret_cast<const void*>(rotate_mma_kernel<true, 128>), (int)kRotSmemBytes, attr_cm);
    if (e != cudaSuccess) return e;
    rotate_mma_kernel<true, 128><<<grid, RT_THREADS, kRotSmemBytes, stream>>>(
        tmX, tmR, rows, plan->G, row_blocks, tiles, terms, r_groups, givens ? 1.0f : 0.088388347648318440550f,
        nullptr, nullptr, chan_max, plan->d_status, plan->G, nullptr, 0.0f, 0);
    return cudaGetLastError();
  }
  // Givens: scale = m / 7.  Hadamard: R = H unnormalised, so y is sqrt(g) times the orthonormal
  // rotation and scale = m / (7 sqrt(g)).
  switch (g) {
    case 64:
      return launch_rotate_mma_g<64>(plan, tmX, tmR, rows, terms, r_groups, givens ? (1.0f / 7.0f) : (1.0f / 56.0f),
                                     codes, scales, stream);
    case 256:
      return launch_rotate_mma_g<256>(plan, tmX, tmR, rows, terms, r_groups, 1.0f / 112.0f, codes, scales, stream);
    default:
      // 8-bit groups: scale = m / 119 (Givens) or m / (119 sqrt(128)) (Hadamard).
      return launch_rotate_mma_g<128>(plan, tmX, tmR, rows, terms, r_groups,
                                      givens ? (1.0f / 7.0f) : 0.012626906806902634f, codes, scales, stream,
                                      givens ? (1.0f / 119.0f) : 0.00074275922393545f, weights);
  }
}

}  // namespace pq
