// Activation transform + INT4 quantisation for a few rows (T <= 16, the decode regime), sm_100a.
//
// The tensor-core kernel (rotate_mma.cu) works on 128-row tiles; for one to a few tokens its
// prologue (tensor-memory allocation, barrier set-up, the matrix load) and its pipeline fill
// dominate.  Here one warp takes one (row, 128-channel tile) and does the whole group in
// registers: lane l holds channels 4l .. 4l + 3 (one 8-byte load, coalesced across the warp).
//   Block Hadamard (Hadamard page §2.1, §4.2): the unnormalised Walsh-Hadamard transform,
//     channel bits 0..1 inside the lane, bits 2..6 (g = 128) or 2..5 (g = 64) across lanes by
//     xor shuffles; 1/sqrt(g) is folded into the stored scale as in the other kernels.
//   Givens + channel scale (ParoQuant page §2.2, §2.3): y = x R with the plan's composed matrix
//     R = R_hi + R_lo (bf16, stored [n][k] per 128-channel tile; two 64-channel groups on the
//     diagonal at g = 64): lane l forms its four outputs from the 128 inputs, which it receives
//     by shuffles, reading its four rows of R_hi and R_lo (2 KB) from L2.
//   Then per group: max |y| by a warp reduction, scale = max * scale_mult, codes = RNE(y * 7 /
//   max) (the FMA with 1.5 * 2^23), four nibbles -> two bytes per lane.
#include <cuda_bf16.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "rows.cuh"

namespace pq {
namespace {

constexpr int RS_WARPS = 4;   // warps per block (one (row, tile) each)

template <bool kGivens, int GW>
__global__ void __launch_bounds__(32 * RS_WARPS) rows_small_kernel(
    const __nv_bfloat16* __restrict__ X, int64_t rows, int64_t ldx, int tiles, const uint16_t* __restrict__ R,
    float scale_mult, uint8_t* __restrict__ codes, float* __restrict__ scales, int G) {
  ptx::griddep_launch_dependents();   // a GEMM launched as this grid's dependent may start now
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * RS_WARPS + (threadIdx.x >> 5);
  if (item >= rows * tiles) return;
  const int64_t row = item / tiles;
  const int ti = (int)(item - row * tiles);
  const uint2 raw = *reinterpret_cast<const uint2*>(X + row * ldx + (int64_t)ti * 128 + 4 * lane);
  float x[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
  float y[4];
  if constexpr (!kGivens) {
    // in-lane bits 0 and 1
    const float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
    y[0] = a0 + a2;
    y[1] = a1 + a3;
    y[2] = a0 - a2;
    y[3] = a1 - a3;
    // lane bits: 5 stages (g = 128) or 4 (g = 64, the two 16-lane halves are the two groups)
#pragma unroll
    for (int b = 1; b < (GW == 64 ? 16 : 32); b <<= 1) {
      const float sgn = (lane & b) ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, y[i], b);
        y[i] = fmaf(y[i], sgn, o);   // low lane: y + o; high lane: o - y
      }
    }
  } else {
    // y[n] = sum_k x[k] (R_hi[n][k] + R_lo[n][k]) for this lane's n = 4 lane + j; the tile's
    // two terms are [2][128 n][128 k]; zeros off the diagonal blocks at g = 64 contribute 0.
    const uint16_t* hi = R + (size_t)ti * 2 * 128 * 128 + (size_t)(4 * lane) * 128;
    const uint16_t* lo = hi + 128 * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = 0.0f;
#pragma unroll 2
    for (int kc = 0; kc < 128; kc += 8) {
      // inputs kc .. kc + 7 live in lanes kc / 4 and kc / 4 + 1
      float xk[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        xk[e] = __shfl_sync(0xffffffffu, x[e], kc >> 2);
        xk[4 + e] = __shfl_sync(0xffffffffu, x[e], (kc >> 2) + 1);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 h = __ldg(reinterpret_cast<const uint4*>(hi + j * 128 + kc));
        const uint4 l = __ldg(reinterpret_cast<const uint4*>(lo + j * 128 + kc));
        float rh[8], rl[8];
        row_bf16x8(h, rh);
        row_bf16x8(l, rl);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[j] = fmaf(xk[e], rh[e] + rl[e], y[j]);
      }
    }
  }
  float m = fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3])));
#pragma unroll
  for (int o = (GW == 64 ? 8 : 16); o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float inv = m > 0.0f ? 7.0f * __frcp_rn(m) : 0.0f;
  uint32_t b[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) b[i] = __float_as_uint(fmaf(y[i], inv, kRowRoundMagic));
  const uint16_t packed = (uint16_t)((b[0] & 0xFu) | ((b[1] & 0xFu) << 4) | ((b[2] & 0xFu) << 8) | ((b[3] & 0xFu) << 12));
  *reinterpret_cast<uint16_t*>(codes + row * (int64_t)G * (GW / 2) + (int64_t)ti * 64 + 2 * lane) = packed;
  if (GW == 64) {
    if ((lane & 15) == 0) scales[row * G + 2 * ti + (lane >> 4)] = m * scale_mult;
  } else if (lane == 0) {
    scales[row * G + ti] = m * scale_mult;
  }
}

template <bool kGivens, int GW>
cudaError_t launch_small(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, uint8_t* codes,
                         float* scales, float scale_mult, cudaStream_t stream) {
  const int tiles = plan->D / 128;
  const int64_t items = rows * tiles;
  const int grid = (int)((items + RS_WARPS - 1) / RS_WARPS);
  rows_small_kernel<kGivens, GW><<<grid, 32 * RS_WARPS, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(X), rows, ldx, tiles, plan->d_rot, scale_mult, codes, scales, plan->G);
  return cudaGetLastError();
}

}  // namespace

bool rows_small_applies(const pq_plan* plan, int64_t rows) {
  return rows <= kRowsSmallT && plan->n8 == 0 && (plan->g == 64 || plan->g == 128) &&
         (plan->kind == PQ_HADAMARD || plan->kind == PQ_GIVENS);
}

cudaError_t launch_rows_small(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, uint8_t* codes,
                              float* scales, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const bool givens = plan->kind == PQ_GIVENS;
  // Givens: scale = m / 7.  Hadamard: unnormalised H_g, so scale = m / (7 sqrt(g)).
  if (givens)
    return plan->g == 64 ? launch_small<true, 64>(plan, X, rows, ldx, codes, scales, 1.0f / 7.0f, stream)
                         : launch_small<true, 128>(plan, X, rows, ldx, codes, scales, 1.0f / 7.0f, stream);
  return plan->g == 64 ? launch_small<false, 64>(plan, X, rows, ldx, codes, scales, 1.0f / 56.0f, stream)
                       : launch_small<false, 128>(plan, X, rows, ldx, codes, scales, 0.012626906806902634f, stream);
}

}  // namespace pq
