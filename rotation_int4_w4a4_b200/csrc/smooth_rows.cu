// Runtime smoothing + block Hadamard + per-group INT4 quantisation, one thread per row (sm_100a).
//
// Computes, per row and 128-channel group, y = ((x * a) H_128) * b with per-channel vectors a, b,
// then scale = max|y| / (7 sqrt(128)) and codes = RNE(y * 7 / max|y|), nibble-packed (the same
// outputs as the other transform kernels; H is applied unnormalised and 1/sqrt(128) is folded
// into the stored scale, which absmax quantisation allows).
//
//   mode COLMAX (activations, smoothing first): a = 1/s, s[j] = max over the tile's 128 rows of
//               |x[., j]| (0 -> 1), written to smooth_out when given (RRS page, main equation:
//               s_j = max |X_j| and X diag(s)^-1, taken per 128-token block; Hadamard page §6.1).
//   mode PRE    (weights, smoothing first): a = a caller vector (smooth_w), b = 1.
//   mode POST   (weights, the RRS page's rotate-then-smooth order): a = 1, b = a caller vector.
//   mode NONE   a = b = 1.
//
// A tile is 128 rows x one group (128 channels, 32 KB of bf16), brought into shared memory by
// TMA with the 128-byte swizzle.  Each of the 128 threads then owns one row of the tile: it
// reads its 256 bytes from shared memory, so the whole 128-point transform (7 radix-2 stages),
// the group absmax and the packing run in its registers with no cross-lane traffic.  Column
// maxima are read from the same shared-memory tile by column (16 rows x 8 channels per thread)
// and combined through a small shared array.  Persistent CTAs walk the tiles with a two-stage
// TMA ring, so the next tile streams in while the current one is transformed.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "rows.cuh"

namespace pq {
namespace {

constexpr int SR_ROWS = 128;                          // rows per tile = threads per CTA
constexpr int SR_STAGES = 2;
constexpr uint32_t kSrTileBytes = SR_ROWS * 128 * 2;  // one tile: 32 KB of bf16
constexpr uint64_t kSrWaitNs = 2000000000ull;         // 2 s
constexpr float kSrScaleHadamard = 0.012626906806902634f;   // 1/(7*sqrt(128)), float-rounded

enum : int { SR_COLMAX = PQ_SR_COLMAX, SR_PRE = PQ_SR_PRE, SR_POST = PQ_SR_POST, SR_NONE = PQ_SR_NONE };

struct __align__(1024) SrSmem {
  uint8_t x[SR_STAGES][2][SR_ROWS * 128];   // [stage][K-block of 64 channels][row][128 B, swizzled]
  uint32_t red[8][64];                      // column-max partials: [row slot][channel pair], |bf16| bits
  float mul[128];                           // this tile's per-channel multiplier (1/s, a or b)
  uint64_t full[SR_STAGES];
  int abort_flag;
};
constexpr size_t kSrSmemBytes = sizeof(SrSmem) + 1024;

// Byte offset of the 16-byte chunk j (channels 8j..8j+7 of a K-block) of row r in a tile
// loaded with the 128-byte swizzle: chunk index XOR (row mod 8).
__device__ __forceinline__ uint32_t sr_chunk(int r, int j) { return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)); }

// The mode is a template parameter so that each mode's code is allocated registers on its own.
template <int mode>
__global__ void __launch_bounds__(SR_ROWS, 3) smooth_rows_kernel(
    const __grid_constant__ CUtensorMap tmX, int64_t rows, int G, int64_t num_tiles,
    const float* __restrict__ vec, uint8_t* __restrict__ codes, float* __restrict__ scales,
    float* __restrict__ smooth_out, unsigned int* status) {
  extern __shared__ unsigned char smem_raw[];
  SrSmem& S = *reinterpret_cast<SrSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                         ~static_cast<uintptr_t>(1023));
  const int t = threadIdx.x, lane = t & 31;
  const int64_t first = blockIdx.x, stride = gridDim.x;
  const int64_t D = (int64_t)G * 128;
  ptx::griddep_launch_dependents();   // a programmatic dependent may start (it waits before reading)

  if (t == 0) {
    for (int s = 0; s < SR_STAGES; ++s) ptx::mbar_init(&S.full[s], 1);
    S.abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  // Tiles are numbered row-block major, group fastest: consecutive CTAs read adjacent 256-byte
  // runs of the same rows.
  auto issue = [&](int64_t tile, int s) {
    const int rb = (int)(tile / G), gi = (int)(tile - (int64_t)rb * G);
    ptx::mbar_arrive_expect_tx(&S.full[s], kSrTileBytes);
    ptx::tma_load_2d(S.x[s][0], &tmX, &S.full[s], gi * 128, rb * SR_ROWS);
    ptx::tma_load_2d(S.x[s][1], &tmX, &S.full[s], gi * 128 + 64, rb * SR_ROWS);
  };
  if (t == 0) {
    ptx::prefetch_tmap(&tmX);
    for (int s = 0; s < SR_STAGES; ++s)
      if (first + s * stride < num_tiles) issue(first + s * stride, s);
  }

  int k = 0;
  for (int64_t tile = first; tile < num_tiles; tile += stride, ++k) {
    const int s = k & 1;
    const uint32_t ph = (uint32_t)(k >> 1) & 1u;
    const int rb = (int)(tile / G), gi = (int)(tile - (int64_t)rb * G);
    // Tile landed?  One lane per warp polls (bounded); the block agrees on the outcome, so every
    // thread leaves the loop at the same iteration.
    int ok = 1;
    if (lane == 0 && !ptx::mbar_wait_bounded(&S.full[s], ph, &S.abort_flag, kSrWaitNs)) {
      S.abort_flag = 1;
      atomicOr(status, PQ_DEV_TIMEOUT);
      ok = 0;
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!__syncthreads_and(ok)) break;

    if constexpr (mode == SR_COLMAX) {
      // Thread (slot r0, chunk c) takes the maximum of |x| over rows 16 r0 .. 16 r0 + 15 for the
      // 8 channels of chunk c; |bf16| is compared as an unsigned 16-bit integer (exact).
      const int r0 = t >> 4, c = t & 15, kb = c >> 3, j = c & 7;
      const uint8_t* base = S.x[s][kb];
      uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = r0 * 16 + i;
        const uint4 v = *reinterpret_cast<const uint4*>(base + sr_chunk(r, j));
        m0 = __vmaxu2(m0, v.x & 0x7FFF7FFFu);
        m1 = __vmaxu2(m1, v.y & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
        m3 = __vmaxu2(m3, v.w & 0x7FFF7FFFu);
      }
      *reinterpret_cast<uint4*>(&S.red[r0][c * 4]) = make_uint4(m0, m1, m2, m3);
      __syncthreads();
      if (t < 64) {
        // Word t holds channels 2t and 2t + 1 (chunk c = t / 4 covers channels 8c .. 8c + 7).
        uint32_t mm = S.red[0][t];
#pragma unroll
        for (int r = 1; r < 8; ++r) mm = __vmaxu2(mm, S.red[r][t]);
        const float a = __uint_as_float(mm << 16), b = __uint_as_float(mm & 0xFFFF0000u);
        const float sa = a > 0.0f ? a : 1.0f, sb = b > 0.0f ? b : 1.0f;
        S.mul[2 * t] = __frcp_rn(sa);
        S.mul[2 * t + 1] = __frcp_rn(sb);
        if (smooth_out)
          *reinterpret_cast<float2*>(smooth_out + (int64_t)rb * D + gi * 128 + 2 * t) = make_float2(sa, sb);
      }
    } else if constexpr (mode != SR_NONE) {
      S.mul[t] = __ldg(vec + (int64_t)gi * 128 + t);
    }

    // This thread's row of the tile, 16 chunks of 8 channels.
    float v[128];
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
      for (int j = 0; j < 8; ++j)
        row_bf16x8(*reinterpret_cast<const uint4*>(S.x[s][kb] + sr_chunk(t, j)), v + 64 * kb + 8 * j);
    // The next load into stage s is an async-proxy write: order this thread's generic-proxy reads
    // of the stage before it (without the fence the copy can overwrite bytes not yet read).
    ptx::fence_proxy_async_smem();
    __syncthreads();   // every row (and column) of stage s is read; S.mul is complete
    if (t == 0 && tile + 2 * stride < num_tiles) issue(tile + 2 * stride, s);

    if constexpr (mode == SR_COLMAX || mode == SR_PRE) {
#pragma unroll
      for (int i = 0; i < 128; i += 4) {
        const float4 f = *reinterpret_cast<const float4*>(&S.mul[i]);
        ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(v[i], v[i + 1]), ptx::f2_pack(f.x, f.y)), v[i], v[i + 1]);
        ptx::f2_unpack(ptx::f2_mul(ptx::f2_pack(v[i + 2], v[i + 3]), ptx::f2_pack(f.z, f.w)), v[i + 2], v[i + 3]);
      }
    }
    row_fwht128(v);
    if constexpr (mode == SR_POST) {
#pragma unroll
      for (int i = 0; i < 128; i += 4) {
        const float4 f = *reinterpret_cast<const float4*>(&S.mul[i]);
        v[i] *= f.x;
        v[i + 1] *= f.y;
        v[i + 2] *= f.z;
        v[i + 3] *= f.w;
      }
    }
    const float m = row_absmax<128>(v);
    const float inv = m > 0.0f ? 7.0f * __frcp_rn(m) : 0.0f;
    const int64_t row = (int64_t)rb * SR_ROWS + t;
    if (row < rows) {
      uint4* dst = reinterpret_cast<uint4*>(codes + row * (D / 2) + gi * 64);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_uint4(row_pack8(v + 32 * q, inv), row_pack8(v + 32 * q + 8, inv),
                            row_pack8(v + 32 * q + 16, inv), row_pack8(v + 32 * q + 24, inv));
      scales[row * G + gi] = m * kSrScaleHadamard;
    }
  }
  // Drain: a CTA that stopped early (a timeout at iteration k) waits, bounded, for the loads it
  // had issued and not consumed (tiles k and k + 1), so none lands after the CTA has exited.
  if (t == 0 && S.abort_flag) {
    int never = 0;
    for (int j = k; j < k + SR_STAGES; ++j)
      if (first + (int64_t)j * stride < num_tiles)
        (void)ptx::mbar_wait_bounded(&S.full[j & 1], (uint32_t)(j >> 1) & 1u, &never, kSrWaitNs);
  }
}

}  // namespace

namespace {

template <int mode>
cudaError_t launch_smooth_rows_mode(const pq_plan* plan, const CUtensorMap& tmX, int64_t rows, const float* vec,
                                    uint8_t* codes, float* scales, float* smooth_out, cudaStream_t stream) {
  static std::atomic<bool> attr_done[kMaxDevices];
  cudaError_t e = set_kernel_attributes(reinterpret_cast<const void*>(smooth_rows_kernel<mode>), (int)kSrSmemBytes,
                                        attr_done);
  if (e != cudaSuccess) return e;
  static std::atomic<int> per_sm_cache{0};
  int per_sm = per_sm_cache.load(std::memory_order_relaxed);
  if (per_sm < 1) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, smooth_rows_kernel<mode>, SR_ROWS, kSrSmemBytes) !=
            cudaSuccess || per_sm < 1)
      per_sm = 1;
    per_sm_cache.store(per_sm, std::memory_order_relaxed);
  }
  const int64_t row_blocks = (rows + SR_ROWS - 1) / SR_ROWS;
  const int64_t tiles = row_blocks * plan->G;
  const int64_t cap = (int64_t)device_sm_count() * per_sm;
  const int grid = (int)(tiles < cap ? tiles : cap);
  smooth_rows_kernel<mode><<<grid, SR_ROWS, kSrSmemBytes, stream>>>(tmX, rows, plan->G, tiles, vec, codes, scales,
                                                                    smooth_out, plan->d_status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_smooth_rows(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, int mode,
                               const float* vec, uint8_t* codes, float* scales, float* smooth_out,
                               cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  CUtensorMap tmX;
  cudaError_t e = make_bf16_tile_map(&tmX, X, rows, plan->D, ldx);
  if (e != cudaSuccess) return e;
  switch (mode) {
    case SR_COLMAX: return launch_smooth_rows_mode<SR_COLMAX>(plan, tmX, rows, vec, codes, scales, smooth_out, stream);
    case SR_PRE: return launch_smooth_rows_mode<SR_PRE>(plan, tmX, rows, vec, codes, scales, smooth_out, stream);
    case SR_POST: return launch_smooth_rows_mode<SR_POST>(plan, tmX, rows, vec, codes, scales, smooth_out, stream);
    default: return launch_smooth_rows_mode<SR_NONE>(plan, tmX, rows, vec, codes, scales, smooth_out, stream);
  }
}

}  // namespace pq
