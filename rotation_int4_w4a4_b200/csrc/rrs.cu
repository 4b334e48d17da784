// Rotated runtime smoothing with channel reordering (RRS page, main equation and Fig. 4), sm_100a.
//
// Preparation (one call over the batch's activations X):
//   1. chan_max[j] = max over every row of |(X R)[:, j]|, R the block Hadamard H_128 / sqrt(128)
//      (rotate_mma.cu in its column-maximum mode: the tensor cores rotate each 128-row tile and
//      each thread reduces one channel over the tile's rows).
//   2. inv_perm[j] = the position of channel j after sorting by descending maximum (ties: lower
//      index first) = #{k : m_k > m_j} + #{k < j : m_k = m_j}, counted in 2-D blocks of
//      (channel, other channel) pairs and added up atomically (integer counts: exact, any order).
//   3. perm[inv_perm[j]] = j, and the smoothing scale of each reordered group of 128 channels,
//      its first (largest) member's maximum (0 -> 1).
// Transform of a row (activations or weights), one CTA per row at a time:
//   the row is staged in shared memory, each thread rotates one 128-channel group in registers
//   (unnormalised H_128), the rotated row goes back to shared memory, and then it is read in the
//   reordered order perm.
//   activations: v_k = y[perm[k]] / s_(k / 128), quantised per row: scale = max|v| / 7.
//   weights:     v_k = y[perm[k]], quantised per reordered group of 128; the stored scale is the
//                group's scale times its smoothing scale s_G (the factor the GEMM applies per
//                block, RRS page Fig. 4 (3)).
// Both staged layouts are XOR-swizzled by group so that thread-per-group accesses spread over
// all shared-memory banks.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "rows.cuh"

namespace pq {
namespace {

constexpr float kRrSqrt128 = 11.313708498984760390f;         // sqrt(128), float-rounded
constexpr float kRrScaleHadamard = 0.012626906806902634f;     // 1/(7*sqrt(128)), float-rounded
constexpr int RK_J = 256;    // channels per rank block
constexpr int RK_K = 2048;   // other channels per rank block

__global__ void __launch_bounds__(RK_J) rrs_rank_kernel(const unsigned int* __restrict__ chan_max, int D,
                                                       int* __restrict__ inv_perm) {
  __shared__ __align__(16) unsigned int mk[RK_K];
  const int j = blockIdx.x * RK_J + threadIdx.x;
  const int k0 = blockIdx.y * RK_K;
  const int nk = min(RK_K, D - k0);   // a multiple of 128 (D is)
  for (int i = threadIdx.x; i < nk; i += RK_J) mk[i] = chan_max[k0 + i];
  __syncthreads();
  if (j >= D) return;
  const unsigned int mj = chan_max[j];   // float bits of a non-negative value: bit order = numeric order
  const uint4* m4 = reinterpret_cast<const uint4*>(mk);
  int cnt = 0;
  if (k0 + nk <= j) {
    // every channel of the block precedes j: it ranks first when its maximum is at least m_j
    for (int i = 0; i < nk / 4; ++i) {
      const uint4 v = m4[i];
      cnt += (v.x >= mj) + (v.y >= mj) + (v.z >= mj) + (v.w >= mj);
    }
  } else if (k0 > j) {
    // every channel of the block follows j: it ranks first only with a larger maximum
    for (int i = 0; i < nk / 4; ++i) {
      const uint4 v = m4[i];
      cnt += (v.x > mj) + (v.y > mj) + (v.z > mj) + (v.w > mj);
    }
  } else {
    for (int i = 0; i < nk; ++i) {
      const unsigned int m = mk[i];
      cnt += (m > mj || (m == mj && k0 + i < j)) ? 1 : 0;
    }
  }
  if (cnt) atomicAdd(inv_perm + j, cnt);
}

__global__ void __launch_bounds__(256) rrs_scatter_kernel(const unsigned int* __restrict__ chan_max, int D,
                                                         const int* __restrict__ inv_perm, int* __restrict__ perm,
                                                         float* __restrict__ group_scale) {
  const int j = blockIdx.x * 256 + threadIdx.x;
  if (j >= D) return;
  const int r = inv_perm[j];
  perm[r] = j;
  if ((r & 127) == 0) {
    const float m = __uint_as_float(chan_max[j]);
    group_scale[r >> 7] = m > 0.0f ? m : 1.0f;
  }
}

// ------------------------------------------------------------------------ row transform
// Geometry of one CTA: each row takes 4 threads per original 128-channel group (rounded up to
// whole warps, RR_ROW_THREADS), and a CTA transforms R rows at a time (R * row threads <= 512).
__host__ __device__ constexpr int rr_row_threads(int G) { return (4 * G + 31) / 32 * 32; }
__host__ __device__ constexpr int rr_rows_per_cta(int G) {
  return 256 / rr_row_threads(G) < 1 ? 1 : (256 / rr_row_threads(G) > 8 ? 8 : 256 / rr_row_threads(G));
}
constexpr int RR_MAX_THREADS = 512;
constexpr uint64_t kRrWaitNs = 2000000000ull;   // 2 s

// Shared-memory layout (byte offsets from a 1024-byte aligned base), the same on host and device.
struct RrLayout {
  uint32_t xbuf, x0, x1, y, off, inv_s, red, bars, total;
  __host__ __device__ RrLayout(int G) {
    const uint32_t D = (uint32_t)G * 128, R = (uint32_t)rr_rows_per_cta(G);
    xbuf = (R * D * 2 + 1023u) & ~1023u;   // one TMA buffer of R rows (1024-aligned: swizzle atoms)
    x0 = 0;
    x1 = xbuf;
    y = 2 * xbuf;                           // R rows of rotated float32 values
    off = y + R * D * 4;                    // D uint16: byte offset in a y row of channel perm[k]
    inv_s = (off + D * 2 + 15u) & ~15u;     // G floats: 1 / (s_G sqrt(128))
    red = inv_s + (uint32_t)G * 4;          // 16 floats: per-warp maxima
    bars = (red + 64 + 7u) & ~7u;           // 2 mbarriers, then the abort flag
    total = bars + 24;
  }
};

// Rotated value of channel j of a row (16-byte chunks of 4 floats, chunk c stored at c ^ ((c / 8)
// mod 8): the stage-1 writers, 8 consecutive chunks per thread, then hit 8 different bank groups).
__device__ __forceinline__ uint32_t rr_y_chunk(uint32_t c) { return (c ^ ((c >> 3) & 7u)) << 4; }

template <int MODE>   // 0: activations (per-row scale), 1: weights (per reordered group, s_G folded)
__global__ void __launch_bounds__(RR_MAX_THREADS, 1) rrs_rows_kernel(
    const __grid_constant__ CUtensorMap tmX, int64_t rows, int G, int64_t num_tiles, const int* __restrict__ perm,
    const float* __restrict__ group_scale, uint8_t* __restrict__ codes, float* __restrict__ scales,
    unsigned int* status) {
  extern __shared__ unsigned char smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const RrLayout L(G);
  const int D = G * 128, R = rr_rows_per_cta(G), RT = rr_row_threads(G);
  const int t = threadIdx.x, lane = t & 31;
  const int r = t / RT, p = t - r * RT;            // row of the tile, thread within the row
  const bool s1 = p < 4 * G;                       // stage 1: quarter q of original group gi
  const int gi = p >> 2, q = p & 3;
  uint16_t* off = reinterpret_cast<uint16_t*>(sm + L.off);
  float* inv_s = reinterpret_cast<float*>(sm + L.inv_s);
  float* red = reinterpret_cast<float*>(sm + L.red);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L.bars + 16);
  const uint32_t tile_bytes = (uint32_t)R * (uint32_t)D * 2;
  const int64_t first = blockIdx.x, stride = gridDim.x;

  if (t == 0) {
    ptx::mbar_init(&full[0], 1);
    ptx::mbar_init(&full[1], 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int64_t tile, int b) {
    ptx::mbar_arrive_expect_tx(&full[b], tile_bytes);
    ptx::tma_load_3d(sm + (b ? L.x1 : L.x0), &tmX, &full[b], 0, 0, (int)(tile * R));
  };
  if (t == 0) {
    ptx::prefetch_tmap(&tmX);
    for (int b = 0; b < 2; ++b)
      if (first + b * stride < num_tiles) issue(first + b * stride, b);
  }
  // Per CTA, once: where each reordered position's value sits in a rotated row, and 1 / s.
  for (int k = t; k < D; k += blockDim.x) {
    const uint32_t j = (uint32_t)__ldg(perm + k);
    off[k] = (uint16_t)(rr_y_chunk(j >> 2) + 4u * (j & 3u));
  }
  if (MODE == 0)
    for (int g = t; g < G; g += blockDim.x) inv_s[g] = __frcp_rn(__ldg(group_scale + g) * kRrSqrt128);

  const int chunks8 = D / 8;                       // stage 2: 8 reordered positions per chunk
  int it = 0;
  for (int64_t tile = first; tile < num_tiles; tile += stride, ++it) {
    const int b = it & 1;
    const uint32_t ph = (uint32_t)(it >> 1) & 1u;
    int ok = 1;
    if (lane == 0 && !ptx::mbar_wait_bounded(&full[b], ph, abort_flag, kRrWaitNs)) {
      *abort_flag = 1;
      atomicOr(status, PQ_DEV_TIMEOUT);
      ok = 0;
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!__syncthreads_and(ok)) break;   // also: the previous row's gathers are done, y is free

    // Stage 1: 32 channels (gi * 128 + 32 q ..) of this row, 128-point transform across the quad.
    float v[32];
    {
      const uint8_t* xb = sm + (b ? L.x1 : L.x0);
      const int line = r * (D / 64) + 2 * gi + (q >> 1);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint4 w = make_uint4(0, 0, 0, 0);
        if (s1) w = *reinterpret_cast<const uint4*>(xb + line * 128 + ((((q & 1) * 4 + k) ^ (line & 7)) << 4));
        row_bf16x8(w, v + 8 * k);
      }
    }
    row_fwht32(v);
    // bits 5 and 6 of the channel index are the quad lanes: butterflies with lanes p ^ 1, p ^ 2
#pragma unroll
    for (int bit = 1; bit <= 2; bit <<= 1) {
      const bool hi = (q & bit) != 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, v[i], bit);
        v[i] = hi ? o - v[i] : v[i] + o;
      }
    }
    uint8_t* yrow = sm + L.y + (uint32_t)r * (uint32_t)D * 4;
    if (s1) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        *reinterpret_cast<float4*>(yrow + rr_y_chunk((uint32_t)p * 8 + k)) =
            make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    }
    // The next load into buffer b is an async-proxy write: order this thread's generic-proxy
    // reads of the buffer before it.
    ptx::fence_proxy_async_smem();
    __syncthreads();   // rotated rows complete; TMA buffer b is free
    if (t == 0 && tile + 2 * stride < num_tiles) issue(tile + 2 * stride, b);

    // Stage 2: thread p takes reordered chunks c = p + i * RT (i < 4), 8 positions each.
    const int64_t row = tile * R + r;
    const bool live = row < rows;
    const uint32_t ybase = ptx::smem_addr(yrow);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = p + i * RT;
      if (c < chunks8) {
        const uint4 o = *reinterpret_cast<const uint4*>(off + 8 * c);
        const uint32_t w4[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          v[8 * i + 2 * h] = ptx::lds_f32(ybase + (w4[h] & 0xFFFFu));
          v[8 * i + 2 * h + 1] = ptx::lds_f32(ybase + (w4[h] >> 16));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * i + e] = 0.0f;
      }
    }
    uint8_t* crow = codes + row * (int64_t)(D / 2);
    if (MODE == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = p + i * RT;
        const float is = c < chunks8 ? inv_s[c >> 4] : 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * i + e] *= is;
      }
      float m = row_absmax<32>(v);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int wr = RT / 32;                      // warps per row
      if (lane == 0) red[r * wr + (p >> 5)] = m;
      __syncthreads();
      m = red[r * wr];
      for (int w = 1; w < wr; ++w) m = fmaxf(m, red[r * wr + w]);
      const float inv = m > 0.0f ? 7.0f * __frcp_rn(m) : 0.0f;
      if (live) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = p + i * RT;
          if (c < chunks8) *reinterpret_cast<uint32_t*>(crow + 4 * c) = row_pack8(v + 8 * i, inv);
        }
        if (p == 0) scales[row] = __fdiv_rn(m, 7.0f);
      }
    } else {
      // Reordered group c / 16: 16 consecutive lanes (RT is a multiple of 32) share it.
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = p + i * RT;
        float m = row_absmax<8>(v + 8 * i);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float inv = m > 0.0f ? 7.0f * __frcp_rn(m) : 0.0f;
        if (live && c < chunks8) {
          *reinterpret_cast<uint32_t*>(crow + 4 * c) = row_pack8(v + 8 * i, inv);
          if ((c & 15) == 0) scales[row * G + (c >> 4)] = (m * kRrScaleHadamard) * __ldg(group_scale + (c >> 4));
        }
      }
    }
  }
  // Drain: a CTA that stopped early waits, bounded, for the loads it had issued and not consumed.
  if (t == 0 && *abort_flag) {
    int never = 0;
    for (int j = it; j < it + 2; ++j)
      if (first + (int64_t)j * stride < num_tiles)
        (void)ptx::mbar_wait_bounded(&full[j & 1], (uint32_t)(j >> 1) & 1u, &never, kRrWaitNs);
  }
}

template <int MODE>
cudaError_t launch_rows(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, const int* perm,
                        const float* group_scale, uint8_t* codes, float* scales, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int G = plan->G, R = rr_rows_per_cta(G), threads = R * rr_row_threads(G);
  const size_t smem = rrs_rows_smem_bytes(plan->D);
  CUtensorMap tm;
  cudaError_t e = make_bf16_row_lines_map(&tm, X, rows, plan->D, ldx, R);
  if (e != cudaSuccess) return e;
  static std::atomic<int> smem_set[kMaxDevices];
  e = raise_dynamic_smem(reinterpret_cast<const void*>(rrs_rows_kernel<MODE>), (int)smem, smem_set);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rrs_rows_kernel<MODE>, threads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t tiles = (rows + R - 1) / R;
  const int64_t cap = (int64_t)device_sm_count() * per_sm;
  const int grid = (int)std::min<int64_t>(tiles, cap);
  rrs_rows_kernel<MODE><<<grid, threads, smem, stream>>>(tm, rows, G, tiles, perm, group_scale, codes, scales,
                                                         plan->d_status);
  return cudaGetLastError();
}

}  // namespace

size_t rrs_rows_smem_bytes(int D) { return (size_t)RrLayout(D / 128).total + 1024; }

cudaError_t launch_rrs_prepare(const pq_plan* plan, const void* X, int64_t T, int64_t ldx, float* chan_max,
                               int* perm, int* inv_perm, float* group_scale, cudaStream_t stream) {
  const int D = plan->D;
  cudaError_t e = cudaMemsetAsync(chan_max, 0, (size_t)D * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(inv_perm, 0, (size_t)D * sizeof(int), stream);
  if (e != cudaSuccess) return e;
  e = launch_rotate_mma(plan, X, T, ldx, 0, nullptr, nullptr, stream, reinterpret_cast<unsigned int*>(chan_max));
  if (e != cudaSuccess) return e;
  const dim3 rgrid((unsigned)((D + RK_J - 1) / RK_J), (unsigned)((D + RK_K - 1) / RK_K));
  rrs_rank_kernel<<<rgrid, RK_J, 0, stream>>>(reinterpret_cast<const unsigned int*>(chan_max), D, inv_perm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  rrs_scatter_kernel<<<(D + 255) / 256, 256, 0, stream>>>(reinterpret_cast<const unsigned int*>(chan_max), D,
                                                          inv_perm, perm, group_scale);
  return cudaGetLastError();
}

cudaError_t launch_rrs_rows(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, int weights,
                            const int* perm, const float* group_scale, uint8_t* codes, float* scales,
                            cudaStream_t stream) {
  return weights ? launch_rows<1>(plan, X, rows, ldx, perm, group_scale, codes, scales, stream)
                 : launch_rows<0>(plan, X, rows, ldx, perm, group_scale, codes, scales, stream);
}

}  // namespace pq
