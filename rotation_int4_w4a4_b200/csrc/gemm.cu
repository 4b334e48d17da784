// W4A4 GEMM with per-group scales on tcgen05 tensor cores (sm_100a).
//
// Y[t][n] = sum_G sa[t][G] * sw[n][G] * d_G[t][n],  d_G = sum_{k in group G} qa[t][k] qw[n][k]
// (RRS page, main equation, last line; Fig. 4 step (3): the GEMM's K-block equals the
// quantisation group and the block's scales are applied to the interim integer result).
//
// Persistent kernel, one CTA per SM, tiles of 128 rows (tokens) x 256 columns (output channels),
// the K loop running one 128-wide group per step.  Warp roles (16 warps):
//   warp 0        TMA producer: packed int4 tiles of A (128 x 64 B) and W (256 x 64 B) per
//                 group into a 4-stage ring (64-byte swizzle).
//   warp 1        TMEM allocator and MMA issuer: 4 x tcgen05.mma kind::i8 (M128 N256 K32) per
//                 group into a double-buffered int32 accumulator in tensor memory.
//   warps 4..7    unpack: int4 -> int8 into the 128-byte-swizzled K-major operand layout.  The
//                 low nibbles of a group's bytes become K positions 0..63 and the high nibbles
//                 64..127 (the same permutation on A and W, so every dot product is unchanged),
//                 each byte holding 16*code so no sign extension is needed: d = 256 * dot.
//   warps 8..15   epilogue: per group, read the int32 tile from TMEM, convert exactly, scale
//                 by sa*sw/256 and accumulate in float32 registers (ascending group order);
//                 after the last group, store Y.
// Exact int32 -> float32 conversion: the accumulator is pre-loaded with the bit pattern of
// 1.5*2^23; since |d| <= 2^21, (bits + d) is the float 1.5*2^23 + d, so one FADD recovers d.
// Every mbarrier wait is bounded; a timeout sets a status bit, the CTA drains its own copies and
// MMAs, frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace pq {

__device__ unsigned int g_gemm_status = 0;

namespace {

constexpr int BM = 128;        // tile rows (tokens), MMA M
constexpr int BN = 256;        // tile columns (output channels), MMA N
constexpr int BKB = 64;        // packed bytes of one 128-element group
constexpr int P_STAGES = 4;    // packed ring
constexpr int U_STAGES = 2;    // unpacked ring
constexpr int NUM_THREADS = 512;
constexpr int NUM_UNPACK_WARPS = 4;
constexpr int NUM_EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t kAccBias = 0x4B400000u;          // bit pattern of 1.5 * 2^23
constexpr float kAccBiasF = 12582912.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;    // 2 s
constexpr uint32_t kTxBytes = (BM + BN) * BKB;

struct __align__(1024) GemmSmem {
  uint8_t upA[U_STAGES][BM * 128];
  uint8_t upB[U_STAGES][BN * 128];
  uint8_t pkA[P_STAGES][BM * BKB];
  uint8_t pkB[P_STAGES][BN * BKB];
  float sw_buf[NUM_EPI_WARPS][128];
  uint64_t pk_full[P_STAGES];
  uint64_t pk_empty[P_STAGES];
  uint64_t up_full[U_STAGES];
  uint64_t up_empty[U_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_slot;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(GemmSmem) + 1024;   // + slack for 1024-byte alignment

__device__ __forceinline__ void raise_abort(GemmSmem& S, unsigned int* status) {
  S.abort_flag = 1;
  atomicOr(status, PQ_DEV_TIMEOUT);
}

__device__ __forceinline__ bool wait_or_abort(GemmSmem& S, uint64_t* bar, uint32_t parity,
                                              unsigned int* status) {
  if (ptx::mbar_wait_bounded(bar, parity, &S.abort_flag, kWaitLimitNs)) return true;
  raise_abort(S, status);
  return false;
}

// Wait used while draining: ignores the abort flag, bounded in time only.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int never = 0;
  (void)ptx::mbar_wait_bounded(bar, parity, &never, kWaitLimitNs);
}

__device__ __forceinline__ uint4 unpack_lo(uint4 w) {
  return make_uint4((w.x << 4) & 0xF0F0F0F0u, (w.y << 4) & 0xF0F0F0F0u, (w.z << 4) & 0xF0F0F0F0u,
                    (w.w << 4) & 0xF0F0F0F0u);
}
__device__ __forceinline__ uint4 unpack_hi(uint4 w) {
  return make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
}

__device__ __forceinline__ void cta_producer_mma_unpack(GemmSmem& S, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                                        uint32_t tmem, int G, int m_tiles, int num_tiles,
                                                        unsigned int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int step = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % m_tiles) * BM, n0 = (tile / m_tiles) * BN;
        for (int kg = 0; kg < G; ++kg, ++step) {
          const int s = step % P_STAGES;
          const uint32_t ph = (uint32_t)(step / P_STAGES) & 1u;
          if (!wait_or_abort(S, &S.pk_empty[s], ph ^ 1u, status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&S.pk_full[s], kTxBytes);
          ptx::tma_load_2d(S.pkA[s], &tmA, &S.pk_full[s], kg * BKB, m0);
          ptx::tma_load_2d(S.pkB[s], &tmB, &S.pk_full[s], kg * BKB, n0);
        }
      }
      // Drain: every load issued lands before the CTA may exit.
      for (int j = (step > P_STAGES ? step - P_STAGES : 0); j < step; ++j)
        drain_wait(&S.pk_full[j % P_STAGES], (uint32_t)(j / P_STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_i8(BM, BN);
      int step = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kg = 0; kg < G; ++kg, ++step) {
          const int us = step % U_STAGES;
          const uint32_t uph = (uint32_t)(step / U_STAGES) & 1u;
          const int b = step & 1;
          const uint32_t u = (uint32_t)(step >> 1);
          if (!wait_or_abort(S, &S.acc_empty[b], u & 1u, status)) { ok = false; break; }
          if (!wait_or_abort(S, &S.up_full[us], uph, status)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_addr(S.upA[us]);
          const uint32_t b0 = ptx::smem_addr(S.upB[us]);
          const uint32_t d = tmem + (uint32_t)b * BN;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::umma_i8(d, ptx::smem_desc_sw128(a0 + 32 * k), ptx::smem_desc_sw128(b0 + 32 * k), idesc, 1u);
          ptx::umma_commit(&S.up_empty[us]);
          ptx::umma_commit(&S.acc_full[b]);
        }
      }
      ptx::umma_commit(&S.mma_done);
      drain_wait(&S.mma_done, 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------------ unpack
    const int uw = warp - 4;
    const int r8 = lane & 7, p = lane >> 3;
    int step = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kg = 0; kg < G; ++kg, ++step) {
        const int s = step % P_STAGES;
        const uint32_t ph = (uint32_t)(step / P_STAGES) & 1u;
        const int us = step % U_STAGES;
        const uint32_t uph = (uint32_t)(step / U_STAGES) & 1u;
        if (!__all_sync(0xffffffffu, wait_or_abort(S, &S.pk_full[s], ph, status))) { ok = false; break; }
        if (!__all_sync(0xffffffffu, wait_or_abort(S, &S.up_empty[us], uph ^ 1u, status))) { ok = false; break; }
#pragma unroll 4
        for (int k = 0; k < (BM + BN) / 8 / NUM_UNPACK_WARPS; ++k) {
          const int octet = uw + NUM_UNPACK_WARPS * k;      // 8-row block; 0..15 A, 16..47 W
          const bool isA = octet < BM / 8;
          const int r = (isA ? octet : octet - BM / 8) * 8 + r8;
          const uint8_t* src = (isA ? S.pkA[s] : S.pkB[s]) + r * BKB;
          uint8_t* dst = (isA ? S.upA[us] : S.upB[us]) + r * 128;
          const uint4 w = *reinterpret_cast<const uint4*>(src + ((p ^ ((r >> 1) & 3)) << 4));
          *reinterpret_cast<uint4*>(dst + ((p ^ (r & 7)) << 4)) = unpack_lo(w);
          *reinterpret_cast<uint4*>(dst + (((p + 4) ^ (r & 7)) << 4)) = unpack_hi(w);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(&S.pk_empty[s]);
          ptx::mbar_arrive(&S.up_full[us]);
        }
      }
    }
  }
}

__device__ __forceinline__ void cta_epilogue(GemmSmem& S, uint32_t tmem, const float* __restrict__ scales_A,
                                             const float* __restrict__ scales_W, void* __restrict__ Y, int T, int N,
                                             int G, int out_bf16, int m_tiles, int num_tiles, unsigned int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    // ---------------------------------------------------------------------- epilogue
    const int ew = warp - 8;
    const int sub = ew & 3;            // TMEM lane quarter this warp may access
    const int ch = ew >> 2;            // column half of the tile
    float* swb = S.sw_buf[ew];
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    // Pre-load both accumulator buffers with the conversion bias, then release them.
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int c = 0; c < 8; ++c) ptx::tmem_st16_fill(tmem + lane_base + b * BN + ch * 128 + 16 * c, kAccBias);
    ptx::tmem_st_wait();
    ptx::tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      ptx::mbar_arrive(&S.acc_empty[0]);
      ptx::mbar_arrive(&S.acc_empty[1]);
    }
    int step = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m0 = (tile % m_tiles) * BM, n0 = (tile / m_tiles) * BN;
      const int t = m0 + sub * 32 + lane;
      const int ncol = n0 + ch * 128;
      const bool row_ok = t < T;
      const float* sa_row = scales_A + (int64_t)(row_ok ? t : 0) * G;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      // Prefetch group 0 scales: this lane's 4 columns of sw, and its row's sa.
      float sa_next = row_ok ? __ldg(sa_row) : 0.0f;
      float sw_next[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = ncol + 4 * lane + i;
        sw_next[i] = n < N ? __ldg(scales_W + (int64_t)n * G) : 0.0f;
      }
      for (int kg = 0; kg < G; ++kg, ++step) {
        const int b = step & 1;
        const uint32_t u = (uint32_t)(step >> 1);
        const float sa = sa_next * 0.00390625f;           // folds the 16 x 16 of the unpack
        *reinterpret_cast<float4*>(swb + 4 * lane) = make_float4(sw_next[0], sw_next[1], sw_next[2], sw_next[3]);
        if (kg + 1 < G) {
          sa_next = row_ok ? __ldg(sa_row + kg + 1) : 0.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int n = ncol + 4 * lane + i;
            sw_next[i] = n < N ? __ldg(scales_W + (int64_t)n * G + kg + 1) : 0.0f;
          }
        }
        __syncwarp();
        if (!__all_sync(0xffffffffu, wait_or_abort(S, &S.acc_full[b], u & 1u, status))) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t taddr = tmem + lane_base + (uint32_t)(b * BN + ch * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t r[16];
          ptx::tmem_ld16(taddr + 16 * c, r);
          ptx::tmem_ld_wait();
          ptx::tmem_st16_fill(taddr + 16 * c, kAccBias);
#pragma unroll
          for (int j = 0; j < 16; j += 4) {
            const float4 w = *reinterpret_cast<const float4*>(swb + 16 * c + j);
            acc[16 * c + j + 0] = fmaf(__uint_as_float(r[j + 0]) - kAccBiasF, sa * w.x, acc[16 * c + j + 0]);
            acc[16 * c + j + 1] = fmaf(__uint_as_float(r[j + 1]) - kAccBiasF, sa * w.y, acc[16 * c + j + 1]);
            acc[16 * c + j + 2] = fmaf(__uint_as_float(r[j + 2]) - kAccBiasF, sa * w.z, acc[16 * c + j + 2]);
            acc[16 * c + j + 3] = fmaf(__uint_as_float(r[j + 3]) - kAccBiasF, sa * w.w, acc[16 * c + j + 3]);
          }
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.acc_empty[b]);
      }
      if (!ok) break;
      if (row_ok) {
        if (!out_bf16) {
          float* yrow = reinterpret_cast<float*>(Y) + (int64_t)t * N + ncol;
#pragma unroll
          for (int j = 0; j < 128; j += 4)
            if (ncol + j < N)
              *reinterpret_cast<float4*>(yrow + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
        } else {
          __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(Y) + (int64_t)t * N + ncol;
#pragma unroll
          for (int j = 0; j < 128; j += 8) {
            if (ncol + j < N) {
              uint4 o;
              __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j], acc[j + 1]);
              __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
              __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j + 4], acc[j + 5]);
              __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j + 6], acc[j + 7]);
              o.x = *reinterpret_cast<uint32_t*>(&h0);
              o.y = *reinterpret_cast<uint32_t*>(&h1);
              o.z = *reinterpret_cast<uint32_t*>(&h2);
              o.w = *reinterpret_cast<uint32_t*>(&h3);
              *reinterpret_cast<uint4*>(yrow + j) = o;
            }
          }
        }
      }
    }
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) w4a4_gemm_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const float* __restrict__ scales_A, const float* __restrict__ scales_W, void* __restrict__ Y,
    int T, int N, int G, int out_bf16, int m_tiles, int n_tiles, unsigned int* status) {
  extern __shared__ unsigned char smem_raw[];
  GemmSmem& S = *reinterpret_cast<GemmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = m_tiles * n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      ptx::mbar_init(&S.pk_full[s], 1);
      ptx::mbar_init(&S.pk_empty[s], NUM_UNPACK_WARPS);
    }
    for (int s = 0; s < U_STAGES; ++s) {
      ptx::mbar_init(&S.up_full[s], NUM_UNPACK_WARPS);
      ptx::mbar_init(&S.up_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.acc_full[b], 1);
      ptx::mbar_init(&S.acc_empty[b], NUM_EPI_WARPS);
    }
    ptx::mbar_init(&S.mma_done, 1);
    S.abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&S.tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = S.tmem_slot;

  if (warp < 8) {
    ptx::setmaxnreg_dec<72>();
    cta_producer_mma_unpack(S, tmA, tmB, tmem, G, m_tiles, num_tiles, status);
  } else {
    ptx::setmaxnreg_inc<184>();
    cta_epilogue(S, tmem, scales_A, scales_W, Y, T, N, G, out_bf16, m_tiles, num_tiles, status);
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}


typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

pq_status make_packed_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t D, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    set_error("cuTensorMapEncodeTiled is unavailable from the driver");
    return PQ_ERR_CUDA;
  }
  cuuint64_t dims[2] = {(cuuint64_t)(D / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(D / 2)};
  cuuint32_t box[2] = {(cuuint32_t)BKB, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d) for rows=%lld D=%lld", (int)r, (long long)rows, (long long)D);
    return PQ_ERR_CUDA;
  }
  return PQ_OK;
}

int device_sm_count() {
  int dev = 0, c = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
  return c;
}

}  // namespace

pq_status gemm_run(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                   int64_t T, int64_t N, int64_t D, void* Y, pq_out_dtype out_dtype, cudaStream_t stream) {
  CUtensorMap tmA, tmB;
  pq_status st = make_packed_map(&tmA, codes_A, T, D, BM);
  if (st != PQ_OK) return st;
  st = make_packed_map(&tmB, codes_W, N, D, BN);
  if (st != PQ_OK) return st;
  const int m_tiles = (int)((T + BM - 1) / BM);
  const int n_tiles = (int)((N + BN - 1) / BN);
  const int64_t tiles = (int64_t)m_tiles * n_tiles;
  if (tiles >= ((int64_t)1 << 31)) {
    set_error("too many tiles");
    return PQ_ERR_INVALID_ARG;
  }
  const int sms = device_sm_count();
  const int grid = (int)(tiles < sms ? tiles : sms);
  cudaError_t e = cudaFuncSetAttribute(w4a4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm smem)");
  unsigned int* status = nullptr;
  e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_gemm_status);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(gemm status)");
  w4a4_gemm_kernel<<<grid, NUM_THREADS, kSmemBytes, stream>>>(tmA, tmB, scales_A, scales_W, Y, (int)T, (int)N,
                                                               (int)(D / 128), out_dtype == PQ_OUT_BF16 ? 1 : 0,
                                                               m_tiles, n_tiles, status);
  return cuda_fail(cudaGetLastError(), "w4a4_gemm_kernel launch");
}

pq_status gemm_read_and_clear_status(unsigned int* bits) {
  unsigned int v = 0;
  pq_status st = cuda_fail(cudaMemcpyFromSymbol(&v, g_gemm_status, sizeof(v)), "read gemm status");
  if (st != PQ_OK) return st;
  if (v) {
    const unsigned int zero = 0;
    st = cuda_fail(cudaMemcpyToSymbol(g_gemm_status, &zero, sizeof(zero)), "clear gemm status");
    if (st != PQ_OK) return st;
  }
  *bits = v;
  return PQ_OK;
}

}  // namespace pq
