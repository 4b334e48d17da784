// W4A4 GEMM with per-group scales on tcgen05 tensor cores (sm_100a).
//
// Y[t][n] = sum_G sa[t][G] * sw[n][G] * d_G[t][n],  d_G = sum_{k in group G} qa[t][k] qw[n][k]
// (RRS page, main equation, last line; Fig. 4 step (3): the GEMM's K-block equals the
// quantisation group and the block's scales are applied to the interim integer result).
//
// Two kernels per call, ordered on the caller's stream:
//
// 1. expand_codes_kernel: int4 -> int8 for A and W into stream-ordered scratch.  Within each
//    128-element group the low nibbles of the 64 packed bytes become K positions 0..63 and the
//    high nibbles 64..127 (the same permutation on A and W, so every dot product is unchanged),
//    each byte holding 16*code: no sign extension is needed and d = 256 * dot exactly.  The
//    scratch rows are laid out so that one TMA box of 128 bytes x rows lands directly in the
//    128-byte-swizzled K-major operand layout of the MMA.  (Unpacking inside the contraction
//    kernel costs an extra shared-memory read and a double-size write per operand byte, and
//    tensor-core operand reads take priority over that traffic on the shared-memory banks.)
//
// 2. w4a4_gemm_kernel: persistent, one CTA per SM.  The MMA computes the transposed tile
//    D[n][t] (M = 128 output channels = TMEM lanes, N = 256 tokens), so every epilogue thread owns
//    one output channel and its weight scale is a register constant; only the token scales are
//    broadcast from shared memory.  The K loop runs one 128-wide group per step.  Warp roles
//    (12 warps):
//      warp 0      TMA producer: int8 tiles of W (128 x 128 B) and X (256 x 128 B) per group
//                  into a 4-stage ring.
//      warp 1      TMEM allocator and MMA issuer: 4 x tcgen05.mma kind::i8 (M128 N256 K32) per
//                  group into a double-buffered int32 accumulator in tensor memory.
//      warps 2..3  scale loaders: per group, the tile's 128 weight scales and 256 activation
//                  scales are copied (cp.async, zero-filled past N / T) into an 8-stage ring.
//      warps 4..11 epilogue (2 per TMEM lane quarter, 128 tokens each): per group, read the
//                  int32 tile from TMEM and accumulate
//                  acc += fl(d * sw) * sa / 256 in float32 registers (ascending group order) with
//                  two packed f32x2 FMAs per column pair; after the last group, store Y.
//    Exact int32 -> float32 conversion and weight scaling in one FMA: each accumulator buffer is
//    pre-loaded with the bit pattern of C = 1.5*2^23; since |d| <= 2^21, (bits + d) is the float
//    C + d.  The weight scale is rounded to a 22-bit significand (relative change <= 2^-22), which
//    makes C * sw exact, so fma(C + d, sw, -C * sw) = fl(d * sw) with one rounding.  Weight scales
//    must satisfy |sw| < 2^100 for C * sw to stay finite.  Every mbarrier wait is bounded; a timeout
//    sets a status bit, the CTA drains its own copies and MMAs, frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace pq {

__device__ unsigned int g_gemm_status = 0;

namespace {

constexpr int BM = 128;        // tile rows = output channels (weight rows), MMA M
constexpr int BN = 256;        // tile columns = tokens (activation rows), MMA N
constexpr int BK = 128;        // one quantisation group = 128 int8 = one 128-byte swizzle row
constexpr int OP_STAGES = 4;   // operand ring
constexpr int S_STAGES = 8;    // scale ring
constexpr int NUM_THREADS = 384;
constexpr int NUM_EPI_WARPS = 8;
constexpr int EPI_COLS = BN / (NUM_EPI_WARPS / 4);   // tokens per epilogue warp (64)
constexpr int EPI_WARP0 = 4;
constexpr int NUM_SCALE_THREADS = 64;  // warps 2 and 3
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t kAccBias = 0x4B400000u;          // bit pattern of 1.5 * 2^23
constexpr float kAccBiasF = 12582912.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;    // 2 s
constexpr uint32_t kTxBytes = (BM + BN) * BK;

struct __align__(1024) GemmSmem {
  uint8_t opA[OP_STAGES][BM * BK];   // weights, 16 KB per stage, 128-byte swizzle
  uint8_t opB[OP_STAGES][BN * BK];   // activations, 32 KB per stage
  float sc_w[S_STAGES][BM];          // weight scales of the tile's rows, one group per stage
  float sc_a[S_STAGES][BN];          // activation scales of the tile's columns
  uint64_t op_full[OP_STAGES];
  uint64_t op_empty[OP_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t sc_full[S_STAGES];
  uint64_t sc_empty[S_STAGES];
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

// Warp-wide wait: only lane 0 polls the barrier (32 lanes polling one word serialise on a
// shared-memory bank); the outcome is broadcast and __syncwarp orders the other lanes' later
// accesses after lane 0's acquire.
__device__ __forceinline__ bool warp_wait_or_abort(GemmSmem& S, uint64_t* bar, uint32_t parity,
                                                   unsigned int* status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_or_abort(S, bar, parity, status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Wait used while draining: ignores the abort flag, bounded in time only.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int never = 0;
  (void)ptx::mbar_wait_bounded(bar, parity, &never, kWaitLimitNs);
}

// ------------------------------------------------------------------------------ expand
// One thread per 16 packed bytes (32 codes of one group): writes the 16 low-nibble bytes at K
// offset 16p and the 16 high-nibble bytes at 64 + 16p of the group's 128-byte int8 row.
__global__ void __launch_bounds__(256) expand_codes_kernel(const uint8_t* __restrict__ A, int64_t chunksA,
                                                           const uint8_t* __restrict__ W, int64_t chunksW,
                                                           uint8_t* __restrict__ A8, uint8_t* __restrict__ W8) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunksA + chunksW; i += stride) {
    const bool isA = i < chunksA;
    const int64_t c = isA ? i : i - chunksA;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(isA ? A : W) + c);
    const int64_t group = c >> 2;          // 4 chunks of 16 bytes per 64-byte packed group
    const int p = (int)(c & 3);
    uint8_t* dst = (isA ? A8 : W8) + group * 128 + 16 * p;
    *reinterpret_cast<uint4*>(dst) = make_uint4((w.x << 4) & 0xF0F0F0F0u, (w.y << 4) & 0xF0F0F0F0u,
                                                (w.z << 4) & 0xF0F0F0F0u, (w.w << 4) & 0xF0F0F0F0u);
    *reinterpret_cast<uint4*>(dst + 64) =
        make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
  }
}

// -------------------------------------------------------------------------- control
__device__ __forceinline__ void cta_control(GemmSmem& S, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                            const float* __restrict__ scales_A, const float* __restrict__ scales_W,
                                            uint32_t tmem, int T, int N, int G, int m_tiles, int num_tiles,
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
          const int s = step % OP_STAGES;
          const uint32_t ph = (uint32_t)(step / OP_STAGES) & 1u;
          if (!wait_or_abort(S, &S.op_empty[s], ph ^ 1u, status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&S.op_full[s], kTxBytes);
          ptx::tma_load_2d(S.opA[s], &tmA, &S.op_full[s], kg * BK, m0);
          ptx::tma_load_2d(S.opB[s], &tmB, &S.op_full[s], kg * BK, n0);
        }
      }
      // Drain: every load issued lands before the CTA may exit.
      for (int j = (step > OP_STAGES ? step - OP_STAGES : 0); j < step; ++j)
        drain_wait(&S.op_full[j % OP_STAGES], (uint32_t)(j / OP_STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_i8(BM, BN);
      int step = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kg = 0; kg < G; ++kg, ++step) {
          const int s = step % OP_STAGES;
          const uint32_t ph = (uint32_t)(step / OP_STAGES) & 1u;
          const int b = step & 1;
          const uint32_t u = (uint32_t)(step >> 1);
          if (!wait_or_abort(S, &S.acc_empty[b], u & 1u, status)) { ok = false; break; }
          if (!wait_or_abort(S, &S.op_full[s], ph, status)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_addr(S.opA[s]);
          const uint32_t b0 = ptx::smem_addr(S.opB[s]);
          const uint32_t d = tmem + (uint32_t)b * BN;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::umma_i8(d, ptx::smem_desc_sw128(a0 + 32 * k), ptx::smem_desc_sw128(b0 + 32 * k), idesc, 1u);
          ptx::umma_commit(&S.op_empty[s]);
          ptx::umma_commit(&S.acc_full[b]);
        }
      }
      ptx::umma_commit(&S.mma_done);
      drain_wait(&S.mma_done, 0);
    }
  } else {
    // ---------------------------------------------------------------- scale loaders
    const int j = threadIdx.x - 64;                      // 0..63
    int step = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m0 = (tile % m_tiles) * BM, n0 = (tile / m_tiles) * BN;
      for (int kg = 0; kg < G; ++kg, ++step) {
        const int ss = step % S_STAGES;
        const uint32_t sph = (uint32_t)(step / S_STAGES) & 1u;
        if (!warp_wait_or_abort(S, &S.sc_empty[ss], sph ^ 1u, status)) { ok = false; break; }
#pragma unroll
        for (int i = 0; i < BM / NUM_SCALE_THREADS; ++i) {
          const int n = m0 + j + NUM_SCALE_THREADS * i;
          const bool in = n < N;
          ptx::cp_async4(&S.sc_w[ss][j + NUM_SCALE_THREADS * i], scales_W + (int64_t)(in ? n : 0) * G + kg, in ? 4u : 0u);
        }
#pragma unroll
        for (int i = 0; i < BN / NUM_SCALE_THREADS; ++i) {
          const int t = n0 + j + NUM_SCALE_THREADS * i;
          const bool in = t < T;
          ptx::cp_async4(&S.sc_a[ss][j + NUM_SCALE_THREADS * i], scales_A + (int64_t)(in ? t : 0) * G + kg, in ? 4u : 0u);
        }
        ptx::cp_async_arrive_noinc(&S.sc_full[ss]);
      }
    }
    ptx::cp_async_wait_all();
  }
}

// ------------------------------------------------------------------------- epilogue
__device__ __forceinline__ void cta_epilogue(GemmSmem& S, uint32_t tmem, void* __restrict__ Y, int T, int N,
                                             int G, int out_bf16, int m_tiles, int num_tiles, unsigned int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ew = warp - EPI_WARP0;
  const int sub = warp & 3;          // TMEM lane quarter this warp may access
  const int ch = ew >> 2;            // token half of the tile
  const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
  // Pre-load both accumulator buffers with the conversion bias, then release them.
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int c = 0; c < EPI_COLS / 16; ++c) ptx::tmem_st16_fill(tmem + lane_base + b * BN + ch * EPI_COLS + 16 * c, kAccBias);
  ptx::tmem_st_wait();
  ptx::tc_fence_before();
  __syncwarp();
  if (lane == 0) {
    ptx::mbar_arrive(&S.acc_empty[0]);
    ptx::mbar_arrive(&S.acc_empty[1]);
  }
  int step = 0;
  bool ok = true;
  bool pending = false;              // re-arm stores of the previous step not yet waited for
  int prev_b = 0, prev_ss = 0;
  for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
    const int m0 = (tile % m_tiles) * BM, n0 = (tile / m_tiles) * BN;
    const int n = m0 + sub * 32 + lane;        // this thread's output channel
    const int tcol = n0 + ch * EPI_COLS;       // first of this warp's tokens
    float acc[EPI_COLS];                       // Y[tcol + j][n], float32
#pragma unroll
    for (int i = 0; i < EPI_COLS; ++i) acc[i] = 0.0f;
    for (int kg = 0; kg < G; ++kg, ++step) {
      const int b = step & 1;
      const uint32_t u = (uint32_t)(step >> 1);
      const int ss = step % S_STAGES;
      const uint32_t sph = (uint32_t)(step / S_STAGES) & 1u;
      if (!warp_wait_or_abort(S, &S.sc_full[ss], sph, status)) { ok = false; break; }
      // Weight scale / 256 (undoes the 16 x 16 of the expansion, exactly), rounded to a 22-bit
      // significand so that C * sw is exact.
      const float sw = __uint_as_float((__float_as_uint(S.sc_w[ss][sub * 32 + lane] * 0.00390625f) + 2u) & ~3u);
      const float csw = -kAccBiasF * sw;
      const uint64_t sw2 = ptx::f2_pack(sw, sw), csw2 = ptx::f2_pack(csw, csw);
      const float4* sap = reinterpret_cast<const float4*>(&S.sc_a[ss][ch * EPI_COLS]);
      if (!warp_wait_or_abort(S, &S.acc_full[b], u & 1u, status)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t taddr = tmem + lane_base + (uint32_t)(b * BN + ch * EPI_COLS);
#pragma unroll
      for (int c = 0; c < EPI_COLS / 32; ++c) {
        uint32_t r[32];
        ptx::tmem_ld32(taddr + 32 * c, r);
        ptx::tmem_ld_wait();
        if (c == 0 && pending) {
          // The previous buffer's bias stores were issued a whole TMEM load ago: complete them
          // and hand that buffer back to the MMA.
          ptx::tmem_st_wait();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            ptx::mbar_arrive(&S.acc_empty[prev_b]);
            ptx::mbar_arrive(&S.sc_empty[prev_ss]);
          }
          pending = false;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i0 = 32 * c + 4 * j;
          ptx::epi_fma4(acc[i0], acc[i0 + 1], acc[i0 + 2], acc[i0 + 3], sap[8 * c + j], sw2, csw2, r[4 * j],
                        r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        }
      }
      // Re-arm this buffer with the conversion bias for the MMA two steps ahead; completion is
      // awaited after the next step's first TMEM load.
#pragma unroll
      for (int c = 0; c < EPI_COLS / 4; ++c) ptx::tmem_st4_fill(taddr + 4 * c, kAccBias);
      pending = true;
      prev_b = b;
      prev_ss = ss;
    }
    if (!ok) break;
    // Y[t][n]: the 32 lanes of a warp write 32 consecutive channels of one token per store.
    if (n < N) {
      if (!out_bf16) {
        float* ycol = reinterpret_cast<float*>(Y) + (int64_t)tcol * N + n;
#pragma unroll
        for (int j = 0; j < EPI_COLS; ++j)
          if (tcol + j < T) ycol[(int64_t)j * N] = acc[j];
      } else {
        __nv_bfloat16* ycol = reinterpret_cast<__nv_bfloat16*>(Y) + (int64_t)tcol * N + n;
#pragma unroll
        for (int j = 0; j < EPI_COLS; ++j)
          if (tcol + j < T) ycol[(int64_t)j * N] = __float2bfloat16_rn(acc[j]);
      }
    }
  }
  if (pending) {
    ptx::tmem_st_wait();
    ptx::tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      ptx::mbar_arrive(&S.acc_empty[prev_b]);
      ptx::mbar_arrive(&S.sc_empty[prev_ss]);
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
    for (int s = 0; s < OP_STAGES; ++s) {
      ptx::mbar_init(&S.op_full[s], 1);
      ptx::mbar_init(&S.op_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.acc_full[b], 1);
      ptx::mbar_init(&S.acc_empty[b], NUM_EPI_WARPS);
    }
    for (int s = 0; s < S_STAGES; ++s) {
      ptx::mbar_init(&S.sc_full[s], NUM_SCALE_THREADS);
      ptx::mbar_init(&S.sc_empty[s], NUM_EPI_WARPS);
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

  // Register budget: 384 threads x 168 at launch; warps 0..3 give back to 56, warps 4..11 take
  // 224 (128 x 56 + 256 x 224 = 64512 = 384 x 168).
  if (warp < EPI_WARP0) {
    ptx::setmaxnreg_dec<56>();
    cta_control(S, tmA, tmB, scales_A, scales_W, tmem, T, N, G, m_tiles, num_tiles, status);
  } else {
    ptx::setmaxnreg_inc<224>();
    cta_epilogue(S, tmem, Y, T, N, G, out_bf16, m_tiles, num_tiles, status);
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

// int8 [rows][D] operand, box of 128 bytes (one group) x box_rows, 128-byte swizzle.
pq_status make_operand_map(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t D, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    set_error("cuTensorMapEncodeTiled is unavailable from the driver");
    return PQ_ERR_CUDA;
  }
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d) for rows=%lld D=%lld", (int)r, (long long)rows, (long long)D);
    return PQ_ERR_CUDA;
  }
  return PQ_OK;
}

// Library-owned stream-ordered pool per device.  Its release threshold is unlimited, so memory
// freed at the end of one call is reused by the next instead of being unmapped at every
// synchronisation (which made each call pay for fresh page mappings).
cudaError_t scratch_pool(cudaMemPool_t* out) {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = UINT64_MAX;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return e;
    }
    pools[dev] = pool;
  }
  *out = pools[dev];
  return cudaSuccess;
}

int device_sm_count() {
  int dev = 0, c = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
  return c;
}

}  // namespace

size_t gemm_scratch_bytes(int64_t T, int64_t N, int64_t D) { return (size_t)(T + N) * (size_t)D; }

pq_status gemm_launch(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                      int64_t T, int64_t N, int64_t D, void* Y, pq_out_dtype out_dtype, uint8_t* scratch,
                      unsigned int* status, cudaStream_t stream) {
  uint8_t* A8 = scratch;
  uint8_t* W8 = scratch + (size_t)T * (size_t)D;
  // MMA operand A = weights (M = output channels), B = activations (N = tokens).
  CUtensorMap tmA, tmB;
  pq_status st = make_operand_map(&tmA, W8, N, D, BM);
  if (st != PQ_OK) return st;
  st = make_operand_map(&tmB, A8, T, D, BN);
  if (st != PQ_OK) return st;
  const int m_tiles = (int)((N + BM - 1) / BM);
  const int n_tiles = (int)((T + BN - 1) / BN);
  const int64_t tiles = (int64_t)m_tiles * n_tiles;
  if (tiles >= ((int64_t)1 << 31)) {
    set_error("too many tiles");
    return PQ_ERR_INVALID_ARG;
  }
  const int sms = device_sm_count();
  const int64_t chunksA = T * (D / 32), chunksW = N * (D / 32);   // 16 packed bytes each
  const int64_t want = (chunksA + chunksW + 255) / 256;
  const int egrid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  expand_codes_kernel<<<egrid, 256, 0, stream>>>(codes_A, chunksA, codes_W, chunksW, A8, W8);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "expand_codes_kernel launch");
  const int grid = (int)(tiles < sms ? tiles : sms);
  e = cudaFuncSetAttribute(w4a4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm smem)");
  w4a4_gemm_kernel<<<grid, NUM_THREADS, kSmemBytes, stream>>>(tmA, tmB, scales_A, scales_W, Y, (int)T, (int)N,
                                                               (int)(D / 128), out_dtype == PQ_OUT_BF16 ? 1 : 0,
                                                               m_tiles, n_tiles, status);
  return cuda_fail(cudaGetLastError(), "w4a4_gemm_kernel launch");
}

pq_status gemm_run(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                   int64_t T, int64_t N, int64_t D, void* Y, pq_out_dtype out_dtype, cudaStream_t stream) {
  unsigned int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_gemm_status);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(gemm status)");
  // Stream-ordered scratch for the int8 operands: allocated and released on the caller's
  // stream, so concurrent calls on different streams never share it.
  cudaMemPool_t pool = nullptr;
  e = scratch_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "scratch memory pool");
  void* scratch = nullptr;
  e = cudaMallocFromPoolAsync(&scratch, gemm_scratch_bytes(T, N, D), pool, stream);
  if (e != cudaSuccess) {
    set_error("cudaMallocFromPoolAsync(%zu bytes of GEMM scratch): %s", gemm_scratch_bytes(T, N, D),
              cudaGetErrorString(e));
    return PQ_ERR_ALLOC;
  }
  pq_status st = gemm_launch(codes_A, scales_A, codes_W, scales_W, T, N, D, Y, out_dtype,
                             static_cast<uint8_t*>(scratch), status, stream);
  e = cudaFreeAsync(scratch, stream);
  if (st == PQ_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(gemm scratch)");
  return st;
}

cudaError_t gemm_status_address(unsigned int** status) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(status), g_gemm_status);
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
