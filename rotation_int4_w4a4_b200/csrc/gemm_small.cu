// W4A4 GEMM for few tokens (4 < T <= 128; at most 4 tokens take the CUDA-core kernel of gemv.cu) on
// tcgen05 tensor cores (sm_100a).
//
// Y[t][n] = sum_G sa[t][G] * sw[n][G] * d_G[t][n] (RRS page, main equation, last line; Fig. 4
// step (3) with block size = group size), as in gemm.cu, for calls whose cost is streaming the
// packed weights: W is read from HBM once, as int4, and nothing is written back but Y.
//
// A work unit is 128 weight rows x a range of groups; persistent CTAs take the units in turn.
// Codes move in K-blocks of 128 (64 packed bytes per row); a group is g / 128 of a block (g = 64),
// one block (g = 128) or two (g = 256).
//   warp 0      TMA: four K-blocks per stage, as two boxes of two blocks (128 contiguous bytes of
//               each row, 128-byte swizzle) for the unit's 128 weight rows and for the NT token
//               rows (rows past T read as zeros), into a ring of 2..4 stages.  Row segments of
//               128 bytes keep the L2 and DRAM requests large.
//   warp 1      TMEM allocator and MMA issuer: g / 32 tcgen05.mma kind::i8 (M128, N = NT, K32) per
//               group into a ring of int32 accumulators (the first of them overwrites).
//   warps 4..7  widening (one warp per scheduler), one K-block at a time into a ring of operand
//               stages deep enough to cover the MMA's completion latency: each packed byte's two
//               nibbles become two int8 values q * 16 (the nibble moved to the byte's top: one
//               shift and one mask per four bytes, exact), written in the 128-byte-swizzled
//               K-major operand layout.  Within each 128-code block the low nibbles land at K
//               positions 0..63 and the high nibbles at 64..127 (g = 64: within each 64-code
//               half, 0..31 and 32..63), on both operands alike, so every group's dot product is
//               unchanged; it comes out as 256 d_G, exact in int32 (|256 d_G| <= 2^22).  Eight
//               consecutive threads take eight consecutive rows of one 16-byte column, which the
//               swizzle spreads over all banks.
//   warps 8..11 epilogue: one thread per weight row (TMEM lane), NT tokens; per group
//               acc += float(256 d_G) * (sw / 256) * sa, the same float32 value and rounding as
//               fl(d_G * sw) * sa, groups in ascending order.
//   (warps 2..3 have no role.)  The warpgroups re-divide the registers with setmaxnreg: the
//   control and widening warps need few, the epilogue holds NT float accumulators per thread.
// Units cover all groups (one launch writes Y) unless the weights are too few rows to fill the
// device; then the groups are split into ranges (multiples of 4 groups) whose float32 partial
// tiles are summed in ascending range order by a second kernel.  Every mbarrier wait is bounded;
// a timeout sets the status bit and the CTA drains its copies and MMAs before freeing tensor
// memory.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace pq {
namespace {

constexpr int GS_M = 128;           // weight rows per unit (MMA M = TMEM lanes)
constexpr int GS_GPS = 4;           // group ranges are multiples of 4 groups
constexpr int GS_KPS = 4;           // K-blocks (128 codes, 64 packed bytes) per packed-code stage
constexpr int GS_SC = 8;            // groups of token scales staged per epilogue warp at a time
constexpr int GS_THREADS = 384;     // warp 0 TMA, 1 MMA, 4..7 widening, 8..11 epilogue
constexpr int GS_WIDEN0 = 4;        // first widening warp
constexpr int GS_WIDEN = 4;         // widening warps
constexpr int GS_EPI0 = 8;          // first epilogue warp
constexpr uint64_t kGsWaitNs = 2000000000ull;   // 2 s
// Registers per thread: at launch (384 threads), then per warpgroup after setmaxnreg.  The
// shares must fit in the launch allocation, so the host checks the compiled count.
constexpr uint32_t GS_REG_CTRL = 72, GS_REG_WIDEN = 80, GS_REG_EPI = 232;
constexpr uint32_t kGsRegBudget = 128 * (GS_REG_CTRL + GS_REG_WIDEN + GS_REG_EPI);
static_assert(kGsRegBudget <= 65536, "register shares exceed the SM");

// Ring depths per token width, as deep as shared memory (227 KB) and tensor memory allow:
// packed-code stages (4 groups each), int8 operand stages (1 group), accumulator buffers.
template <int NT>
constexpr int raw_stages() { return NT <= 16 ? 4 : NT <= 64 ? (NT == 32 ? 3 : 2) : 2; }
template <int NT>
constexpr int op_stages() { return NT <= 64 ? 4 : 2; }
template <int NT>
constexpr int acc_bufs() { return NT <= 64 ? 4 : 2; }

template <int NT>
struct __align__(1024) SmallSmem {
  static constexpr int RAW = raw_stages<NT>(), OPS = op_stages<NT>(), NACC = acc_bufs<NT>();
  uint8_t opW[OPS][GS_M * 128];         // int8 q * 16, 128-byte-swizzled K-major rows
  uint8_t opA[OPS][NT * 128];
  uint8_t rawW[RAW][2][GS_M * 128];     // packed codes, two groups per 128-byte swizzled row
  uint8_t rawA[RAW][2][NT * 128];
  float sa[4][2][GS_SC][NT];            // token scales per epilogue warp, double-buffered: [group][token]
  uint64_t raw_full[RAW], raw_empty[RAW];
  uint64_t op_full[OPS], op_empty[OPS];
  uint64_t acc_full[NACC], acc_empty[NACC];
  uint64_t mma_done;
  uint32_t tmem_slot;
  int abort_flag;
};

template <int NT>
constexpr size_t small_smem_bytes() { return sizeof(SmallSmem<NT>) + 1024; }

template <int NT>
__device__ __forceinline__ bool gs_wait(SmallSmem<NT>& S, uint64_t* bar, uint32_t parity, unsigned int* status) {
  if (ptx::mbar_wait_bounded(bar, parity, &S.abort_flag, kGsWaitNs)) return true;
  S.abort_flag = 1;
  atomicOr(status, PQ_DEV_TIMEOUT);
  return false;
}

template <int NT>
__device__ __forceinline__ bool gs_warp_wait(SmallSmem<NT>& S, uint64_t* bar, uint32_t parity, unsigned int* status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = gs_wait(S, bar, parity, status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ void gs_drain(uint64_t* bar, uint32_t parity) {
  int never = 0;
  (void)ptx::mbar_wait_bounded(bar, parity, &never, kGsWaitNs);
}

// One K-block (128 codes) of ROWS rows: the 64 packed bytes of row r sit in the `half` 64-byte
// half of the row's 128-byte swizzled segment in `raw`; they become 128 int8 values in the row's
// 128-byte swizzled operand row in `op` (16-byte chunk c stored at c XOR (row mod 8) in both).
// Task i: row i % ROWS, 16-byte column p = i / ROWS.  g >= 128: low nibbles -> chunk p, high ->
// chunk p + 4; g = 64 (two groups per block): low -> chunk 4 (p / 2) + p % 2, high -> that + 2,
// so that each group's codes stay within its own 64 K positions.  All loads are issued before
// any store.
template <int ROWS>
__device__ __forceinline__ void widen_block(const uint8_t* raw, uint8_t* op, int half, int ct, int g64) {
  constexpr int TASKS = ROWS * 4, NTH = 32 * GS_WIDEN, PER = (TASKS + NTH - 1) / NTH;
  uint4 v[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int i = ct + NTH * q;
    if (TASKS % NTH == 0 || i < TASKS) {
      const int row = i % ROWS, p = i / ROWS;
      v[q] = *reinterpret_cast<const uint4*>(raw + row * 128 + (((half * 4 + p) ^ (row & 7)) << 4));
    }
  }
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int i = ct + NTH * q;
    if (TASKS % NTH == 0 || i < TASKS) {
      const int row = i % ROWS, p = i / ROWS;
      const int lo = g64 ? (((p & 2) << 1) | (p & 1)) : p, hi = lo + (g64 ? 2 : 4);
      const uint4 w = v[q];
      uint8_t* base = op + row * 128;
      *reinterpret_cast<uint4*>(base + ((lo ^ (row & 7)) << 4)) =
          make_uint4((w.x << 4) & 0xF0F0F0F0u, (w.y << 4) & 0xF0F0F0F0u, (w.z << 4) & 0xF0F0F0F0u,
                     (w.w << 4) & 0xF0F0F0F0u);
      *reinterpret_cast<uint4*>(base + ((hi ^ (row & 7)) << 4)) =
          make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
    }
  }
}

struct Unit {
  int m0, kr, k0, k1;
};

__device__ __forceinline__ Unit unit_of(int u, int ranges, int gs, int G) {
  Unit w;
  const int tile = u / ranges;
  w.kr = u - tile * ranges;
  w.m0 = tile * GS_M;
  w.k0 = w.kr * gs;
  w.k1 = min(G, w.k0 + gs);
  return w;
}

// kRow: scales_W holds per-(row, group) factors and scales_A one scale per token: per group
// acc += float(256 d) * (F / 256), and the token's scale multiplies the sum at the end.
template <int NT, bool kRow, int GSL>
__global__ void __launch_bounds__(GS_THREADS, 1) w4a4_gemm_small_kernel(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
    const float* __restrict__ scales_A, const float* __restrict__ scales_W, void* __restrict__ Y,
    float* __restrict__ ws, int T, int N, int G, int ranges, int gs, int units, int out_bf16, int pdl,
    unsigned int* status) {
  // pdl: launched as the programmatic dependent of the kernel that writes codes_A and scales_A
  // (pq_w4a4_linear).  The weights were written before that kernel started, so the first ring
  // of weight tiles is requested at once; activation codes and scales are read only after
  // griddepcontrol.wait (every role that reads them waits first).
  // GSL: K32 slices per group (g / 32 = 2, 4 or 8); a K-block of 128 codes holds 4, an operand
  // stage is one K-block and a packed-code stage four.  Group ranges start on K-block boundaries.
  using Smem = SmallSmem<NT>;
  constexpr int gsl = GSL;
  ptx::griddep_launch_dependents();   // the range reduction may launch now; it waits for this grid
  const int g64 = GSL == 2 ? 1 : 0;
  constexpr int RAW = Smem::RAW, GS_OPS = Smem::OPS, GS_NACC = Smem::NACC;
  constexpr uint32_t kTmemCols = GS_NACC * NT < 32 ? 32 : GS_NACC * NT;
  constexpr uint32_t kRawBytes = 2 * GS_M * 128 + 2 * NT * 128;
  extern __shared__ unsigned char smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW; ++s) {
      ptx::mbar_init(&S.raw_full[s], 1);
      ptx::mbar_init(&S.raw_empty[s], GS_WIDEN);
    }
    for (int o = 0; o < GS_OPS; ++o) {
      ptx::mbar_init(&S.op_full[o], GS_WIDEN);
      ptx::mbar_init(&S.op_empty[o], 1);    // MMA commit
    }
    for (int b = 0; b < GS_NACC; ++b) {
      ptx::mbar_init(&S.acc_full[b], 1);    // MMA commit
      ptx::mbar_init(&S.acc_empty[b], 4);   // the 4 epilogue warps
    }
    ptx::mbar_init(&S.mma_done, 1);
    S.abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmW);
    ptx::prefetch_tmap(&tmA);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&S.tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = S.tmem_slot;

  // Each warpgroup sets its register share at the top of its own branch (every warp of the
  // group executes it), so that the compiler allocates each role's code within that share.
  if (warp < GS_WIDEN0) {
    ptx::setmaxnreg_dec<GS_REG_CTRL>();
  if (warp == 0) {
    // ---------------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int ss = 0;   // stages issued
      bool ok = true;
      // Activation boxes of the first ring fill are deferred (pdl): their stages' weight boxes go
      // out first, then griddepcontrol.wait, then these.
      int pend_kq[RAW];
      int npend = 0;
      bool waited = pdl == 0;
      auto release_pending = [&]() {
        ptx::griddep_wait();
        for (int i = 0; i < npend; ++i)
          for (int b = 0; b < 2; ++b)
            ptx::tma_load_2d(S.rawA[i][b], &tmA, &S.raw_full[i], (pend_kq[i] + 2 * b) * 64, 0);
        npend = 0;
        waited = true;
      };
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit w = unit_of(u, ranges, gs, G);
        const int kb1 = w.k1 * gsl / 4;
        for (int kq = w.k0 * gsl / 4; kq < kb1; kq += GS_KPS, ++ss) {
          const int s = ss % RAW;
          if (!waited && ss == RAW) release_pending();
          if (!gs_wait(S, &S.raw_empty[s], ((uint32_t)(ss / RAW) & 1u) ^ 1u, status)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&S.raw_full[s], kRawBytes);
          for (int b = 0; b < 2; ++b) {   // K-blocks kq + 2b, kq + 2b + 1 (bytes past a row read as zeros)
            ptx::tma_load_2d(S.rawW[s][b], &tmW, &S.raw_full[s], (kq + 2 * b) * 64, w.m0);
            if (waited) ptx::tma_load_2d(S.rawA[s][b], &tmA, &S.raw_full[s], (kq + 2 * b) * 64, 0);
          }
          if (!waited) pend_kq[npend++] = kq;   // ss < RAW: stage s == ss
        }
      }
      if (!waited) release_pending();   // fewer stages than the ring (or an abort): still land them
      // Every load issued lands before the CTA may exit.
      for (int j = ss > RAW ? ss - RAW : 0; j < ss; ++j)
        gs_drain(&S.raw_full[j % RAW], (uint32_t)(j / RAW) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_s8_s32(GS_M, NT);
      int step = 0;    // groups
      int kstep = 0;   // operand stages (K-blocks) consumed
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Unit w = unit_of(u, ranges, gs, G);
        for (int kg = w.k0; kg < w.k1 && ok; ++kg, ++step) {
          const int b = step % GS_NACC;
          if (!gs_wait(S, &S.acc_empty[b], ((uint32_t)(step / GS_NACC) & 1u) ^ 1u, status)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(b * NT);
          // K32 per MMA = 32 bytes along the swizzled row; a stage is awaited at its first slice
          // and released after its fourth; slice 0 of the group overwrites the buffer.  The
          // slices are unrolled (GSL is a template parameter) so the MMAs issue back to back.
          const int h = GSL == 2 ? ((kg - w.k0) & 1) : 0;
#pragma unroll
          for (int sl = 0; sl < GSL; ++sl) {
            const int sub = GSL == 2 ? 2 * h + sl : (sl & 3);
            const int o = kstep % GS_OPS;
            if (sub == 0) {
              if (!gs_wait(S, &S.op_full[o], (uint32_t)(kstep / GS_OPS) & 1u, status)) { ok = false; break; }
              ptx::tc_fence_after();
            }
            const uint32_t a0 = ptx::smem_addr(S.opW[o]), b0 = ptx::smem_addr(S.opA[o]);
            ptx::umma_s8(d, ptx::smem_desc_sw128(a0 + 32 * sub), ptx::smem_desc_sw128(b0 + 32 * sub), idesc,
                         sl > 0 ? 1u : 0u);
            if (sub == 3) {
              ptx::umma_commit(&S.op_empty[o]);
              ++kstep;
            }
          }
          if (!ok) break;
          ptx::umma_commit(&S.acc_full[b]);
        }
      }
      ptx::umma_commit(&S.mma_done);
      gs_drain(&S.mma_done, 0);   // every MMA issued has completed
    }
  }
  } else if (warp < GS_EPI0) {
    ptx::setmaxnreg_dec<GS_REG_WIDEN>();
    // -------------------------------------------------------------------------- widening
    const int ct = threadIdx.x - 32 * GS_WIDEN0;   // 0 .. 32 GS_WIDEN - 1
    int ss = 0, step = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const Unit w = unit_of(u, ranges, gs, G);
      const int kb1 = w.k1 * gsl / 4;
      for (int kq = w.k0 * gsl / 4; kq < kb1 && ok; kq += GS_KPS, ++ss) {
        const int s = ss % RAW;
        if (!gs_warp_wait(S, &S.raw_full[s], (uint32_t)(ss / RAW) & 1u, status)) { ok = false; break; }
        const int nk = min(GS_KPS, kb1 - kq);
        for (int j = 0; j < nk; ++j, ++step) {
          const int o = step % GS_OPS;
          if (!gs_warp_wait(S, &S.op_empty[o], ((uint32_t)(step / GS_OPS) & 1u) ^ 1u, status)) { ok = false; break; }
          widen_block<GS_M>(S.rawW[s][j >> 1], S.opW[o], j & 1, ct, g64);
          widen_block<NT>(S.rawA[s][j >> 1], S.opA[o], j & 1, ct, g64);
          ptx::fence_proxy_async_smem();   // the tensor core reads these bytes through the async proxy
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&S.op_full[o]);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.raw_empty[s]);
      }
    }
  } else {
    ptx::setmaxnreg_inc<GS_REG_EPI>();
    if (pdl) ptx::griddep_wait();   // token scales come from the preceding grid
    // -------------------------------------------------------------------------- epilogue
    const int ew = warp - GS_EPI0;              // 0..3
    const int quarter = warp & 3;               // TMEM lane quarter this warp may access
    const int rl = quarter * 32 + lane;         // weight row within the unit
    float* sa_w = &S.sa[ew][0][0][0];
    // Token scales of groups kg0 .. kg0 + GS_SC - 1 (within the unit) into buffer buf of this
    // warp's copy, [group][token], by asynchronous copies (tokens past T: zeros).
    auto stage = [&](int kg0, int k1, int buf) {
      const int kn = min(GS_SC, k1 - kg0);
      float* dst = sa_w + buf * GS_SC * NT;
      for (int i = lane; i < kn * NT; i += 32) {
        const int gg = i / NT, t = i - gg * NT;
        const bool in = t < T;
        ptx::cp_async4(dst + gg * NT + t, in ? scales_A + (int64_t)t * G + kg0 + gg : scales_A, in ? 4u : 0u);
      }
    };
    int step = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const Unit w = unit_of(u, ranges, gs, G);
      const int n = w.m0 + rl;
      float acc[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
      __syncwarp();                  // the previous unit's reads of the staged scales are done
      if (!kRow) stage(w.k0, w.k1, 0);
      for (int kg = w.k0; kg < w.k1; ++kg, ++step) {
        const int g = (kg - w.k0) % GS_SC;
        const int buf = ((kg - w.k0) / GS_SC) & 1;
        if (!kRow && g == 0) {
          // This batch's scales have landed; start copying the next batch into the other buffer.
          ptx::cp_async_wait_all();
          __syncwarp();
          if (kg + GS_SC < w.k1) stage(kg + GS_SC, w.k1, buf ^ 1);
        }
        // The dot arrives as 256 d: the weight scale carries the exact factor 1/256.
        const float swv = n < N ? __ldg(scales_W + (int64_t)n * G + kg) * 0.00390625f : 0.0f;
        const int b = step % GS_NACC;
        if (!gs_warp_wait(S, &S.acc_full[b], (uint32_t)(step / GS_NACC) & 1u, status)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * NT);
        const float* sag = sa_w + (buf * GS_SC + g) * NT;
#pragma unroll
        for (int c = 0; c < NT / 16; ++c) {
          uint32_t d[16];
          ptx::tmem_ld32x16(ta + 16 * c, d);
          ptx::tmem_ld_wait();
          if (c == NT / 16 - 1) {
            // The whole accumulator is read: hand the buffer back before the arithmetic.
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&S.acc_empty[b]);
          }
          if (kRow) {
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[16 * c + j] = fmaf(__int2float_rn((int)d[j]), swv, acc[16 * c + j]);
          } else {
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              const float4 s4 = *reinterpret_cast<const float4*>(sag + 16 * c + j);
              acc[16 * c + j] = fmaf(__int2float_rn((int)d[j]) * swv, s4.x, acc[16 * c + j]);
              acc[16 * c + j + 1] = fmaf(__int2float_rn((int)d[j + 1]) * swv, s4.y, acc[16 * c + j + 1]);
              acc[16 * c + j + 2] = fmaf(__int2float_rn((int)d[j + 2]) * swv, s4.z, acc[16 * c + j + 2]);
              acc[16 * c + j + 3] = fmaf(__int2float_rn((int)d[j + 3]) * swv, s4.w, acc[16 * c + j + 3]);
            }
          }
        }
      }
      if (!ok) break;
      if (kRow) {
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (t < T) acc[t] *= __ldg(scales_A + t);
      }
      if (n < N) {
        // Token t of row n: consecutive threads write consecutive channels.
        if (ranges > 1) {
          float* dst = ws + (int64_t)w.kr * T * N + n;
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < T) dst[(int64_t)t * N] = acc[t];
        } else if (out_bf16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(Y) + n;
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < T) dst[(int64_t)t * N] = __float2bfloat16_rn(acc[t]);
        } else {
          float* dst = reinterpret_cast<float*>(Y) + n;
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < T) dst[(int64_t)t * N] = acc[t];
        }
      }
    }
    ptx::cp_async_wait_all();   // no copy may land after the CTA has left (abort path)
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int NT, bool kRow, int GSL>
pq_status launch_small(const CUtensorMap& tmW, const CUtensorMap& tmA, const float* scales_A, const float* scales_W,
                       void* Y, float* ws, int T, int N, int G, int ranges, int gs, int units, int out_bf16,
                       bool pdl, unsigned int* status, cudaStream_t stream) {
  static std::atomic<bool> attr_done[kMaxDevices];
  cudaError_t e = set_kernel_attributes(reinterpret_cast<const void*>(w4a4_gemm_small_kernel<NT, kRow, GSL>),
                                        (int)small_smem_bytes<NT>(), attr_done);
  if (e != cudaSuccess) return cuda_fail(e, "w4a4_gemm_small_kernel attributes");
  // The warpgroups' setmaxnreg shares are drawn from the launch allocation (compiled registers x
  // threads); a smaller allocation would leave the epilogue's increase waiting for ever.
  static std::atomic<int> regs_cache{-1};
  int regs = regs_cache.load(std::memory_order_relaxed);
  if (regs < 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, w4a4_gemm_small_kernel<NT, kRow, GSL>);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(w4a4_gemm_small_kernel)");
    regs = fa.numRegs;
    regs_cache.store(regs, std::memory_order_relaxed);
  }
  if ((uint32_t)regs * GS_THREADS < kGsRegBudget) {
    set_error("w4a4_gemm_small_kernel compiled with %d registers per thread: %u needed for its register split",
              regs, (kGsRegBudget + GS_THREADS - 1) / GS_THREADS);
    return PQ_ERR_CUDA;
  }
  const int grid = std::min(units, device_sm_count());
  if (!pdl) {
    w4a4_gemm_small_kernel<NT, kRow, GSL><<<grid, GS_THREADS, small_smem_bytes<NT>(), stream>>>(
        tmW, tmA, scales_A, scales_W, Y, ws, T, N, G, ranges, gs, units, out_bf16, 0, status);
    return cuda_fail(cudaGetLastError(), "w4a4_gemm_small_kernel launch");
  }
  // Programmatic dependent of the preceding kernel on `stream` (the activation transform).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(GS_THREADS, 1, 1);
  cfg.dynamicSmemBytes = small_smem_bytes<NT>();
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cuda_fail(cudaLaunchKernelEx(&cfg, w4a4_gemm_small_kernel<NT, kRow, GSL>, tmW, tmA, scales_A, scales_W, Y, ws, T,
                                      N, G, ranges, gs, units, out_bf16, 1, status),
                   "w4a4_gemm_small_kernel launch (programmatic dependent)");
}

static_assert(small_smem_bytes<16>() <= 232448 && small_smem_bytes<32>() <= 232448 &&
                  small_smem_bytes<64>() <= 232448 && small_smem_bytes<128>() <= 232448,
              "shared memory exceeds 227 KB");

}  // namespace

// Group ranges per 128-row weight tile: as many as keep every unit in one wave over the SMs (a
// second, partial wave would double the time of the CTAs that run it), and only while the
// float32 partial tiles of the ranges (written and read back, 8 T N bytes per range, mostly in
// L2) stay within the packed weight bytes (N D / 2).  A range is a multiple of 4 groups.
int gemm_small_ranges(int64_t T, int64_t N, int64_t D, int g, int* gs_out) {
  const int G = (int)(D / g);
  if (T <= kGemvT) {            // the CUDA-core kernel: one launch over all groups
    if (gs_out) *gs_out = G;
    return 1;
  }
  const int64_t m_tiles = (N + GS_M - 1) / GS_M;
  const int64_t fill = device_sm_count() / m_tiles;
  const int64_t traffic = std::max<int64_t>(1, D / (16 * T));
  int r = (int)std::max<int64_t>(1, std::min<int64_t>({fill, traffic, (int64_t)((G + GS_GPS - 1) / GS_GPS)}));
  int gs = (G + r - 1) / r;
  gs = (gs + GS_GPS - 1) / GS_GPS * GS_GPS;
  r = (G + gs - 1) / gs;
  if (r == 1) gs = G;
  if (gs_out) *gs_out = gs;
  return r;
}

pq_status gemm_small_launch(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W,
                            const float* scales_W, int64_t T, int64_t N, int64_t D, int g, void* Y,
                            pq_out_dtype out_dtype, float* ws, unsigned int* status, cudaStream_t stream,
                            bool row_scale, bool pdl) {
  if (T <= kGemvT)
    return gemv_launch(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype, stream, row_scale, pdl);
  const int NT = T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : 128;
  const int G = (int)(D / g), gsl = g / 32;
  int gs = G;
  const int ranges = ws ? gemm_small_ranges(T, N, D, g, &gs) : 1;
  if (ranges == 1) gs = G;
  const int64_t m_tiles = (N + GS_M - 1) / GS_M;
  const int64_t units = m_tiles * ranges;
  if (units >= ((int64_t)1 << 31)) {
    set_error("too many work units");
    return PQ_ERR_INVALID_ARG;
  }
  // Packed codes, [rows][D/2] bytes: boxes of two groups (128 bytes) x 128 weight rows or NT
  // token rows, 128-byte swizzle; token rows past T and bytes past a row read as zeros.
  CUtensorMap tmW, tmA;
  cudaError_t e = make_u8_tile_map(&tmW, codes_W, N, D / 2, 128, GS_M, true);
  if (e != cudaSuccess) return cuda_fail(e, "tensor map (packed weights)");
  e = make_u8_tile_map(&tmA, codes_A, T, D / 2, 128, NT, true);
  if (e != cudaSuccess) return cuda_fail(e, "tensor map (packed activations)");
  const int bf16 = out_dtype == PQ_OUT_BF16 ? 1 : 0;
  pq_status st;
#define PQ_SMALL_CASE3(W, GSL)                                                                                  \
  st = row_scale ? launch_small<W, true, GSL>(tmW, tmA, scales_A, scales_W, Y, ws, (int)T, (int)N, G, ranges, gs, \
                                              (int)units, bf16, pdl, status, stream)                              \
                 : launch_small<W, false, GSL>(tmW, tmA, scales_A, scales_W, Y, ws, (int)T, (int)N, G, ranges, gs, \
                                               (int)units, bf16, pdl, status, stream)
#define PQ_SMALL_CASE(W)                          \
  if (gsl == 2) PQ_SMALL_CASE3(W, 2);             \
  else if (gsl == 8) PQ_SMALL_CASE3(W, 8);        \
  else PQ_SMALL_CASE3(W, 4)
  switch (NT) {
    case 16: PQ_SMALL_CASE(16); break;
    case 32: PQ_SMALL_CASE(32); break;
    case 64: PQ_SMALL_CASE(64); break;
    default: PQ_SMALL_CASE(128); break;
  }
#undef PQ_SMALL_CASE3
#undef PQ_SMALL_CASE
  if (st != PQ_OK || ranges == 1) return st;
  return launch_splitk_reduce(ws, ranges, T, N, Y, bf16, stream);
}

}  // namespace pq
