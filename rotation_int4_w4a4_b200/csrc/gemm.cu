// W4A4 GEMM with per-group scales on tcgen05 tensor cores (sm_100a).
//
// Y[t][n] = sum_G sa[t][G] * sw[n][G] * d_G[t][n],  d_G = sum_{k in group G} qa[t][k] qw[n][k]
// (RRS page, main equation, last line; Fig. 4 step (3): the GEMM's K-block equals the
// quantisation group and the block's scales are applied to the interim integer result).
//
// Two kernels per call, ordered on the caller's stream:
//
// 1. expand_codes_kernel: int4 codes -> E4M3 bytes for A and W into stream-ordered scratch.
//    Every code in -8..7 is exact in E4M3, so the MMA's products and group sums (integers of
//    magnitude <= 128 * 64 = 2^13) are exact in its float32 accumulator: d_G arrives in tensor
//    memory as an exact float.  Within each 128-element group the low nibbles of the 64 packed
//    bytes become K positions 0..63 and the high nibbles 64..127 (the same permutation on A and
//    W, so every dot product is unchanged).  One TMA box of 128 bytes x rows then lands directly
//    in the 128-byte-swizzled K-major operand layout.  (Unpacking inside the contraction kernel
//    costs a shared-memory read and a double-size write per operand byte, and tensor-core operand
//    reads take priority over that traffic on the shared-memory banks.)
//
// 2. w4a4_gemm_kernel: persistent, one CTA per SM, launched as clusters of two CTAs (a CTA
//    pair on one SM pair) that share every MMA (tcgen05 cta_group::2).  A pair's tile is
//    256 output channels x 256 tokens: the even CTA's MMA (M = 256, N = 256) reads weight rows
//    0..127 and tokens 0..127 from its own shared memory and weight rows 128..255 and tokens
//    128..255 from its peer's, and each CTA's tensor memory receives its own 128 channels x
//    256 tokens (D[n][t], channels = TMEM lanes).  Each SM thus loads 32 KB of operands per
//    group instead of the 48 KB a single CTA needs for 128 x 256, for the same tensor-core
//    work.  The K loop runs one 128-wide group per step.  Warp roles (12 warps per CTA):
//      warp 0      TMA producer: this CTA's 128 weight rows and 128 tokens per group into a
//                  6-stage ring; the bytes of both CTAs complete on the even CTA's barrier.
//      warp 1      TMEM allocator (both CTAs) and, in the even CTA only, the MMA issuer:
//                  4 x tcgen05.mma.cta_group::2 kind::f8f6f4 (M256 N256 K32) per group into a
//                  double-buffered float32 accumulator (the first of the four overwrites the
//                  buffer); one multicast commit frees both CTAs' stage, another tells both
//                  epilogues the group is done.
//      warps 2..3  scale loaders: the CTA's weight scales and the tile's activation scales for
//                  4 groups at a time (cp.async, zero-filled past N / T / G) into a 4-stage ring.
//      warps 4..11 epilogue: 2 warps per TMEM lane quarter, 128 tokens each.  Tensor memory is
//                  read with the 16x256b shape, so each thread holds 4 output channels x 32
//                  tokens: per group it needs 4 weight scales and 32 token scales (a quarter of
//                  the shared-memory traffic of one channel x 128 tokens per thread).  Per element
//                  acc += fl(d * sw) * sa in float32 registers, groups in ascending order, with
//                  one packed multiply and one packed FMA per element pair; each warp hands its
//                  part of the buffer back to the even CTA's MMA issuer; after the last group
//                  the tile is stored to Y.
//    Every mbarrier wait is bounded; a timeout sets a status bit, the CTA drains its own copies
//    and MMAs, meets its peer (bounded), frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace pq {

__device__ unsigned int g_gemm_status = 0;

namespace {

constexpr int BM = 128;          // output channels (weight rows) per CTA = its TMEM lanes
constexpr int PAIR_M = 2 * BM;   // a CTA pair's MMA has M = 256 (128 rows in each CTA)
constexpr int BN = 256;          // tile columns = tokens (activation rows), MMA N
constexpr int BN_HALF = BN / 2;  // tokens staged by each CTA of the pair
constexpr int BK = 128;          // one quantisation group = 128 bytes = one 128-byte swizzle row
constexpr int OP_STAGES = 6;     // operand ring
constexpr int SC_GROUPS = 4;     // groups per scale stage
constexpr int S_STAGES = 4;      // scale ring
constexpr int NUM_EPI_WARPS = 8;   // 2 per TMEM lane quarter
constexpr int EPI_WARP0 = 4;       // warps 0..3 control, then the epilogue
constexpr int NUM_THREADS = 32 * (EPI_WARP0 + NUM_EPI_WARPS);
constexpr int EPI_COLS = BN / (NUM_EPI_WARPS / 4);   // tokens per epilogue warp: 128
constexpr int EPI_CHUNKS = EPI_COLS / 16;            // 16-token chunks of the accumulator layout
// Tokens per tensor-memory wait (per lane half).  16 (one 16x256b.x2 load per lane half) was
// measured faster than 32 or than overlapping the next chunk's load with this chunk's math.
constexpr int EPI_LDC = 16;
constexpr int EPI_NX = EPI_LDC / 8;                  // 16x256b repetitions per load
constexpr int NUM_SCALE_THREADS = 64;                // warps 2 and 3
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;     // 2 s
constexpr uint32_t kTxBytes = 2 * (BM + BN_HALF) * BK;   // both CTAs' tiles, on the even CTA's barrier
// Register budget (setmaxnreg): launch allocation per thread and the control and epilogue
// warps' shares; 128 * REG_CTRL + 32 * NUM_EPI_WARPS * REG_EPI must not exceed
// NUM_THREADS * REG_LAUNCH.
constexpr uint32_t REG_LAUNCH = 168;
constexpr uint32_t REG_CTRL = 56;
constexpr uint32_t REG_EPI = 224;
static_assert(REG_CTRL * 32 * EPI_WARP0 + REG_EPI * 32 * NUM_EPI_WARPS <= REG_LAUNCH * NUM_THREADS,
              "setmaxnreg shares exceed the launch allocation");
static_assert(REG_LAUNCH * NUM_THREADS <= 65536, "launch register allocation exceeds the SM");

struct __align__(1024) GemmSmem {
  uint8_t opA[OP_STAGES][BM * BK];          // this CTA's 128 weight rows, 16 KB per stage, 128-byte swizzle
  uint8_t opB[OP_STAGES][BN_HALF * BK];     // this CTA's 128 of the tile's 256 tokens, 16 KB per stage
  float sc_w[S_STAGES][BM][SC_GROUPS];      // weight scales: [tile row][group of the stage]
  float sc_a[S_STAGES][BN][SC_GROUPS];      // activation scales: [tile token][group]
  uint64_t op_full[OP_STAGES];
  uint64_t op_empty[OP_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t sc_full[S_STAGES];
  uint64_t sc_empty[S_STAGES];
  uint64_t mma_done;
  uint64_t pair_done;
  uint32_t tmem_slot;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(GemmSmem) + 1024;   // + slack for 1024-byte alignment
static_assert(kSmemBytes <= 232448, "shared memory exceeds 227 KB");

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
// Four codes (one per byte of x, each 0..15 as two's-complement nibbles) -> four E4M3 bytes.
// Byte permutes look the magnitudes up in two 8-entry tables (codes 0..7 and -8..-1); bit 3 of
// each code selects between them.
__device__ __forceinline__ uint32_t codes_to_e4m3(uint32_t x) {
  constexpr uint32_t kPos0 = 0x44403800u, kPos1 = 0x4E4C4A48u;   // 0, 1, 2, 3 | 4, 5, 6, 7
  constexpr uint32_t kNeg0 = 0xCACCCED0u, kNeg1 = 0xB8C0C4C8u;   // -8, -7, -6, -5 | -4, -3, -2, -1
  const uint32_t idx = x & 0x07070707u;
  const uint32_t t = idx | (idx >> 4);
  const uint32_t sel = (t & 0xFFu) | ((t >> 8) & 0xFF00u);     // four 3-bit indices as nibbles
  const uint32_t pos = __byte_perm(kPos0, kPos1, sel);
  const uint32_t neg = __byte_perm(kNeg0, kNeg1, sel);
  const uint32_t m = ((x >> 3) & 0x01010101u) * 0xFFu;
  return (pos & ~m) | (neg & m);
}

// One thread per 16 packed bytes (32 codes): K-block kb (128 codes, 64 packed bytes) holds the
// chunk's 16 low-nibble codes and 16 high-nibble codes.  g >= 128: at K offsets 16p and 64 + 16p
// of the block (the permutation stays inside each 128-code block, so inside each group);
// g = 64: inside each 64-code half h = p / 2, at 64 h + 16 (p % 2) and 64 h + 32 + 16 (p % 2).
__global__ void __launch_bounds__(256) expand_codes_kernel(const uint8_t* __restrict__ A, int64_t chunksA,
                                                           const uint8_t* __restrict__ W, int64_t chunksW,
                                                           uint8_t* __restrict__ A8, uint8_t* __restrict__ W8,
                                                           int g64) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunksA + chunksW; i += stride) {
    const bool isA = i < chunksA;
    const int64_t c = isA ? i : i - chunksA;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(isA ? A : W) + c);
    const int64_t kb = c >> 2;             // 4 chunks of 16 bytes per 64-byte packed K-block
    const int p = (int)(c & 3);
    const int lo = g64 ? 64 * (p >> 1) + 16 * (p & 1) : 16 * p;
    const int hi = lo + (g64 ? 32 : 64);
    uint8_t* base = (isA ? A8 : W8) + kb * 128;
    *reinterpret_cast<uint4*>(base + lo) =
        make_uint4(codes_to_e4m3(w.x & 0x0F0F0F0Fu), codes_to_e4m3(w.y & 0x0F0F0F0Fu),
                   codes_to_e4m3(w.z & 0x0F0F0F0Fu), codes_to_e4m3(w.w & 0x0F0F0F0Fu));
    *reinterpret_cast<uint4*>(base + hi) =
        make_uint4(codes_to_e4m3((w.x >> 4) & 0x0F0F0F0Fu), codes_to_e4m3((w.y >> 4) & 0x0F0F0F0Fu),
                   codes_to_e4m3((w.z >> 4) & 0x0F0F0F0Fu), codes_to_e4m3((w.w >> 4) & 0x0F0F0F0Fu));
  }
}

// Tile order: weight tiles fastest, so the CTA pairs running at the same time share a token
// tile.  A tile is PAIR_M weight rows x BN tokens, computed by one CTA pair; m0 is the pair's
// first row.  (Token-fastest and banded orders were measured no faster.)
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int& m0, int& n0) {
  (void)n_tiles;
  m0 = (tile % m_tiles) * PAIR_M;
  n0 = (tile / m_tiles) * BN;
}

// Work units: an output tile and a range of groups.  With split-K (ksplit > 1) the groups of a
// tile are divided into ranges of gs (a multiple of SC_GROUPS) and each unit writes a float32
// partial tile; a reduction kernel then sums the ranges in ascending order.
struct Work {
  int m_tiles, n_tiles, num_tiles;
  int ksplit, gs, G;
  int units;
  int first, stride;     // this CTA pair's first unit and the number of pairs in the grid
  int rank;              // 0 = even CTA (issues the pair's MMAs), 1 = odd CTA
};

__device__ __forceinline__ void unit_coords(int u, const Work& wk, int& m0, int& n0, int& kr, int& k0, int& k1) {
  const int tile = u / wk.ksplit;
  kr = u - tile * wk.ksplit;
  tile_coords(tile, wk.m_tiles, wk.n_tiles, m0, n0);
  k0 = kr * wk.gs;
  k1 = min(wk.G, k0 + wk.gs);
}

// -------------------------------------------------------------------------- control
// kRow: scales_W holds per-(row, group) factors and scales_A one scale per token (applied in the
// epilogue after the groups), so the loaders fetch only the weight rows' factors.
template <bool kRow, int GSL>
__device__ __forceinline__ void cta_control(GemmSmem& S, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                            const float* __restrict__ scales_A, const float* __restrict__ scales_W,
                                            uint32_t tmem, int T, int N, int G, int scales_vec16, const Work& wk,
                                            unsigned int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // Both CTAs of the pair load their own halves (weight rows m0 + 128 rank, tokens
    // n0 + 128 rank); all bytes complete on the even CTA's full barrier, whose MMA reads both.
    if (lane == 0) {
      const uint32_t full0 = ptx::mapa_shared(ptx::smem_addr(&S.op_full[0]), 0);
      int step = 0;
      bool ok = true;
      for (int u = wk.first; u < wk.units && ok; u += wk.stride) {
        int m0, n0, kr, k0, k1;
        unit_coords(u, wk, m0, n0, kr, k0, k1);
        // the unit's K-blocks (its groups start on a K-block boundary: ranges are 4 groups)
        const int kb0 = k0 * GSL / 4, kb1 = k1 * GSL / 4;
        for (int kb = kb0; kb < kb1; ++kb, ++step) {
          const int s = step % OP_STAGES;
          const uint32_t ph = (uint32_t)(step / OP_STAGES) & 1u;
          if (!wait_or_abort(S, &S.op_empty[s], ph ^ 1u, status)) { ok = false; break; }
          if (wk.rank == 0) ptx::mbar_arrive_expect_tx(&S.op_full[s], kTxBytes);
          ptx::tma_load_2d_pair(S.opA[s], &tmA, full0 + 8u * s, kb * BK, m0 + BM * wk.rank);
          ptx::tma_load_2d_pair(S.opB[s], &tmB, full0 + 8u * s, kb * BK, n0 + BN_HALF * wk.rank);
        }
      }
      // Drain: every stage's last use is released by the pair's MMAs (so every load issued has
      // landed and every release aimed at this CTA has arrived) before the CTA may exit.
      if (wk.rank == 0)
        for (int j = (step > OP_STAGES ? step - OP_STAGES : 0); j < step; ++j)
          drain_wait(&S.op_full[j % OP_STAGES], (uint32_t)(j / OP_STAGES) & 1u);
      for (int j = (step > OP_STAGES ? step - OP_STAGES : 0); j < step; ++j)
        drain_wait(&S.op_empty[j % OP_STAGES], (uint32_t)(j / OP_STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA issuer
    // The even CTA issues M256 x N256 pair MMAs: its tensor memory receives weight rows
    // m0 .. m0 + 127, the odd CTA's rows m0 + 128 ..; both CTAs' stages and accumulator buffers
    // are released by one multicast commit.
    if (lane == 0 && wk.rank == 0) {
      constexpr uint32_t idesc = ptx::idesc_e4m3_f32(PAIR_M, BN);
      int step = 0;    // groups
      int kstep = 0;   // K-blocks (operand stages) consumed
      bool ok = true;
      for (int u = wk.first; u < wk.units && ok; u += wk.stride) {
        int m0, n0, kr, k0, k1;
        unit_coords(u, wk, m0, n0, kr, k0, k1);
        for (int kg = k0; kg < k1 && ok; ++kg, ++step) {
          const int b = step & 1;
          const uint32_t u = (uint32_t)(step >> 1);
          // the first use of each buffer passes at once (parity of the phase before the first)
          if (!wait_or_abort(S, &S.acc_empty[b], (u & 1u) ^ 1u, status)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t d = tmem + (uint32_t)b * BN;
          // The group's GSL K32 slices (compile-time, so the MMAs issue back to back): a K-block's
          // stage is awaited at its first slice and released after its fourth; slice 0 of the
          // group overwrites the buffer.  GSL = 2: the group is the first or second half of a
          // K-block (by its parity within the unit).
          const int h = GSL == 2 ? ((kg - k0) & 1) : 0;
#pragma unroll
          for (int sl = 0; sl < GSL; ++sl) {
            const int sub = GSL == 2 ? 2 * h + sl : (sl & 3);
            const int s = kstep % OP_STAGES;
            if (sub == 0) {
              if (!wait_or_abort(S, &S.op_full[s], (uint32_t)(kstep / OP_STAGES) & 1u, status)) { ok = false; break; }
              ptx::tc_fence_after();
            }
            const uint32_t a0 = ptx::smem_addr(S.opA[s]);
            const uint32_t b0 = ptx::smem_addr(S.opB[s]);
            ptx::umma_e4m3_pair(d, ptx::smem_desc_sw128(a0 + 32 * sub), ptx::smem_desc_sw128(b0 + 32 * sub), idesc,
                                sl > 0 ? 1u : 0u);
            if (sub == 3) {
              ptx::umma_commit_pair(&S.op_empty[s], 0x3);
              ++kstep;
            }
          }
          if (!ok) break;
          ptx::umma_commit_pair(&S.acc_full[b], 0x3);
        }
      }
      ptx::umma_commit_pair(&S.mma_done, 0x1);
      drain_wait(&S.mma_done, 0);
      // Both CTAs' epilogues release the last two buffers here before this CTA may exit.
      for (int j = (step > 2 ? step - 2 : 0); j < step; ++j)
        drain_wait(&S.acc_empty[j & 1], (uint32_t)(j >> 1) & 1u);
    }
  } else {
    // ---------------------------------------------------------------- scale loaders
    // Per stage: SC_GROUPS consecutive groups of the tile's 128 weight rows and 256 tokens.
    const int j = threadIdx.x - 64;                      // 0..63
    int cs = 0;                                          // scale stages filled so far
    bool ok = true;
    for (int u = wk.first; u < wk.units && ok; u += wk.stride) {
      int m0, n0, kr, k0, k1;
      unit_coords(u, wk, m0, n0, kr, k0, k1);
      for (int kg0 = k0; kg0 < k1; kg0 += SC_GROUPS, ++cs) {
        const int st = cs % S_STAGES;
        const uint32_t sph = (uint32_t)(cs / S_STAGES) & 1u;
        if (!warp_wait_or_abort(S, &S.sc_empty[st], sph ^ 1u, status)) { ok = false; break; }
#pragma unroll
        for (int i = 0; i < (BM + BN) / NUM_SCALE_THREADS; ++i) {
          const int r = j + NUM_SCALE_THREADS * i;       // 0..127 weight rows, 128..383 tokens
          const bool isw = r < BM;
          if (kRow && !isw) continue;                    // token scales are not per group
          const int row = isw ? m0 + BM * wk.rank + r : n0 + (r - BM);
          const bool in = row < (isw ? N : T);
          const float* src = (isw ? scales_W : scales_A) + (int64_t)(in ? row : 0) * G + kg0;
          float* dst = isw ? S.sc_w[st][r] : S.sc_a[st][r - BM];
          if (scales_vec16) {
            ptx::cp_async16(dst, src, in ? 16u : 0u);    // G % 4 == 0: 16-byte aligned rows
          } else {
#pragma unroll
            for (int e = 0; e < SC_GROUPS; ++e)
              ptx::cp_async4(dst + e, in && kg0 + e < k1 ? src + e : src - kg0, in && kg0 + e < k1 ? 4u : 0u);
          }
        }
        ptx::cp_async_arrive_noinc(&S.sc_full[st]);
      }
    }
    ptx::cp_async_wait_all();
  }
}

// ------------------------------------------------------------------------- epilogue
// Thread layout (16x256b loads): in warp ew, TMEM lane quarter sub = warp % 4 (rows 32 sub ..),
// token half ch = ew / 4 (tokens 128 ch ..); lane L has g = L / 4, q = L % 4.  Its rows are
// 32 sub + 16 h + g + 8 k and its tokens 128 ch + 16 c + 8 x + 2 q + e (h, k, x, e in {0, 1},
// c in 0..7).  acc index: ((h * 2 + k) * 8 + c) * 4 + x * 2 + e.
// kRow: per group acc += d * F (one packed FMA per element pair, F the row's factor for the
// group), and each token's scale from token_scales multiplies the sum before it is stored.
template <bool kRow>
__device__ __forceinline__ void cta_epilogue(GemmSmem& S, uint32_t tmem, void* __restrict__ Y, int T, int N,
                                             int G, int out_bf16, const Work& wk, float* __restrict__ ws,
                                             const float* __restrict__ token_scales, unsigned int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ew = warp - EPI_WARP0;
  const int sub = warp & 3;          // TMEM lane quarter this warp may access
  const int ch = ew >> 2;            // token half of the tile
  const int g = lane >> 2, q = lane & 3;
  // Accumulator buffers are handed back to the even CTA, whose thread issues the pair's MMAs.
  const uint32_t acc_empty0 = ptx::mapa_shared(ptx::smem_addr(&S.acc_empty[0]), 0);
  int step = 0, cs = 0;
  bool ok = true;
  for (int u = wk.first; u < wk.units && ok; u += wk.stride) {
    int m0, n0, kr, k0, k1;
    unit_coords(u, wk, m0, n0, kr, k0, k1);
    constexpr int kAcc2 = 4 * EPI_CHUNKS * 2;         // rows (h, k) x chunks x x; e is the pair
    static_assert(2 * kAcc2 == EPI_COLS, "4 channels x EPI_COLS / 4 tokens per thread");
    uint64_t acc2[kAcc2];                            // float32 pairs (tokens 2q, 2q + 1)
#pragma unroll
    for (int i = 0; i < kAcc2; ++i) acc2[i] = 0ull;
    for (int kg = k0; kg < k1; ++kg, ++step) {
      const int b = step & 1;
      const uint32_t u = (uint32_t)(step >> 1);
      const int st = cs % S_STAGES;
      const int gi = (kg - k0) % SC_GROUPS;
      if (gi == 0 && !warp_wait_or_abort(S, &S.sc_full[st], (uint32_t)(cs / S_STAGES) & 1u, status)) {
        ok = false;
        break;
      }
      // This step's scales: one shared-memory base address each, every offset a constant.
      const uint32_t swb = ptx::smem_addr(&S.sc_w[st][32 * sub + g][gi]);
      const uint32_t sab = ptx::smem_addr(&S.sc_a[st][ch * EPI_COLS + 2 * q][gi]);
      uint64_t sw2[4];                               // weight scale of row (h, k), twice
#pragma unroll
      for (int hk = 0; hk < 4; ++hk) {
        const float sw = ptx::lds_f32(swb + 4 * SC_GROUPS * (16 * (hk >> 1) + 8 * (hk & 1)));
        sw2[hk] = ptx::f2_pack(sw, sw);
      }
      if (!warp_wait_or_abort(S, &S.acc_full[b], u & 1u, status)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(32 * sub) << 16) + (uint32_t)(b * BN + ch * EPI_COLS);
      // EPI_LDC tokens x both lane halves per TMEM wait.
#pragma unroll
      for (int cc = 0; cc < EPI_COLS / EPI_LDC; ++cc) {
        uint32_t d0[4 * EPI_NX], d1[4 * EPI_NX];     // lane halves h = 0, 1
        ptx::tmem_ld_16x256b<EPI_NX>(tbase + EPI_LDC * cc, d0);
        ptx::tmem_ld_16x256b<EPI_NX>(tbase + (16u << 16) + EPI_LDC * cc, d1);
        uint64_t sa2[EPI_NX];                        // token scales of columns LDC cc + 8x + 2q + {0, 1}
        if (!kRow) {
#pragma unroll
          for (int x = 0; x < EPI_NX; ++x)
            sa2[x] = ptx::lds_pair<4 * SC_GROUPS>(sab + 4 * SC_GROUPS * (EPI_LDC * cc + 8 * x));
        }
        const uint32_t after = ptx::tmem_ld_wait_token();
        if (cc == EPI_COLS / EPI_LDC - 1) {
          // The whole group's tile is read: hand the buffer back to the MMA before the math.
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive_remote(acc_empty0 + 8u * b);
        }
#pragma unroll
        for (int x = 0; x < EPI_NX; ++x)
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int xx = (EPI_LDC / 8) * cc + x;          // 8-token block of the warp's 128
            const int c = xx >> 1;                          // 16-token chunk of the accumulator layout
            const int i0 = ((0 * 2 + k) * EPI_CHUNKS + c) * 2 + (xx & 1);
            const int i1 = ((1 * 2 + k) * EPI_CHUNKS + c) * 2 + (xx & 1);
            if (kRow) {
              ptx::fma2(acc2[i0], d0[4 * x + 2 * k], d0[4 * x + 2 * k + 1], sw2[0 * 2 + k], after);
              ptx::fma2(acc2[i1], d1[4 * x + 2 * k], d1[4 * x + 2 * k + 1], sw2[1 * 2 + k], after);
            } else {
              ptx::mul_fma2(acc2[i0], d0[4 * x + 2 * k], d0[4 * x + 2 * k + 1], sw2[0 * 2 + k], sa2[x], after);
              ptx::mul_fma2(acc2[i1], d1[4 * x + 2 * k], d1[4 * x + 2 * k + 1], sw2[1 * 2 + k], sa2[x], after);
            }
          }
      }
      if (gi == SC_GROUPS - 1 || kg == k1 - 1) {
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.sc_empty[st]);
        ++cs;
      }
    }
    if (!ok) break;
    // Y[t][n]: per store, 8 lanes (same q) write 8 consecutive channels of one token.  The
    // thread's channels are nb + {0, 8, 16, 24}, its tokens tb + 16 c + 8 x + e.
    const int nb = m0 + BM * wk.rank + 32 * sub + g;
    const int tb = n0 + ch * EPI_COLS + 2 * q;
    bool nin[4];
#pragma unroll
    for (int hk = 0; hk < 4; ++hk) nin[hk] = nb + 8 * hk < N;
    // Split-K: this unit's float32 partial tile goes to ws[kr]; the reduction writes Y.
    const bool partial = wk.ksplit > 1;
    const int bf16_out = partial ? 0 : out_bf16;
    void* dstY = partial ? static_cast<void*>(ws + (int64_t)kr * T * N) : Y;
    const size_t esz = bf16_out ? 2 : 4;
    char* row = reinterpret_cast<char*>(dstY) + ((int64_t)tb * N + nb) * esz;
    const int64_t row_step = (int64_t)N * esz;
#pragma unroll
    for (int c = 0; c < EPI_CHUNKS; ++c) {
#pragma unroll
      for (int xe = 0; xe < 4; ++xe) {
        const int dt = 8 * (xe >> 1) + (xe & 1);
        if (tb + 16 * c + dt < T) {
          char* p = row + dt * row_step;
          const float ts = kRow ? __ldg(token_scales + tb + 16 * c + dt) : 1.0f;
#pragma unroll
          for (int hk = 0; hk < 4; ++hk) {
            if (!nin[hk]) continue;
            float lo, hi;                                            // rows 16 h + 8 k = 8 hk
            ptx::unpack2(acc2[(hk * EPI_CHUNKS + c) * 2 + (xe >> 1)], lo, hi);
            const float v = kRow ? ((xe & 1) ? hi : lo) * ts : ((xe & 1) ? hi : lo);
            if (!bf16_out) reinterpret_cast<float*>(p)[8 * hk] = v;
            else reinterpret_cast<__nv_bfloat16*>(p)[8 * hk] = __float2bfloat16_rn(v);
          }
        }
      }
      row += 16 * row_step;
    }
  }
}

// GSL: K32 tensor-core slices per group (g / 32 = 2, 4 or 8; a 128-code K-block holds 4).
template <bool kRow, int GSL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1) w4a4_gemm_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const float* __restrict__ scales_A, const float* __restrict__ scales_W, void* __restrict__ Y,
    int T, int N, int G, int scales_vec16, int out_bf16, int m_tiles, int n_tiles, int ksplit, int gs,
    float* __restrict__ ws, unsigned int* status) {
  extern __shared__ unsigned char smem_raw[];
  GemmSmem& S = *reinterpret_cast<GemmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The split-K reduction, launched as this grid's programmatic dependent, may start now (it
  // waits for this grid before reading).
  ptx::griddep_launch_dependents();
  Work wk;
  wk.m_tiles = m_tiles;
  wk.n_tiles = n_tiles;
  wk.num_tiles = m_tiles * n_tiles;
  wk.ksplit = ksplit;
  wk.gs = gs;
  wk.G = G;
  wk.units = wk.num_tiles * ksplit;
  wk.rank = (int)ptx::cluster_ctarank();
  wk.first = (int)(blockIdx.x >> 1);
  wk.stride = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < OP_STAGES; ++s) {
      ptx::mbar_init(&S.op_full[s], 1);
      ptx::mbar_init(&S.op_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&S.acc_full[b], 1);
      ptx::mbar_init(&S.acc_empty[b], 2 * NUM_EPI_WARPS);   // both CTAs' epilogue warps
    }
    for (int s = 0; s < S_STAGES; ++s) {
      ptx::mbar_init(&S.sc_full[s], NUM_SCALE_THREADS);
      ptx::mbar_init(&S.sc_empty[s], NUM_EPI_WARPS);
    }
    ptx::mbar_init(&S.mma_done, 1);
    ptx::mbar_init(&S.pair_done, 1);
    S.abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&S.tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();   // both CTAs' barriers initialised and tensor memory allocated
  ptx::tc_fence_after();
  const uint32_t tmem = S.tmem_slot;

  if (warp < EPI_WARP0) {
    ptx::setmaxnreg_dec<REG_CTRL>();
    cta_control<kRow, GSL>(S, tmA, tmB, scales_A, scales_W, tmem, T, N, G, scales_vec16, wk, status);
  } else {
    ptx::setmaxnreg_inc<REG_EPI>();
    cta_epilogue<kRow>(S, tmem, Y, T, N, G, out_bf16, wk, ws, scales_A, status);
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  // Neither CTA leaves while its peer may still arrive on its barriers or read its tiles.
  if (threadIdx.x == 0) {
    ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_addr(&S.pair_done), (uint32_t)wk.rank ^ 1u));
    int never = 0;
    if (!ptx::mbar_wait_bounded_cl(&S.pair_done, 0, &never, kWaitLimitNs)) atomicOr(status, PQ_DEV_TIMEOUT);
  }
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// Split-K reduction: Y = sum over kr of ws[kr] (ascending), float32 or bf16 (RNE) out.
// Launched as the programmatic dependent of the kernel that writes the partial tiles: it may start
// while that kernel runs and waits for its completion before reading them.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float4* __restrict__ ws, int ksplit, int64_t n4,
                                                            void* __restrict__ Y, int out_bf16) {
  ptx::griddep_wait();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = ws[i];
    for (int kr = 1; kr < ksplit; ++kr) {
      const float4 b = ws[(int64_t)kr * n4 + i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    if (!out_bf16) {
      reinterpret_cast<float4*>(Y)[i] = a;
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
      reinterpret_cast<uint2*>(Y)[i] =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
  }
}

// Diagnostic: one thread waits on an mbarrier that never completes, with the same bounded
// wait every pipeline barrier above uses; when it gives up it sets the GEMM status word.
__global__ void wait_timeout_kernel(uint64_t limit_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  __shared__ int never;
  if (threadIdx.x != 0) return;
  never = 0;
  ptx::mbar_init(&bar, 1);
  ptx::fence_mbar_init();
  if (!ptx::mbar_wait_bounded(&bar, 0, &never, limit_ns)) atomicOr(status, PQ_DEV_TIMEOUT);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> cache{nullptr};
  EncodeTiledFn fn = cache.load(std::memory_order_acquire);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
      cache.store(fn, std::memory_order_release);
    }
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
  static cudaMemPool_t pools[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
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

// CTA pairs (clusters of 2) of w4a4_gemm_kernel resident at once on the current device: one
// per SM pair when every pair can host one.
pq_status gemm_max_pairs(int sms, int* out) {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const bool slot = dev >= 0 && dev < kMaxDevices;
  int n = slot ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (n < 1) {
    // Every instantiation has the same block and shared memory, so one stands for all; its
    // shared-memory limit must be raised before the occupancy is asked (whichever instantiation
    // the caller is about to launch).
    static std::atomic<bool> attr_done[kMaxDevices];
    e = set_kernel_attributes(reinterpret_cast<const void*>(w4a4_gemm_kernel<false, 4>), (int)kSmemBytes, attr_done);
    if (e != cudaSuccess) return cuda_fail(e, "w4a4_gemm_kernel attributes");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    e = cudaOccupancyMaxActiveClusters(&n, w4a4_gemm_kernel<false, 4>, &cfg);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(gemm)");
    if (n < 1) {
      set_error("w4a4_gemm_kernel: no CTA pair fits on this device");
      return PQ_ERR_UNSUPPORTED;
    }
    if (slot) cache[dev].store(n, std::memory_order_relaxed);
  }
  *out = n;
  return PQ_OK;
}

// Shared-memory attribute of one contraction instantiation, and the register guard: the warp
// roles re-divide the launch's registers with setmaxnreg, which only works when the kernel was
// compiled with exactly the budgeted count (otherwise an increase would never be granted).
template <bool kRow, int GSL>
pq_status pair_gemm_prepare() {
  static std::atomic<bool> attr_done[kMaxDevices];
  cudaError_t e = set_kernel_attributes(reinterpret_cast<const void*>(w4a4_gemm_kernel<kRow, GSL>), (int)kSmemBytes,
                                        attr_done);
  if (e != cudaSuccess) return cuda_fail(e, "w4a4_gemm_kernel attributes");
  static std::atomic<int> num_regs_cache{-1};   // a property of the kernel binary
  int num_regs = num_regs_cache.load(std::memory_order_relaxed);
  if (num_regs < 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, w4a4_gemm_kernel<kRow, GSL>);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(gemm)");
    num_regs = fa.numRegs;
    num_regs_cache.store(num_regs, std::memory_order_relaxed);
  }
  if (num_regs != (int)REG_LAUNCH) {
    set_error("w4a4_gemm_kernel compiled with %d registers per thread, %u expected", num_regs, REG_LAUNCH);
    return PQ_ERR_CUDA;
  }
  return PQ_OK;
}

}  // namespace

size_t gemm_scratch_bytes(int64_t T, int64_t N, int64_t D) {
  return T <= kGemmSmallT ? 0 : (size_t)(T + N) * (size_t)D;
}

// Few tokens: the few-token kernel's group ranges.  Otherwise split-K when the tiles fill at most
// half of the CTA pairs the device can run at once.
int gemm_ksplit(int64_t T, int64_t N, int64_t D, int g, int* gs_out) {
  if (T <= kGemmSmallT) return gemm_small_ranges(T, N, D, g, gs_out);
  const int G = (int)(D / g);
  const int64_t tiles = ((N + PAIR_M - 1) / PAIR_M) * ((T + BN - 1) / BN);
  const int pairs = device_sm_count() / 2;
  int ks = 1, gs = G;
  if (G >= 2 * SC_GROUPS && tiles * 2 <= pairs) {
    const int want = (int)std::min<int64_t>(pairs / tiles, G / SC_GROUPS);
    gs = ((G + want - 1) / want + SC_GROUPS - 1) / SC_GROUPS * SC_GROUPS;   // multiple of 4 groups
    ks = (G + gs - 1) / gs;
    if (ks < 2) { ks = 1; gs = G; }
  }
  if (gs_out) *gs_out = gs;
  return ks;
}

size_t gemm_workspace_bytes(int64_t T, int64_t N, int64_t D, int g) {
  const int ks = gemm_ksplit(T, N, D, g, nullptr);
  return ks > 1 ? (size_t)ks * (size_t)T * (size_t)N * sizeof(float) : 0;
}

pq_status launch_splitk_reduce(const float* ws, int ksplit, int64_t T, int64_t N, void* Y, int out_bf16,
                               cudaStream_t stream) {
  const int64_t n4 = T * N / 4;                              // N % 16 == 0
  const int64_t rwant = (n4 + 255) / 256;
  const int64_t cap = (int64_t)device_sm_count() * 8;
  const int rgrid = (int)(rwant < cap ? rwant : cap);
  // Programmatic dependent of the GEMM kernel just launched on `stream` (which releases its
  // dependents at its start), so the launch overlaps the GEMM; the kernel waits before reading.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rgrid, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cuda_fail(cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, reinterpret_cast<const float4*>(ws), ksplit, n4, Y,
                                      out_bf16),
                   "splitk_reduce_kernel launch");
}

pq_status gemm_launch(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                      int64_t T, int64_t N, int64_t D, int g, void* Y, pq_out_dtype out_dtype, uint8_t* scratch,
                      float* ws, unsigned int* status, cudaStream_t stream, bool row_scale) {
  if (T <= kGemmSmallT)
    return gemm_small_launch(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype, ws, status, stream,
                             row_scale);
  uint8_t* A8 = scratch;
  uint8_t* W8 = scratch + (size_t)T * (size_t)D;
  // MMA operand A = weights (M = output channels), B = activations (N = tokens).
  CUtensorMap tmA, tmB;
  pq_status st = make_operand_map(&tmA, W8, N, D, BM);
  if (st != PQ_OK) return st;
  st = make_operand_map(&tmB, A8, T, D, BN_HALF);
  if (st != PQ_OK) return st;
  const int m_tiles = (int)((N + PAIR_M - 1) / PAIR_M);
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
  static std::atomic<bool> attr_expand[kMaxDevices];
  cudaError_t e = set_kernel_attributes(reinterpret_cast<const void*>(expand_codes_kernel), 0, attr_expand);
  if (e != cudaSuccess) return cuda_fail(e, "expand_codes_kernel attributes");
  // The contraction's attributes are set before the expansion is launched, so that a failure
  // leaves nothing enqueued.
  st = g == 64 ? (row_scale ? pair_gemm_prepare<true, 2>() : pair_gemm_prepare<false, 2>())
       : g == 256 ? (row_scale ? pair_gemm_prepare<true, 8>() : pair_gemm_prepare<false, 8>())
                  : (row_scale ? pair_gemm_prepare<true, 4>() : pair_gemm_prepare<false, 4>());
  if (st != PQ_OK) return st;
  expand_codes_kernel<<<egrid, 256, 0, stream>>>(codes_A, chunksA, codes_W, chunksW, A8, W8, g == 64 ? 1 : 0);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "expand_codes_kernel launch");
  int gs = (int)(D / g);
  const int ksplit = ws ? gemm_ksplit(T, N, D, g, &gs) : 1;
  const int64_t units = tiles * ksplit;
  int max_pairs = 0;
  st = gemm_max_pairs(sms, &max_pairs);
  if (st != PQ_OK) return st;
  const int64_t pairs = max_pairs;
  const int grid = 2 * (int)(units < pairs ? units : pairs);
  const int G = (int)(D / g);
  const int scales_vec16 = (G % SC_GROUPS == 0) ? 1 : 0;   // rows of 16-byte multiples
  const int bf16 = out_dtype == PQ_OUT_BF16 ? 1 : 0;
#define PQ_PAIR_CASE(ROW, GSL)                                                                                  \
  w4a4_gemm_kernel<ROW, GSL><<<grid, NUM_THREADS, kSmemBytes, stream>>>(tmA, tmB, scales_A, scales_W, Y, (int)T, \
                                                                         (int)N, G, scales_vec16, bf16, m_tiles, \
                                                                         n_tiles, ksplit, gs, ws, status)
  if (g == 64) {
    if (row_scale) PQ_PAIR_CASE(true, 2); else PQ_PAIR_CASE(false, 2);
  } else if (g == 256) {
    if (row_scale) PQ_PAIR_CASE(true, 8); else PQ_PAIR_CASE(false, 8);
  } else {
    if (row_scale) PQ_PAIR_CASE(true, 4); else PQ_PAIR_CASE(false, 4);
  }
#undef PQ_PAIR_CASE
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "w4a4_gemm_kernel launch");
  if (ksplit > 1) return launch_splitk_reduce(ws, ksplit, T, N, Y, out_dtype == PQ_OUT_BF16 ? 1 : 0, stream);
  return PQ_OK;
}

pq_status gemm_run(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                   int64_t T, int64_t N, int64_t D, int g, void* Y, pq_out_dtype out_dtype, cudaStream_t stream,
                   bool row_scale) {
  unsigned int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_gemm_status);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(gemm status)");
  // Stream-ordered scratch for the int8 operands: allocated and released on the caller's
  // stream, so concurrent calls on different streams never share it.
  cudaMemPool_t pool = nullptr;
  e = scratch_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "scratch memory pool");
  // Operand scratch, then (small problems) the split-K partial tiles.
  const size_t op_bytes = (gemm_scratch_bytes(T, N, D) + 255) & ~(size_t)255;
  const size_t ws_bytes = gemm_workspace_bytes(T, N, D, g);
  if (op_bytes + ws_bytes == 0)   // the few-token kernel without a split needs no scratch
    return gemm_launch(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype, nullptr, nullptr, status, stream,
                       row_scale);
  void* scratch = nullptr;
  e = cudaMallocFromPoolAsync(&scratch, op_bytes + ws_bytes, pool, stream);
  if (e != cudaSuccess) {
    set_error("cudaMallocFromPoolAsync(%zu bytes of GEMM scratch): %s", op_bytes + ws_bytes, cudaGetErrorString(e));
    return PQ_ERR_ALLOC;
  }
  float* ws = ws_bytes ? reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + op_bytes) : nullptr;
  pq_status st = gemm_launch(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype,
                             static_cast<uint8_t*>(scratch), ws, status, stream, row_scale);
  e = cudaFreeAsync(scratch, stream);
  if (st == PQ_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(gemm scratch)");
  return st;
}

pq_status gemm_run_linear(transform_launcher transform, const void* ctx, const uint8_t* codes_A, const float* scales_A,
                          const uint8_t* codes_W, const float* scales_W, int64_t T, int64_t N, int64_t D, int g,
                          void* Y, pq_out_dtype out_dtype, cudaStream_t stream) {
  if (T > kGemmSmallT) {
    pq_status st = cuda_fail(transform(ctx), "pq_w4a4_linear transform launch");
    if (st != PQ_OK) return st;
    return gemm_run(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype, stream, false);
  }
  unsigned int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_gemm_status);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(gemm status)");
  // The split workspace is taken before the transform, so that the GEMM directly follows it on
  // the stream and can be its programmatic dependent.
  const size_t ws_bytes = gemm_workspace_bytes(T, N, D, g);
  void* scratch = nullptr;
  if (ws_bytes) {
    cudaMemPool_t pool = nullptr;
    e = scratch_pool(&pool);
    if (e != cudaSuccess) return cuda_fail(e, "scratch memory pool");
    e = cudaMallocFromPoolAsync(&scratch, ws_bytes, pool, stream);
    if (e != cudaSuccess) {
      set_error("cudaMallocFromPoolAsync(%zu bytes of GEMM scratch): %s", ws_bytes, cudaGetErrorString(e));
      return PQ_ERR_ALLOC;
    }
  }
  pq_status st = cuda_fail(transform(ctx), "pq_w4a4_linear transform launch");
  if (st == PQ_OK)
    st = gemm_small_launch(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype, static_cast<float*>(scratch),
                           status, stream, false, /*pdl=*/true);
  if (scratch) {
    e = cudaFreeAsync(scratch, stream);
    if (st == PQ_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(gemm scratch)");
  }
  return st;
}

pq_status gemm_wait_timeout_selftest(uint64_t limit_ns, cudaStream_t stream) {
  unsigned int* status = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_gemm_status);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(gemm status)");
  wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns, status);
  return cuda_fail(cudaGetLastError(), "wait_timeout_kernel launch");
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
