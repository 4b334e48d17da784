// W4A4 GEMM for a handful of tokens (T <= kGemvT = 4: single-token decode and small batches) on
// the CUDA cores, sm_100a.
//
// Y[t][n] = sum_G sa[t][G] * sw[n][G] * d_G[t][n] (RRS page, main equation, last line; Fig. 4
// step (3) with block size = group size).  With one to a few tokens the product is a
// matrix-vector product: each packed weight byte is used T times, so the call streams N D / 2
// bytes of weights for 2 T N D integer operations and is bound by HBM and by latency, not by the
// tensor cores.  The tensor-core kernels' fixed costs (tensor-memory allocation, barrier set-up,
// pipeline fill, the widening of packed codes into a second buffer) dominate there; this kernel
// keeps the weights in the registers they are loaded into:
//   - a warp owns R = 2 weight rows; lane l reads 16 packed bytes (32 codes) of each row per
//     512-byte K-step at byte l * 16, so every load instruction covers 512 contiguous bytes of a
//     row, and it issues the loads of four K-steps before it uses the first (2 KB per row in
//     flight per warp; at decode sizes the warps of one wave request most of the weight matrix
//     at once);
//   - the nibbles become int8 values q * 16 (low nibble: shift left by 4 and mask; high nibble:
//     mask), and __dp4a gives 256 times the dot product of each 32-code slice with the token's
//     slice, exact in int32;
//   - a group (g codes = g / 2 bytes) is g / 32 consecutive lanes: their R x T partial dots are
//     summed by xor shuffles that also spread the (row, token) pairs over the lanes (each step
//     halves the values a lane holds), so each lane finishes R T / (g / 32) of the group's dots;
//   - per finished dot: acc += fl(float(256 d) * (sw / 256)) * sa, i.e. fl(d * sw) * sa as in
//     the other GEMM kernels (row-scale mode: acc += float(256 d) * (F / 256), the token scale at
//     the store); each lane's groups are taken in ascending order, and the lanes' sums over the
//     warp's group slots are added by a final shuffle tree: float32 rounding of a different
//     summation order, the integer dots themselves unchanged.
// No shared memory, no barriers, no waits: nothing in the kernel can block.
//
// Measured alternatives that were slower on B200 (decode sizes, L2 flushed): a persistent grid
// with 8-warp blocks and the token codes in shared memory (more registers, fewer warps in
// flight), and a per-warp ring of 1-D bulk copies into shared memory (16 warps per SM, 4 x 2 KB
// slots each).  Beyond 4 tokens the dp4a work makes the tensor-core kernel the faster one at
// N = 14336.
#include <cuda_bf16.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace pq {
namespace {

constexpr int GV_WARPS = 4;      // warps per block
constexpr int GV_R = 2;          // weight rows per warp
constexpr int GV_UB = 4;         // 512-byte K-steps whose loads are issued together

// Packed bytes (16) -> int8 q * 16 for the low nibbles (lo) and the high nibbles (hi).
__device__ __forceinline__ void gv_widen(const uint4& w, int (&lo)[4], int (&hi)[4]) {
  lo[0] = (int)((w.x << 4) & 0xF0F0F0F0u);
  lo[1] = (int)((w.y << 4) & 0xF0F0F0F0u);
  lo[2] = (int)((w.z << 4) & 0xF0F0F0F0u);
  lo[3] = (int)((w.w << 4) & 0xF0F0F0F0u);
  hi[0] = (int)(w.x & 0xF0F0F0F0u);
  hi[1] = (int)(w.y & 0xF0F0F0F0u);
  hi[2] = (int)(w.z & 0xF0F0F0F0u);
  hi[3] = (int)(w.w & 0xF0F0F0F0u);
}

// Weights are read once: no L1 allocation, so the token codes keep the L1.
__device__ __forceinline__ uint4 gv_load_stream(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

template <int NT, int GW>
__global__ void __launch_bounds__(32 * GV_WARPS) w4a4_gemv_kernel(
    const uint8_t* __restrict__ codes_A, const float* __restrict__ scales_A, const uint8_t* __restrict__ codes_W,
    const float* __restrict__ scales_W, void* __restrict__ Y, int T, int N, int D2, int G, int row_scale,
    int out_bf16, int pdl) {
  constexpr int LPG = GW / 32;                           // lanes per group
  constexpr int P = GV_R * NT;                           // (row, token) pairs, index p = r NT + t
  constexpr int KH = ilog2(P < LPG ? P : LPG);           // halving shuffle steps
  constexpr int NV = P >> KH;                            // dots each lane finishes per K-step
  const int lane = threadIdx.x & 31;
  const int q = lane & (LPG - 1);                        // lane within its group
  const int64_t n0 = ((int64_t)blockIdx.x * GV_WARPS + (threadIdx.x >> 5)) * GV_R;
  if (n0 >= N) return;
  // After the halving steps lane q holds pairs p = i 2^KH + (q mod 2^KH); lanes that differ
  // only in the bits of q above KH hold the same sums, and only the one with those bits clear
  // accumulates them.
  const bool owner = (q >> KH) == 0;
  const int qlow = q & ((1 << KH) - 1);
  const int nsteps = (D2 + 511) / 512;

  float acc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) acc[i] = 0.0f;

  for (int s0 = 0; s0 < nsteps; s0 += GV_UB) {
    uint4 w[GV_UB][GV_R];
#pragma unroll
    for (int u = 0; u < GV_UB; ++u) {
      const int off = (s0 + u) * 512 + lane * 16;
#pragma unroll
      for (int r = 0; r < GV_R; ++r)
        w[u][r] = (off < D2 && n0 + r < N) ? gv_load_stream(codes_W + (n0 + r) * (int64_t)D2 + off)
                                           : make_uint4(0u, 0u, 0u, 0u);
    }
    // Launched as the dependent of the kernel that writes the token codes and scales: the first
    // weight loads are in flight before the wait, every read of codes_A / scales_A after it.
    if (pdl && s0 == 0) ptx::griddep_wait();
#pragma unroll
    for (int u = 0; u < GV_UB; ++u) {
      if (s0 + u >= nsteps) break;                       // the same for the whole warp
      const int off = (s0 + u) * 512 + lane * 16;
      int wl[GV_R][4], wh[GV_R][4];
#pragma unroll
      for (int r = 0; r < GV_R; ++r) gv_widen(w[u][r], wl[r], wh[r]);
      int v[P];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const uint4 a = (t < T && off < D2) ? __ldg(reinterpret_cast<const uint4*>(codes_A + (int64_t)t * D2 + off))
                                            : make_uint4(0u, 0u, 0u, 0u);
        int al[4], ah[4];
        gv_widen(a, al, ah);
#pragma unroll
        for (int r = 0; r < GV_R; ++r) {
          int d0 = __dp4a(wl[r][0], al[0], 0);
          int d1 = __dp4a(wh[r][0], ah[0], 0);
#pragma unroll
          for (int j = 1; j < 4; ++j) {
            d0 = __dp4a(wl[r][j], al[j], d0);
            d1 = __dp4a(wh[r][j], ah[j], d1);
          }
          v[r * NT + t] = d0 + d1;
        }
      }
      // Sum over the group's lanes.  Halving step with lane bit b: keep the pairs whose index
      // bit matches b, send the others to the partner lane (which keeps those), add.
#pragma unroll
      for (int k = 0; k < ilog2(LPG); ++k) {
        const int b = 1 << k;
        const bool up = (lane & b) != 0;
        if (k < KH) {
#pragma unroll
          for (int i = 0; i < (P >> (k + 1)); ++i) {
            const int keep = up ? v[2 * i + 1] : v[2 * i];
            const int send = up ? v[2 * i] : v[2 * i + 1];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, b);
          }
        } else {
          v[0] += __shfl_xor_sync(0xffffffffu, v[0], b);
        }
      }
      const int grp = off / (GW / 2);                    // this lane's group
      if (owner && off < D2) {
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int p = (i << KH) + qlow;
          const int r = p / NT, t = p % NT;
          if (n0 + r < N && t < T) {
            const float sw = __ldg(scales_W + (n0 + r) * (int64_t)G + grp) * 0.00390625f;
            const float d256 = __int2float_rn(v[i]);
            acc[i] = row_scale ? fmaf(d256, sw, acc[i]) : fmaf(d256 * sw, __ldg(scales_A + (int64_t)t * G + grp), acc[i]);
          }
        }
      }
    }
  }
  // Add the group slots: lanes with the same q, from lane bit log2(g / 32) up.
#pragma unroll
  for (int o = LPG; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < NV; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  if (lane < LPG && owner) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int p = (i << KH) + qlow;
      const int r = p / NT, t = p % NT;
      if (n0 + r < N && t < T) {
        const float y = row_scale ? acc[i] * __ldg(scales_A + t) : acc[i];
        const int64_t idx = (int64_t)t * N + n0 + r;
        if (out_bf16) reinterpret_cast<__nv_bfloat16*>(Y)[idx] = __float2bfloat16_rn(y);
        else reinterpret_cast<float*>(Y)[idx] = y;
      }
    }
  }
}

template <int NT, int GW>
cudaError_t launch_gemv(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                        void* Y, int T, int N, int D2, int G, int row_scale, int out_bf16, bool pdl,
                        cudaStream_t stream) {
  const int rows_per_block = GV_R * GV_WARPS;
  const unsigned grid = (unsigned)((N + rows_per_block - 1) / rows_per_block);
  if (!pdl) {
    w4a4_gemv_kernel<NT, GW><<<grid, 32 * GV_WARPS, 0, stream>>>(codes_A, scales_A, codes_W, scales_W, Y, T, N, D2,
                                                                  G, row_scale, out_bf16, 0);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(32 * GV_WARPS, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, w4a4_gemv_kernel<NT, GW>, codes_A, scales_A, codes_W, scales_W, Y, T, N, D2, G,
                            row_scale, out_bf16, 1);
}

template <int GW>
cudaError_t launch_gemv_g(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                          void* Y, int T, int N, int D2, int G, int row_scale, int out_bf16, bool pdl,
                          cudaStream_t stream) {
  if (T <= 1) return launch_gemv<1, GW>(codes_A, scales_A, codes_W, scales_W, Y, T, N, D2, G, row_scale, out_bf16, pdl, stream);
  if (T <= 2) return launch_gemv<2, GW>(codes_A, scales_A, codes_W, scales_W, Y, T, N, D2, G, row_scale, out_bf16, pdl, stream);
  return launch_gemv<4, GW>(codes_A, scales_A, codes_W, scales_W, Y, T, N, D2, G, row_scale, out_bf16, pdl, stream);
}

static_assert(kGemvT <= 4, "the CUDA-core kernel is instantiated for at most 4 tokens");

}  // namespace

pq_status gemv_launch(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                      int64_t T, int64_t N, int64_t D, int g, void* Y, pq_out_dtype out_dtype, cudaStream_t stream,
                      bool row_scale, bool pdl) {
  if (T <= 0 || N <= 0) return PQ_OK;
  const int D2 = (int)(D / 2), G = (int)(D / g);
  const int rs = row_scale ? 1 : 0, bf = out_dtype == PQ_OUT_BF16 ? 1 : 0;
  cudaError_t e;
  if (g == 64)
    e = launch_gemv_g<64>(codes_A, scales_A, codes_W, scales_W, Y, (int)T, (int)N, D2, G, rs, bf, pdl, stream);
  else if (g == 256)
    e = launch_gemv_g<256>(codes_A, scales_A, codes_W, scales_W, Y, (int)T, (int)N, D2, G, rs, bf, pdl, stream);
  else
    e = launch_gemv_g<128>(codes_A, scales_A, codes_W, scales_W, Y, (int)T, (int)N, D2, G, rs, bf, pdl, stream);
  return cuda_fail(e, pdl ? "w4a4_gemv_kernel launch (programmatic dependent)" : "w4a4_gemv_kernel launch");
}

}  // namespace pq
