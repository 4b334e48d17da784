// Runtime smoothing in the RRS page's order (rotate, then smooth the rotated channels) + per-group
// INT4 quantisation, on a 128-row x 128-channel tile per CTA (sm_100a).  The other order and the
// weight transforms run in smooth_rows.cu.
//
// Block Hadamard (Hadamard page §2.1/§4.2/§6.1, RRS page R = (1/sqrt(K))[s_ij]): a 128-channel
// group is held by 4 lanes, 32 consecutive channels each (four 16-byte loads per lane).  H_128
// = H_4 (x) H_32 in Sylvester order: channel bits 0..4 are transformed in registers (5 radix-2
// stages), bits 5..6 across the 4 lanes with two xor-shuffle stages.  The 1/sqrt(128) factor
// never touches the data: the codes do not depend on a uniform factor, so it is folded into the
// stored scale.  The rotated channels' maxima over the tile's rows are combined across lanes
// and warps, which needs every row of the tile in the CTA's registers at once.
//
// Quantisation (RRS page: alpha = max|X| / 7, codes in -8..7, RTN): m = max|y| over the group
// (two xor-shuffles), inv = 7/m, q = RNE(y * inv) by one FMA with 1.5 * 2^23, whose low 4 bits
// are already the two's-complement nibble; nibbles are packed with byte permutes.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "rows.cuh"

namespace pq {
namespace {

constexpr float kRoundMagic = 12582912.0f;                   // 1.5 * 2^23
constexpr float kInvSqrt128 = 0.088388347648318440550f;     // 1/sqrt(128), float-rounded
constexpr float kScaleHadamard = 0.012626906806902634f;     // 1/(7*sqrt(128)), float-rounded

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& w, float* v) {
  v[0] = __uint_as_float(w.x << 16);
  v[1] = __uint_as_float(w.x & 0xFFFF0000u);
  v[2] = __uint_as_float(w.y << 16);
  v[3] = __uint_as_float(w.y & 0xFFFF0000u);
  v[4] = __uint_as_float(w.z << 16);
  v[5] = __uint_as_float(w.z & 0xFFFF0000u);
  v[6] = __uint_as_float(w.w << 16);
  v[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

// Unnormalised Walsh-Hadamard transform of 32 register values (Sylvester order).  The first
// stage pairs neighbours; the other four run on packed float pairs (two butterflies per
// add.f32x2 / sub.f32x2, bit-identical to the scalar form).
__device__ __forceinline__ void fwht32(float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = a + b;
    v[i + 1] = a - b;
  }
#pragma unroll
  for (int h = 2; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if ((i & h) == 0) {
        const uint64_t P = ptx::f2_pack(v[i], v[i + 1]), Q = ptx::f2_pack(v[i + h], v[i + h + 1]);
        ptx::f2_unpack(ptx::f2_add(P, Q), v[i], v[i + 1]);
        ptx::f2_unpack(ptx::f2_sub(P, Q), v[i + h], v[i + h + 1]);
      }
    }
  }
}

// The two remaining radix-2 stages across the 4 lanes (lane bits 0,1 = channel bits 5,6):
// the lane holding the low half keeps a + b, the other keeps a - b (as +-v + partner).
__device__ __forceinline__ void fwht_across4(float (&v)[32], int lane) {
  const float s1 = (lane & 1) ? -1.0f : 1.0f;
  const float s2 = (lane & 2) ? -1.0f : 1.0f;
  const uint64_t S1 = ptx::f2_pack(s1, s1), S2 = ptx::f2_pack(s2, s2);
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float p0 = __shfl_xor_sync(0xffffffffu, v[i], 1), p1 = __shfl_xor_sync(0xffffffffu, v[i + 1], 1);
    ptx::f2_unpack(ptx::f2_fma(S1, ptx::f2_pack(v[i], v[i + 1]), ptx::f2_pack(p0, p1)), v[i], v[i + 1]);
  }
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float p0 = __shfl_xor_sync(0xffffffffu, v[i], 2), p1 = __shfl_xor_sync(0xffffffffu, v[i + 1], 2);
    ptx::f2_unpack(ptx::f2_fma(S2, ptx::f2_pack(v[i], v[i + 1]), ptx::f2_pack(p0, p1)), v[i], v[i + 1]);
  }
}

__device__ __forceinline__ float absmax32(const float (&v)[32]) { return row_absmax<32>(v); }

__device__ __forceinline__ float group_max4(float m) {
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  return m;
}

__device__ __forceinline__ float quant_inv(float m) { return m > 0.0f ? 7.0f * __frcp_rn(m) : 0.0f; }

// 8 values -> 8 nibbles in one word: byte k = q[2k] | q[2k+1] << 4.
__device__ __forceinline__ uint32_t quant_pack8(const float* v, float inv) {
  uint32_t b[8];
  const uint64_t I2 = ptx::f2_pack(inv, inv), M2 = ptx::f2_pack(kRoundMagic, kRoundMagic);
#pragma unroll
  for (int k = 0; k < 8; k += 2) {
    float lo, hi;
    ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(v[k], v[k + 1]), I2, M2), lo, hi);
    b[k] = __float_as_uint(lo);
    b[k + 1] = __float_as_uint(hi);
  }
  const uint32_t even = __byte_perm(__byte_perm(b[0], b[2], 0x0040), __byte_perm(b[4], b[6], 0x0040), 0x5410);
  const uint32_t odd = __byte_perm(__byte_perm(b[1], b[3], 0x0040), __byte_perm(b[5], b[7], 0x0040), 0x5410);
  return (even & 0x0F0F0F0Fu) | ((odd << 4) & 0xF0F0F0F0u);
}

__device__ __forceinline__ uint4 quant_pack32(const float (&v)[32], float inv) {
  return make_uint4(quant_pack8(v, inv), quant_pack8(v + 8, inv), quant_pack8(v + 16, inv),
                    quant_pack8(v + 24, inv));
}

// ---------------------------------------------------------------------------------------
// Runtime smoothing + Hadamard on a 128-row x 128-channel tile (one CTA, 4 warps).  Lane
// (warp w, slot = lane/4, q = lane%4) holds rows 32k + 8w + slot (k = 0..3), channels 32q..+31.
// after_rotate = false: s = max|x| per channel over the tile's rows, y = (x / s) H.
// after_rotate = true:  s = max|x H| per channel (rotated channels), y = (x H) / s.
// Four CTAs per SM (128 registers per thread): the kernel is latency-bound, and the extra
// resident tiles outweigh a few spilled registers (measured on down_proj: 217 -> 172 us).
__global__ void __launch_bounds__(128, 4) smooth_hadamard_kernel(
    const __nv_bfloat16* __restrict__ X, int64_t T, int64_t ldx, int G, int after_rotate,
    uint8_t* __restrict__ codes, float* __restrict__ scales, float* __restrict__ smooth_out) {
  __shared__ __align__(16) float red[4][4][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, q = lane & 3, slot = lane >> 2;
  const int64_t b = blockIdx.x;
  const int gi = blockIdx.y;
  const int c0 = gi * 128 + q * 32;
  const int64_t D = (int64_t)G * 128;

  uint4 x[4][4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t t = b * 128 + 32 * k + 8 * w + slot;
    if (t < T) {
      const uint4* p = reinterpret_cast<const uint4*>(X + t * ldx + c0);
#pragma unroll
      for (int j = 0; j < 4; ++j) x[k][j] = ld_stream(p + j);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) x[k][j] = make_uint4(0, 0, 0, 0);
    }
  }

  // Per-channel maximum over the tile -> s (32 channels per lane).
  float s[32];
  if (!after_rotate) {
    // |bf16| compared as unsigned 16-bit integers (sign bit cleared): exact, no conversion.
    uint32_t mw[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) mw[j] = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(&x[k][0]);
#pragma unroll
      for (int j = 0; j < 16; ++j) mw[j] = __vmaxu2(mw[j], xw[j] & 0x7FFF7FFFu);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      mw[j] = __vmaxu2(mw[j], __shfl_xor_sync(0xffffffffu, mw[j], 4));
      mw[j] = __vmaxu2(mw[j], __shfl_xor_sync(0xffffffffu, mw[j], 8));
      mw[j] = __vmaxu2(mw[j], __shfl_xor_sync(0xffffffffu, mw[j], 16));
    }
    if (slot == 0) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        red[w][q][2 * j] = __uint_as_float(mw[j] << 16);
        red[w][q][2 * j + 1] = __uint_as_float(mw[j] & 0xFFFF0000u);
      }
    }
  } else {
    float cm[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) cm[i] = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float v[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) bf16x8_to_f32(x[k][j], v + 8 * j);
      fwht32(v);
      fwht_across4(v, lane);
#pragma unroll
      for (int i = 0; i < 32; ++i) cm[i] = fmaxf(cm[i], fabsf(v[i]));
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      cm[i] = fmaxf(cm[i], __shfl_xor_sync(0xffffffffu, cm[i], 4));
      cm[i] = fmaxf(cm[i], __shfl_xor_sync(0xffffffffu, cm[i], 8));
      cm[i] = fmaxf(cm[i], __shfl_xor_sync(0xffffffffu, cm[i], 16));
    }
    if (slot == 0) {
#pragma unroll
      for (int i = 0; i < 32; ++i) red[w][q][i] = cm[i];
    }
  }
  __syncthreads();
  float rs[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float m = fmaxf(fmaxf(red[0][q][i], red[1][q][i]), fmaxf(red[2][q][i], red[3][q][i]));
    // Reported s is for the normalised rotation; the kernel divides unnormalised values by the
    // unnormalised maximum, which gives the same quotient.
    s[i] = m > 0.0f ? (after_rotate ? m * kInvSqrt128 : m) : 1.0f;
    rs[i] = m > 0.0f ? __frcp_rn(m) : 0.0f;
  }
  if (smooth_out && w == 0 && slot == 0) {
    float4* dst = reinterpret_cast<float4*>(smooth_out + b * D + c0);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_float4(s[4 * j], s[4 * j + 1], s[4 * j + 2], s[4 * j + 3]);
  }

#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t t = b * 128 + 32 * k + 8 * w + slot;
    float v[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) bf16x8_to_f32(x[k][j], v + 8 * j);
    if (!after_rotate) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= rs[i];
    }
    fwht32(v);
    fwht_across4(v, lane);
    if (after_rotate) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= rs[i];
    }
    const float m = group_max4(absmax32(v));
    const uint4 packed = quant_pack32(v, quant_inv(m));
    if (t < T) {
      *reinterpret_cast<uint4*>(codes + t * (D / 2) + gi * 64 + q * 16) = packed;
      // before the rotation the values are x/s (normalised range), after it (x H)/s_unnorm.
      if (q == 0) scales[t * G + gi] = after_rotate ? __fdiv_rn(m, 7.0f) : m * kScaleHadamard;
    }
  }
}

}  // namespace

cudaError_t launch_smooth_hadamard(const pq_plan* plan, const void* X, int64_t T, int64_t ldx,
                                   uint8_t* codes, float* scales, float* smooth_out,
                                   cudaStream_t stream) {
  dim3 grid((unsigned)((T + kSmoothBlock - 1) / kSmoothBlock), (unsigned)plan->G);
  static std::atomic<bool> attr_done[kMaxDevices];
  cudaError_t e = set_kernel_attributes(reinterpret_cast<const void*>(smooth_hadamard_kernel), 0, attr_done);
  if (e != cudaSuccess) return e;
  smooth_hadamard_kernel<<<grid, 128, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(X), T, ldx, plan->G,
      (plan->flags & PQ_FLAG_SMOOTH_AFTER_ROTATE) ? 1 : 0, codes, scales, smooth_out);
  return cudaGetLastError();
}

}  // namespace pq
