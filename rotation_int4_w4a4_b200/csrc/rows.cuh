// Register-resident helpers shared by the row-wise transform kernels (sm_100a): bf16 decoding, the
// unnormalised 128-point Walsh-Hadamard transform and nibble packing.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace pq {

constexpr float kRowRoundMagic = 12582912.0f;          // 1.5 * 2^23

__device__ __forceinline__ void row_bf16x8(const uint4& w, float* v) {
  v[0] = __uint_as_float(w.x << 16);
  v[1] = __uint_as_float(w.x & 0xFFFF0000u);
  v[2] = __uint_as_float(w.y << 16);
  v[3] = __uint_as_float(w.y & 0xFFFF0000u);
  v[4] = __uint_as_float(w.z << 16);
  v[5] = __uint_as_float(w.z & 0xFFFF0000u);
  v[6] = __uint_as_float(w.w << 16);
  v[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

// Unnormalised Walsh-Hadamard transform of 128 register values, Sylvester order (Hadamard page
// §4.2 butterflies): stage h maps (v[i], v[i + h]) to (v[i] + v[i + h], v[i] - v[i + h]).  The
// first stage pairs neighbours; the others run on packed float pairs.
__device__ __forceinline__ void row_fwht128(float (&v)[128]) {
#pragma unroll
  for (int i = 0; i < 128; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = a + b;
    v[i + 1] = a - b;
  }
#pragma unroll
  for (int h = 2; h < 128; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 128; i += 2) {
      if ((i & h) == 0) {
        const uint64_t P = ptx::f2_pack(v[i], v[i + 1]), Q = ptx::f2_pack(v[i + h], v[i + h + 1]);
        ptx::f2_unpack(ptx::f2_add(P, Q), v[i], v[i + 1]);
        ptx::f2_unpack(ptx::f2_sub(P, Q), v[i + h], v[i + h + 1]);
      }
    }
  }
}

// The same transform on 32 register values (the low 5 bits of the channel index); callers
// finish the higher bits across threads.
__device__ __forceinline__ void row_fwht32(float (&v)[32]) {
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

// max |v[i]| over N register values (N a multiple of 8) with eight independent partial maxima,
// so the dependency chain is N/8 + 3 long instead of N; the maximum is exact in any order.
template <int N>
__device__ __forceinline__ float row_absmax(const float* v) {
  static_assert(N % 8 == 0 && N >= 8, "N must be a positive multiple of 8");
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fabsf(v[k]);
#pragma unroll
  for (int i = 8; i < N; ++i) m[i & 7] = fmaxf(m[i & 7], fabsf(v[i]));
#pragma unroll
  for (int w = 4; w > 0; w >>= 1)
#pragma unroll
    for (int k = 0; k < w; ++k) m[k] = fmaxf(m[k], m[k + w]);
  return m[0];
}

// 8 values -> 8 nibbles: byte k = q[2k] | q[2k+1] << 4, q = RNE(v * inv) (|q| <= 7); the FMA with
// 1.5 * 2^23 leaves q's two's-complement low bits in the low byte (packed-pair FMAs, the same
// float32 operation on each value).
__device__ __forceinline__ uint32_t row_pack8(const float* v, float inv) {
  uint32_t b[8];
  const uint64_t inv2 = ptx::f2_pack(inv, inv), magic2 = ptx::f2_pack(kRowRoundMagic, kRowRoundMagic);
#pragma unroll
  for (int k = 0; k < 8; k += 2) {
    float lo, hi;
    ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(v[k], v[k + 1]), inv2, magic2), lo, hi);
    b[k] = __float_as_uint(lo);
    b[k + 1] = __float_as_uint(hi);
  }
  const uint32_t even = __byte_perm(__byte_perm(b[0], b[2], 0x0040), __byte_perm(b[4], b[6], 0x0040), 0x5410);
  const uint32_t odd = __byte_perm(__byte_perm(b[1], b[3], 0x0040), __byte_perm(b[5], b[7], 0x0040), 0x5410);
  return (even & 0x0F0F0F0Fu) | ((odd << 4) & 0xF0F0F0F0u);
}

}  // namespace pq
