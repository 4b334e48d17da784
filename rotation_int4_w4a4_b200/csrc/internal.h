// Internal declarations shared by the host code and the kernel launchers of libpq.
#pragma once

#include <cstdint>
#include <cstdio>
#include <string>

#include <cuda_runtime.h>

#include "../../include/pq.h"

namespace pq {

constexpr int kGroup = 128;            // the only supported group size
constexpr int kSmoothBlock = 128;      // rows per runtime-smoothing block

}  // namespace pq

// Device status word bits.
#define PQ_DEV_TIMEOUT 0x1u

struct pq_plan {
  pq_kind kind;
  int D;
  int g;
  int G;
  int K;
  uint32_t flags;
  int device;
  // Givens: tensor-core operands, bf16 [2 (activations, weights)][G][2 (hi, lo)][128 n][128 k]
  // holding R^T of R = G_0 ... G_{K-1} diag(exp(-+beta)) per group (y = x R).
  uint16_t* d_rot;
  unsigned int* d_status;   // device status word (PQ_DEV_* bits)
};

namespace pq {

// Thread-local last-error text.
void set_error(const char* fmt, ...);
void clear_error();

// Returns PQ_ERR_CUDA (with the message recorded) when err != cudaSuccess.
pq_status cuda_fail(cudaError_t err, const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Kernel launchers (transform.cu, gemm.cu).  Arguments are already validated.
// y = ((x * pre) H) * post per row-group (pre/post per channel, either may be null).
cudaError_t launch_hadamard_rows(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx,
                                 const float* pre_scale, const float* post_scale,
                                 uint8_t* codes, float* scales, cudaStream_t stream);
cudaError_t launch_smooth_hadamard(const pq_plan* plan, const void* X, int64_t T, int64_t ldx,
                                   uint8_t* codes, float* scales, float* smooth_out,
                                   cudaStream_t stream);
// y = x R per group on the tensor cores (rotate_mma.cu); weights = 0: activations, 1: weights.
cudaError_t launch_givens_mma(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, int weights,
                              uint8_t* codes, float* scales, cudaStream_t stream);
pq_status gemm_run(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W,
                   const float* scales_W, int64_t T, int64_t N, int64_t D, void* Y,
                   pq_out_dtype out_dtype, cudaStream_t stream);
// Bytes of int8 operand scratch the GEMM needs: (T + N) * D.
size_t gemm_scratch_bytes(int64_t T, int64_t N, int64_t D);
// Expansion + contraction launches on `stream` using caller-provided scratch.
pq_status gemm_launch(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W,
                      const float* scales_W, int64_t T, int64_t N, int64_t D, void* Y,
                      pq_out_dtype out_dtype, uint8_t* scratch, unsigned int* status,
                      cudaStream_t stream);
pq_status gemm_read_and_clear_status(unsigned int* bits);
// Device address of the GEMM's status word on the current device.
cudaError_t gemm_status_address(unsigned int** status);
// gemm_launch with the fixed device-array scratch of gemm_static_scratch.cu (no allocation).
pq_status gemm_run_static_scratch(const uint8_t* codes_A, const float* scales_A,
                                  const uint8_t* codes_W, const float* scales_W, int64_t T,
                                  int64_t N, int64_t D, void* Y, pq_out_dtype out_dtype,
                                  cudaStream_t stream);

}  // namespace pq
