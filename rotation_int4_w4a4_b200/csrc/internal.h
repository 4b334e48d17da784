// Internal declarations shared by the host code and the kernel launchers of libpq.
#pragma once

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <string>

#include <cuda.h>
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
  // Tensor-core rotation operands (bf16, [n][k] = R[k][n]), one 128 x 128 matrix per tile:
  //   Givens:   [2 (activations, weights)][D/128][2 (hi, lo)][128][128] for R = G_0 ... G_{K-1}
  //             diag(exp(-+beta)) per group (y = x R; two groups on the diagonal at g = 64);
  //   Hadamard: unnormalised H_128, diag(H_64, H_64) (g = 64) or +H_128 and -H_128 (g = 256).
  uint16_t* d_rot;
  unsigned int* d_status;   // device status word (PQ_DEV_* bits)
  // 8-bit outlier groups (g = 128): n8 groups, d_slot8[G] = the group's index among them or -1.
  // Codes and scales then have Gx = G + 3 n8 groups per row (four 4-bit digit groups per 8-bit
  // group: its own slot and three appended at G + 3 j).
  int n8;
  int Gx;
  int16_t* d_slot8;
};

namespace pq {

// Thread-local last-error text.
void set_error(const char* fmt, ...);
void clear_error();

// Returns PQ_ERR_CUDA (with the message recorded) when err != cudaSuccess.
pq_status cuda_fail(cudaError_t err, const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device caches below hold one slot per device index; devices beyond the table are
// served without caching.  Every cached value is the same whichever thread computes it first,
// so concurrent first calls from several host threads only repeat an idempotent query.
constexpr int kMaxDevices = 64;

// Kernel attributes set once per device and kernel (the dynamic shared-memory limit), so that
// launches do not repeat the driver call.  `done` is the caller's per-kernel table.
inline cudaError_t set_kernel_attributes(const void* func, int dyn_smem, std::atomic<bool> (&done)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  if (slot && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  if (dyn_smem > 0) {
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
    if (e != cudaSuccess) return e;
  }
  if (slot) done[dev].store(true, std::memory_order_release);
  return cudaSuccess;
}

// For kernels whose dynamic shared memory depends on the call's sizes: raises the kernel's limit
// whenever a call needs more than the largest value set so far on this device (`largest` is the
// caller's per-kernel table; the limit only grows, so a larger earlier call keeps later ones valid).
inline cudaError_t raise_dynamic_smem(const void* func, int dyn_smem, std::atomic<int> (&largest)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  if (slot && largest[dev].load(std::memory_order_acquire) >= dyn_smem) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
  if (e != cudaSuccess) return e;
  if (slot) {
    int cur = largest[dev].load(std::memory_order_relaxed);
    while (cur < dyn_smem && !largest[dev].compare_exchange_weak(cur, dyn_smem, std::memory_order_acq_rel)) {
    }
  }
  return cudaSuccess;
}

// Multiprocessor count of the current device (148 if it cannot be read).
inline int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  int c = slot ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (c <= 0) {
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
    if (slot) cache[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

// Kernel launchers (transform.cu, smooth_rows.cu, rotate_mma.cu, gemm.cu).  Arguments are
// already validated.
// Tensor map of a bf16 [rows][inner] matrix (row stride ld elements): 64 x 128 boxes, 128-byte
// swizzle, zero fill outside (rotate_mma.cu).
cudaError_t make_bf16_tile_map(CUtensorMap* map, const void* base, int64_t rows, int64_t inner, int64_t ld);
// Tensor map of a dense uint8 [rows][inner] matrix: box_inner bytes x box_rows, zero fill outside,
// optionally the 128-byte swizzle (rotate_mma.cu).
cudaError_t make_u8_tile_map(CUtensorMap* map, const void* base, int64_t rows, int64_t inner, int box_inner,
                             int box_rows, bool swizzle128);
// bf16 rows [rows][D] as lines of 128 bytes: a box of box_rows whole rows, 128-byte swizzle,
// rows past the end zero-filled (D / 64 <= 256).
cudaError_t make_bf16_row_lines_map(CUtensorMap* map, const void* base, int64_t rows, int64_t D, int64_t ld,
                                    int box_rows);
// y = ((x * a) H) * b per row and group, one thread per row (smooth_rows.cu).  mode 0: a = 1/s with
// s the per-channel max |x| over each 128-row block (to smooth_out if non-null); 1: a = vec;
// 2: b = vec; 3: neither.
enum { PQ_SR_COLMAX = 0, PQ_SR_PRE = 1, PQ_SR_POST = 2, PQ_SR_NONE = 3 };
cudaError_t launch_smooth_rows(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, int mode,
                               const float* vec, uint8_t* codes, float* scales, float* smooth_out,
                               cudaStream_t stream);
// Rotated runtime smoothing with channel reordering (rrs.cu): chan_max (float, [D]), perm and
// inv_perm (int32, [D]) and group_scale ([G]) from the activations; then the row transforms
// (weights = 0: per-token activation codes and scales [rows]; 1: per-group weight codes and
// scales with the group's smoothing scale folded in).  rrs_rows_smem_bytes: shared memory per CTA.
cudaError_t launch_rrs_prepare(const pq_plan* plan, const void* X, int64_t T, int64_t ldx, float* chan_max,
                               int* perm, int* inv_perm, float* group_scale, cudaStream_t stream);
cudaError_t launch_rrs_rows(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, int weights,
                            const int* perm, const float* group_scale, uint8_t* codes, float* scales,
                            cudaStream_t stream);
size_t rrs_rows_smem_bytes(int D);
// Runtime smoothing after the rotation (PQ_FLAG_SMOOTH_AFTER_ROTATE activations; transform.cu).
cudaError_t launch_smooth_hadamard(const pq_plan* plan, const void* X, int64_t T, int64_t ldx,
                                   uint8_t* codes, float* scales, float* smooth_out,
                                   cudaStream_t stream);
// y = x R per group on the tensor cores (rotate_mma.cu) for PQ_GIVENS and PQ_HADAMARD plans;
// weights = 0: activations, 1: weights.  With chan_max (float bits, [D], zeroed by the caller)
// nothing is quantised: chan_max[j] becomes max over the rows of |y[:, j]| (normalised rotation).
cudaError_t launch_rotate_mma(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, int weights,
                              uint8_t* codes, float* scales, cudaStream_t stream, unsigned int* chan_max = nullptr);
// Activation transforms of at most this many rows (Hadamard or Givens, g = 64 or 128, no 8-bit
// groups) run one warp per (row, 128-channel tile) on the CUDA cores (rows_small.cu).
constexpr int64_t kRowsSmallT = 16;
bool rows_small_applies(const pq_plan* plan, int64_t rows);
cudaError_t launch_rows_small(const pq_plan* plan, const void* X, int64_t rows, int64_t ldx, uint8_t* codes,
                              float* scales, cudaStream_t stream);
// Calls with at most this many tokens take the few-token kernel (gemm_small.cu): packed codes
// read directly, int8 tensor-core products, no operand scratch.
constexpr int64_t kGemmSmallT = 128;
// Calls with at most this many tokens take the CUDA-core kernel (gemv.cu) instead: weights
// streamed into registers, __dp4a products, one launch, no workspace.
constexpr int64_t kGemvT = 4;
pq_status gemv_launch(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W, const float* scales_W,
                      int64_t T, int64_t N, int64_t D, int g, void* Y, pq_out_dtype out_dtype, cudaStream_t stream,
                      bool row_scale, bool pdl);
// Group ranges per 128-row weight tile of the few-token kernel (1 = no split); g = group size.
int gemm_small_ranges(int64_t T, int64_t N, int64_t D, int g, int* gs_out);
// The few-token GEMM (+ the split reduction when ws != nullptr and the sizes call for it).
// pdl: launch it as the programmatic dependent of the preceding kernel on `stream`, which must be
// the one writing codes_A and scales_A, itself started after everything codes_W and scales_W
// depend on.
pq_status gemm_small_launch(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W,
                            const float* scales_W, int64_t T, int64_t N, int64_t D, int g, void* Y,
                            pq_out_dtype out_dtype, float* ws, unsigned int* status, cudaStream_t stream,
                            bool row_scale, bool pdl = false);
// Y = sum over ksplit float32 partial [T][N] tiles in ws, ascending (gemm.cu).
pq_status launch_splitk_reduce(const float* ws, int ksplit, int64_t T, int64_t N, void* Y, int out_bf16,
                               cudaStream_t stream);
// row_scale: scales_W holds per-(row, group) factors and scales_A one scale per token, applied
// after the groups (the rotated-runtime-smoothing GEMM); otherwise both are per (row, group).
pq_status gemm_run(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W,
                   const float* scales_W, int64_t T, int64_t N, int64_t D, int g, void* Y,
                   pq_out_dtype out_dtype, cudaStream_t stream, bool row_scale = false);
// Bytes of operand scratch the GEMM needs: (T + N) * D for the expanded operands (none for the
// few-token kernel).
size_t gemm_scratch_bytes(int64_t T, int64_t N, int64_t D);
// Split-K factor for a problem (1 = none) and the groups per range; the float32 partial-tile
// workspace it needs (0 when unsplit), for whichever kernel the sizes select.
int gemm_ksplit(int64_t T, int64_t N, int64_t D, int g, int* gs_out);
size_t gemm_workspace_bytes(int64_t T, int64_t N, int64_t D, int g);
// Expansion + contraction (+ split-K reduction) launches on `stream` using caller-provided
// scratch; ws = nullptr disables split-K.
pq_status gemm_launch(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W,
                      const float* scales_W, int64_t T, int64_t N, int64_t D, int g, void* Y,
                      pq_out_dtype out_dtype, uint8_t* scratch, float* ws, unsigned int* status,
                      cudaStream_t stream, bool row_scale);
// pq_w4a4_linear: `transform(ctx)` launches the activation transform (writing codes_A and
// scales_A) on `stream`; the GEMM follows.  T <= 128: the few-token GEMM is launched as the
// transform's programmatic dependent (its weight loads overlap the transform; the split
// workspace, if any, is allocated before the transform).  T > 128: as pq_w4a4_gemm.
typedef cudaError_t (*transform_launcher)(const void* ctx);
pq_status gemm_run_linear(transform_launcher transform, const void* ctx, const uint8_t* codes_A, const float* scales_A,
                          const uint8_t* codes_W, const float* scales_W, int64_t T, int64_t N, int64_t D, int g,
                          void* Y, pq_out_dtype out_dtype, cudaStream_t stream);
pq_status gemm_read_and_clear_status(unsigned int* bits);
// Launches the bounded-wait diagnostic (a wait that cannot complete, limited to limit_ns).
pq_status gemm_wait_timeout_selftest(uint64_t limit_ns, cudaStream_t stream);
// Device address of the GEMM's status word on the current device.
cudaError_t gemm_status_address(unsigned int** status);
// gemm_launch with the fixed device-array scratch of gemm_static_scratch.cu (no allocation).
pq_status gemm_run_static_scratch(const uint8_t* codes_A, const float* scales_A,
                                  const uint8_t* codes_W, const float* scales_W, int64_t T,
                                  int64_t N, int64_t D, int g, void* Y, pq_out_dtype out_dtype,
                                  cudaStream_t stream);

}  // namespace pq
