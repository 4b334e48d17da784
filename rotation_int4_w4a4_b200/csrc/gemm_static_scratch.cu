// W4A4 GEMM entry whose int8 operand scratch is a fixed device array of this module rather than
// a stream-ordered allocation (the entry point pq_w4a4_gemm_noalloc).
//
// Why it exists: pq_w4a4_gemm takes its (T + N) * D bytes of scratch from a library-owned memory
// pool on every call.  Some callers cannot let a library allocate at all: an inference engine
// that has already reserved nearly all device memory for its own caches (so any further
// allocation may fail at an arbitrary moment mid-run), or a serving loop that needs a fixed,
// known device footprint and no allocator work on its steady-state path.  This entry gives them
// the same kernels with a bounded scratch that exists from the moment this module is loaded.
//
// Limits and sharing:
//   * The scratch holds PQ_NOALLOC_SCRATCH_BYTES (32 MiB); calls needing more are rejected
//     before anything touches the device.
//   * There is one scratch array per device, shared by every call on that device: two calls
//     whose GPU work overlaps in time (different streams with no ordering between them) race on
//     it and may silently produce wrong results.
//   * The scratch need not start at zero: every byte the contraction reads is written first by
//     the expansion kernel of the same call, in stream order.  The GEMM status word (shared
//     with pq_w4a4_gemm) must start at zero; it is zero at load and after every
//     pq_check_status.
#include <mutex>

#include "internal.h"

namespace pq {

static __device__ __align__(256) uint8_t g_static_scratch[PQ_NOALLOC_SCRATCH_BYTES];

namespace {

struct DeviceSetup {
  bool ready = false;
  uint8_t* scratch = nullptr;
  unsigned int* status = nullptr;
};

// One-time set-up per device, done with that device current: look up the device addresses of
// the scratch array and the status word.  Neither lookup allocates memory.
pq_status device_setup(int dev, DeviceSetup* out) {
  static std::mutex mu;
  static DeviceSetup setups[kMaxDevices];
  std::lock_guard<std::mutex> lock(mu);
  DeviceSetup& s = setups[dev];
  if (!s.ready) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static GEMM scratch)");
    unsigned int* status = nullptr;
    e = gemm_status_address(&status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(gemm status)");
    s.scratch = static_cast<uint8_t*>(p);
    s.status = status;
    s.ready = true;
  }
  *out = s;
  return PQ_OK;
}

}  // namespace

pq_status gemm_run_static_scratch(const uint8_t* codes_A, const float* scales_A,
                                  const uint8_t* codes_W, const float* scales_W, int64_t T,
                                  int64_t N, int64_t D, int g, void* Y, pq_out_dtype out_dtype,
                                  cudaStream_t stream) {
  const size_t need = gemm_scratch_bytes(T, N, D);
  if (need > (size_t)PQ_NOALLOC_SCRATCH_BYTES) {
    set_error("(T + N) * D = %zu bytes of int8 scratch needed; the fixed scratch holds %zu "
              "(use pq_w4a4_gemm, or split the call along T or N)",
              need, (size_t)PQ_NOALLOC_SCRATCH_BYTES);
    return PQ_ERR_INVALID_ARG;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("device %d: at most %d devices are supported", dev, kMaxDevices);
    return PQ_ERR_UNSUPPORTED;
  }
  DeviceSetup s;
  pq_status st = device_setup(dev, &s);
  if (st != PQ_OK) return st;
  return gemm_launch(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype, s.scratch,
                     /*ws=*/nullptr, s.status, stream, /*row_scale=*/false);
}

}  // namespace pq
