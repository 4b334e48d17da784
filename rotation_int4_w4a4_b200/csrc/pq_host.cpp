// Host side of libpq: argument validation, greedy pair selection, plan tables, status.
#include <cmath>
#include <cstdarg>
#include <cstring>
#include <new>
#include <vector>

#include "internal.h"

namespace pq {

static thread_local char g_last_error[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

void clear_error() { g_last_error[0] = '\0'; }

pq_status cuda_fail(cudaError_t err, const char* what) {
  if (err == cudaSuccess) return PQ_OK;
  set_error("%s: %s (%s)", what, cudaGetErrorString(err), cudaGetErrorName(err));
  return PQ_ERR_CUDA;
}

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014), from its published definition.
struct SplitMix64 {
  uint64_t state;
  explicit SplitMix64(uint64_t seed) : state(seed) {}
  uint64_t next() {
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

}  // namespace pq

using namespace pq;

extern "C" const char* pq_status_string(pq_status s) {
  switch (s) {
    case PQ_OK: return "PQ_OK";
    case PQ_ERR_INVALID_ARG: return "PQ_ERR_INVALID_ARG";
    case PQ_ERR_UNSUPPORTED: return "PQ_ERR_UNSUPPORTED";
    case PQ_ERR_CUDA: return "PQ_ERR_CUDA";
    case PQ_ERR_ALLOC: return "PQ_ERR_ALLOC";
    case PQ_ERR_TIMEOUT: return "PQ_ERR_TIMEOUT";
  }
  return "PQ_ERR_UNKNOWN";
}

extern "C" const char* pq_last_error(void) { return g_last_error; }

// ParoQuant page §2.2, Algorithm A1, per group (see pq.h for the exact shuffle).
extern "C" pq_status pq_select_pairs(uint64_t seed, int D, int g, int K, int N,
                                     uint8_t* pairs_out) {
  clear_error();
  if (!pairs_out) { set_error("pairs_out is NULL"); return PQ_ERR_INVALID_ARG; }
  if (g != 64 && g != 128) { set_error("g=%d: Givens pairs are drawn for g = 64 or 128", g); return PQ_ERR_UNSUPPORTED; }
  if (D < g || D % g != 0) { set_error("D=%d must be a positive multiple of g", D); return PQ_ERR_INVALID_ARG; }
  if (K < 1 || K > 64) { set_error("K=%d out of range 1..64", K); return PQ_ERR_INVALID_ARG; }
  if (N < 1 || N > g / 2) { set_error("N=%d out of range 1..g/2", N); return PQ_ERR_INVALID_ARG; }
  const int G = D / g, half = g / 2;
  std::vector<uint16_t> cand;           // i << 8 | j
  cand.reserve(g * (g - 1) / 2);
  std::vector<uint8_t> avail(g * g), local(g * g);
  SplitMix64 rng(seed);
  std::memset(pairs_out, PQ_NO_PAIR, (size_t)G * K * half * 2);
  for (int gi = 0; gi < G; ++gi) {
    cand.clear();
    for (int i = 0; i < g; ++i)
      for (int j = i + 1; j < g; ++j) cand.push_back((uint16_t)(i << 8 | j));
    for (size_t i = cand.size() - 1; i >= 1; --i) {
      size_t k = (size_t)(rng.next() % (uint64_t)(i + 1));
      uint16_t t = cand[i]; cand[i] = cand[k]; cand[k] = t;
    }
    for (int i = 0; i < g; ++i)
      for (int j = 0; j < g; ++j) avail[i * g + j] = (i != j);
    for (int l = 0; l < K; ++l) {
      local = avail;
      int n = 0;
      uint8_t* dst = pairs_out + ((size_t)(gi * K + l) * half) * 2;
      for (uint16_t c : cand) {
        if (n >= N) break;
        int i = c >> 8, j = c & 0xFF;
        if (!local[i * g + j]) continue;
        dst[2 * n] = (uint8_t)i;
        dst[2 * n + 1] = (uint8_t)j;
        ++n;
        for (int k = 0; k < g; ++k) {
          local[i * g + k] = local[k * g + i] = 0;
          local[j * g + k] = local[k * g + j] = 0;
        }
        avail[i * g + j] = avail[j * g + i] = 0;
      }
    }
  }
  return PQ_OK;
}

static void free_plan_tables(pq_plan* p) {
  if (!p) return;
  if (p->d_rot) cudaFree(p->d_rot);
  if (p->d_status) cudaFree(p->d_status);
  if (p->d_slot8) cudaFree(p->d_slot8);
}

template <class T>
static pq_status upload(T** dst, const T* src, size_t n, const char* what) {
  cudaError_t e = cudaMalloc((void**)dst, n * sizeof(T));
  if (e != cudaSuccess) {
    *dst = nullptr;
    set_error("cudaMalloc(%s, %zu bytes): %s", what, n * sizeof(T), cudaGetErrorString(e));
    return PQ_ERR_ALLOC;
  }
  if (src) {
    e = cudaMemcpy(*dst, src, n * sizeof(T), cudaMemcpyHostToDevice);
  } else {
    e = cudaMemset(*dst, 0, n * sizeof(T));
  }
  return cuda_fail(e, what);
}

// bf16 bit pattern of a float, round to nearest even (finite inputs).
static uint16_t bf16_bits(float f) {
  uint32_t b;
  std::memcpy(&b, &f, 4);
  return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

static float bf16_value(uint16_t h) {
  const uint32_t b = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &b, 4);
  return f;
}

// Givens, tensor-core operands.  Per group of g channels, R = G_0 G_1 ... G_{K-1} in float64
// for the row-vector convention y = x R: layer l's pair (i, j, theta) replaces columns (i, j) of
// R by (c col_i - s col_j, s col_i + c col_j).  Column n is then scaled by exp(-beta_n) for the
// activations and exp(+beta_n) for the weights (R diag(exp(beta)) = M^-T, the rotations being
// orthogonal).  The kernels take one 128 x 128 matrix per 128-channel tile: the group's R for
// g = 128, the two groups' matrices on the diagonal for g = 64.  Stored transposed (entry
// [n][k] = R[k][n]) as bf16 R_hi + R_lo, laid out [activations / weights][tile][term][n][k].
static void build_rotation_operands(int D, int g, int K, const uint8_t* pairs, const float* angles, const float* beta,
                                    std::vector<uint16_t>& out) {
  constexpr int TW = 128;
  const int G = D / g, tiles = D / TW, half = g / 2;
  out.assign((size_t)2 * tiles * 2 * TW * TW, 0);
  std::vector<double> R((size_t)g * g);
  for (int gi = 0; gi < G; ++gi) {
    std::fill(R.begin(), R.end(), 0.0);
    for (int k = 0; k < g; ++k) R[(size_t)k * g + k] = 1.0;
    for (int l = 0; l < K; ++l) {
      for (int p = 0; p < half; ++p) {
        const size_t slot = (size_t)(gi * K + l) * half + p;
        const int i = pairs[2 * slot], j = pairs[2 * slot + 1];
        if (i == PQ_NO_PAIR || j == PQ_NO_PAIR) continue;
        const double c = std::cos((double)angles[slot]), s = std::sin((double)angles[slot]);
        for (int r = 0; r < g; ++r) {
          const double ri = R[(size_t)r * g + i], rj = R[(size_t)r * g + j];
          R[(size_t)r * g + i] = c * ri - s * rj;
          R[(size_t)r * g + j] = s * ri + c * rj;
        }
      }
    }
    const int ti = gi * g / TW, off = gi * g % TW;   // tile and the group's offset on its diagonal
    for (int which = 0; which < 2; ++which) {
      uint16_t* hi = out.data() + ((size_t)(which * tiles + ti) * 2 + 0) * TW * TW;
      uint16_t* lo = out.data() + ((size_t)(which * tiles + ti) * 2 + 1) * TW * TW;
      for (int n = 0; n < g; ++n) {
        const double cs = beta ? std::exp((which == 0 ? -1.0 : 1.0) * (double)beta[gi * g + n]) : 1.0;
        for (int k = 0; k < g; ++k) {
          const double v = R[(size_t)k * g + n] * cs;
          const uint16_t h = bf16_bits((float)v);
          hi[(size_t)(off + n) * TW + off + k] = h;
          lo[(size_t)(off + n) * TW + off + k] = bf16_bits((float)(v - (double)bf16_value(h)));
        }
      }
    }
  }
}

static pq_status make_plan(pq_plan** out, pq_kind kind, int D, int g, int K, const uint8_t* pairs,
                           const float* angles, const float* beta, uint32_t flags, int n8, const int32_t* groups8) {
  if (!out) { set_error("out is NULL"); return PQ_ERR_INVALID_ARG; }
  if (kind != PQ_HADAMARD && kind != PQ_GIVENS && kind != PQ_SMOOTH_HADAMARD) {
    set_error("unknown kind %d", (int)kind);
    return PQ_ERR_INVALID_ARG;
  }
  // Group sizes: 128 everywhere; 64 for Givens and Hadamard; 256 for Hadamard (its uint8 pair
  // slots and the 128 x 128 tensor-core tiles bound the Givens groups to 128 channels).
  const bool g_ok = g == kGroup || (g == 64 && kind != PQ_SMOOTH_HADAMARD) || (g == 256 && kind == PQ_HADAMARD);
  if (!g_ok) {
    set_error("g=%d is not supported for this plan kind (Hadamard: 64, 128, 256; Givens: 64, 128; smoothing: 128)", g);
    return PQ_ERR_UNSUPPORTED;
  }
  if (D < 128 || D % 128 != 0 || D % g != 0) {
    set_error("D=%d must be a positive multiple of 128 and of g=%d", D, g);
    return PQ_ERR_INVALID_ARG;
  }
  if (flags & ~PQ_FLAG_SMOOTH_AFTER_ROTATE) { set_error("unknown flags 0x%x", flags); return PQ_ERR_INVALID_ARG; }
  if ((flags & PQ_FLAG_SMOOTH_AFTER_ROTATE) && kind != PQ_SMOOTH_HADAMARD) {
    set_error("PQ_FLAG_SMOOTH_AFTER_ROTATE needs PQ_SMOOTH_HADAMARD");
    return PQ_ERR_INVALID_ARG;
  }
  const int G = D / g, half = g / 2;
  // 8-bit outlier groups (ParoQuant page §4.1): distinct group indices, rotation plans at g = 128.
  std::vector<int16_t> slot8;
  if (n8 != 0) {
    if (n8 < 0 || n8 > G || !groups8) { set_error("n8=%d: 0..G groups and a group list are needed", n8); return PQ_ERR_INVALID_ARG; }
    if ((kind != PQ_HADAMARD && kind != PQ_GIVENS) || g != kGroup) {
      set_error("8-bit outlier groups need a PQ_HADAMARD or PQ_GIVENS plan with g = 128");
      return PQ_ERR_UNSUPPORTED;
    }
    slot8.assign(G, -1);
    for (int j = 0; j < n8; ++j) {
      const int32_t gi = groups8[j];
      if (gi < 0 || gi >= G || slot8[gi] >= 0) {
        set_error("groups8[%d]=%d must be distinct group indices below G=%d", j, gi, G);
        return PQ_ERR_INVALID_ARG;
      }
      slot8[gi] = (int16_t)j;
    }
  }
  if (kind == PQ_GIVENS) {
    if (K < 1 || K > 64) { set_error("K=%d out of range 1..64", K); return PQ_ERR_INVALID_ARG; }
    if (!pairs || !angles) { set_error("Givens plan needs pairs and angles"); return PQ_ERR_INVALID_ARG; }
    std::vector<uint8_t> seen(g);
    for (int gi = 0; gi < G; ++gi) {
      for (int l = 0; l < K; ++l) {
        std::fill(seen.begin(), seen.end(), 0);
        for (int p = 0; p < half; ++p) {
          size_t slot = (size_t)(gi * K + l) * half + p;
          uint8_t i = pairs[2 * slot], j = pairs[2 * slot + 1];
          if (i == PQ_NO_PAIR || j == PQ_NO_PAIR) continue;
          if (!(i < j && j < g)) {
            set_error("group %d layer %d slot %d: pair (%d,%d) must satisfy i<j<%d", gi, l, p, i, j, g);
            return PQ_ERR_INVALID_ARG;
          }
          if (seen[i] || seen[j]) {
            set_error("group %d layer %d: channel used twice (pairs must be disjoint)", gi, l);
            return PQ_ERR_INVALID_ARG;
          }
          seen[i] = seen[j] = 1;
          if (!std::isfinite(angles[slot])) { set_error("non-finite angle at slot %zu", slot); return PQ_ERR_INVALID_ARG; }
        }
      }
    }
    if (beta) {
      for (int c = 0; c < D; ++c)
        if (!std::isfinite(beta[c])) { set_error("non-finite beta[%d]", c); return PQ_ERR_INVALID_ARG; }
    }
  } else {
    K = 0;
  }
  pq_plan* p = new (std::nothrow) pq_plan();
  if (!p) { set_error("host allocation failed"); return PQ_ERR_ALLOC; }
  *p = pq_plan{};
  p->kind = kind;
  p->D = D;
  p->g = g;
  p->G = G;
  p->K = K;
  p->flags = flags;
  pq_status st = cuda_fail(cudaGetDevice(&p->device), "cudaGetDevice");
  if (st == PQ_OK && kind == PQ_GIVENS) {
    std::vector<uint16_t> rot;
    build_rotation_operands(D, g, K, pairs, angles, beta, rot);
    st = upload(&p->d_rot, rot.data(), rot.size(), "givens tensor-core operands");
  }
  if (st == PQ_OK && kind == PQ_HADAMARD) {
    // Unnormalised Sylvester H_b: entry (k, n) = (-1)^popcount(k & n) (Hadamard page §2.1),
    // symmetric, so [n][k] = [k][n]; +-1 in bf16 is 0x3F80 / 0xBF80, 0 is 0.  g = 128: H_128;
    // g = 64: diag(H_64, H_64) (zero where k and n lie in different halves); g = 256: H_128 then
    // -H_128 (H_256 = [[H, H], [H, -H]] is applied as products with these two).
    constexpr int TW = 128;
    const int mats = g == 256 ? 2 : 1;
    std::vector<uint16_t> h((size_t)mats * TW * TW);
    for (int m = 0; m < mats; ++m)
      for (int k = 0; k < TW; ++k)
        for (int n = 0; n < TW; ++n) {
          uint16_t v;
          if (g == 64 && ((k ^ n) & 64)) v = 0;
          else v = ((__builtin_popcount(k & n & (g == 64 ? 63 : 127)) + m) & 1) ? 0xBF80 : 0x3F80;
          h[((size_t)m * TW + n) * TW + k] = v;
        }
    st = upload(&p->d_rot, h.data(), h.size(), "hadamard tensor-core operand");
  }
  if (st == PQ_OK) st = upload<unsigned int>(&p->d_status, nullptr, 1, "status word");
  p->n8 = n8;
  p->Gx = G + 3 * n8;
  if (st == PQ_OK && n8 > 0) st = upload(&p->d_slot8, slot8.data(), slot8.size(), "8-bit group slots");
  if (st != PQ_OK) {
    free_plan_tables(p);
    delete p;
    return st;
  }
  *out = p;
  return PQ_OK;
}

extern "C" pq_status pq_make_plan(pq_plan** out, pq_kind kind, int D, int g, int K,
                                  const uint8_t* pairs, const float* angles, const float* beta,
                                  uint32_t flags) {
  clear_error();
  return make_plan(out, kind, D, g, K, pairs, angles, beta, flags, 0, nullptr);
}

extern "C" pq_status pq_make_plan_outliers(pq_plan** out, pq_kind kind, int D, int g, int K,
                                           const uint8_t* pairs, const float* angles, const float* beta,
                                           uint32_t flags, int n8, const int32_t* groups8) {
  clear_error();
  return make_plan(out, kind, D, g, K, pairs, angles, beta, flags, n8, groups8);
}

extern "C" void pq_destroy_plan(pq_plan* plan) {
  if (!plan) return;
  free_plan_tables(plan);
  delete plan;
}

static pq_status check_plan(const pq_plan* plan) {
  if (!plan) { set_error("plan is NULL"); return PQ_ERR_INVALID_ARG; }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) {
    set_error("plan was created on device %d, current device is %d", plan->device, dev);
    return PQ_ERR_INVALID_ARG;
  }
  return PQ_OK;
}

namespace {

// Argument checks of the activation transform; nothing here touches the device.
pq_status check_transform_args(const pq_plan* plan, const void* X, int64_t T, int64_t ldx, const uint8_t* codes,
                               const float* scales, const float* smooth_out) {
  if (!plan) { set_error("plan is NULL"); return PQ_ERR_INVALID_ARG; }
  if (!X || !codes || !scales) { set_error("X, codes and scales must be non-NULL"); return PQ_ERR_INVALID_ARG; }
  if (T < 1) { set_error("T=%lld must be >= 1", (long long)T); return PQ_ERR_INVALID_ARG; }
  if (ldx < plan->D || ldx % 8 != 0) {
    set_error("ldx=%lld must be >= D=%d and a multiple of 8", (long long)ldx, plan->D);
    return PQ_ERR_INVALID_ARG;
  }
  if (!aligned16(X) || !aligned16(codes) || !aligned16(scales) ||
      (smooth_out && !aligned16(smooth_out))) {
    set_error("device pointers must be 16-byte aligned");
    return PQ_ERR_INVALID_ARG;
  }
  if (smooth_out && plan->kind != PQ_SMOOTH_HADAMARD) {
    set_error("smooth_out must be NULL for this plan kind");
    return PQ_ERR_INVALID_ARG;
  }
  if (T >= ((int64_t)1 << 31)) { set_error("T=%lld must be < 2^31", (long long)T); return PQ_ERR_INVALID_ARG; }
  return PQ_OK;
}

cudaError_t launch_transform(const pq_plan* plan, const void* X, int64_t T, int64_t ldx, uint8_t* codes,
                             float* scales, float* smooth_out, cudaStream_t s) {
  switch (plan->kind) {
    case PQ_HADAMARD:
    case PQ_GIVENS:
      if (rows_small_applies(plan, T)) return launch_rows_small(plan, X, T, ldx, codes, scales, s);
      return launch_rotate_mma(plan, X, T, ldx, 0, codes, scales, s);
    case PQ_SMOOTH_HADAMARD:
      if (plan->flags & PQ_FLAG_SMOOTH_AFTER_ROTATE)
        return launch_smooth_hadamard(plan, X, T, ldx, codes, scales, smooth_out, s);
      return launch_smooth_rows(plan, X, T, ldx, PQ_SR_COLMAX, nullptr, codes, scales, smooth_out, s);
  }
  return cudaErrorInvalidValue;
}

struct TransformCall {
  const pq_plan* plan;
  const void* X;
  int64_t T, ldx;
  uint8_t* codes;
  float* scales;
  cudaStream_t stream;
};

cudaError_t transform_thunk(const void* ctx) {
  const TransformCall& c = *static_cast<const TransformCall*>(ctx);
  return launch_transform(c.plan, c.X, c.T, c.ldx, c.codes, c.scales, nullptr, c.stream);
}

}  // namespace

extern "C" pq_status pq_transform_quant(const pq_plan* plan, const void* X, int64_t T,
                                        int64_t ldx, uint8_t* codes, float* scales,
                                        float* smooth_out, void* stream) {
  clear_error();
  pq_status st = check_transform_args(plan, X, T, ldx, codes, scales, smooth_out);
  if (st != PQ_OK) return st;
  st = check_plan(plan);
  if (st != PQ_OK) return st;
  return cuda_fail(launch_transform(plan, X, T, ldx, codes, scales, smooth_out, reinterpret_cast<cudaStream_t>(stream)),
                   "pq_transform_quant launch");
}

extern "C" pq_status pq_pack_weights(const pq_plan* plan, const void* W, int64_t N,
                                     const float* smooth_w, uint8_t* codes_W, float* scales_W,
                                     void* stream) {
  clear_error();
  if (!plan) { set_error("plan is NULL"); return PQ_ERR_INVALID_ARG; }
  if (!W || !codes_W || !scales_W) { set_error("W, codes_W and scales_W must be non-NULL"); return PQ_ERR_INVALID_ARG; }
  if (N < 1 || N >= ((int64_t)1 << 31)) { set_error("N=%lld must be in [1, 2^31)", (long long)N); return PQ_ERR_INVALID_ARG; }
  if (!aligned16(W) || !aligned16(codes_W) || !aligned16(scales_W) ||
      (smooth_w && !aligned16(smooth_w))) {
    set_error("device pointers must be 16-byte aligned");
    return PQ_ERR_INVALID_ARG;
  }
  if (smooth_w && plan->kind != PQ_SMOOTH_HADAMARD) {
    set_error("smooth_w must be NULL for this plan kind");
    return PQ_ERR_INVALID_ARG;
  }
  pq_status st = check_plan(plan);
  if (st != PQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  switch (plan->kind) {
    case PQ_HADAMARD:
      e = launch_rotate_mma(plan, W, N, plan->D, 1, codes_W, scales_W, s);
      break;
    case PQ_GIVENS:
      e = launch_rotate_mma(plan, W, N, plan->D, 1, codes_W, scales_W, s);
      break;
    case PQ_SMOOTH_HADAMARD:
      if (!smooth_w)
        e = launch_smooth_rows(plan, W, N, plan->D, PQ_SR_NONE, nullptr, codes_W, scales_W, nullptr, s);
      else if (plan->flags & PQ_FLAG_SMOOTH_AFTER_ROTATE)
        e = launch_smooth_rows(plan, W, N, plan->D, PQ_SR_POST, smooth_w, codes_W, scales_W, nullptr, s);
      else
        e = launch_smooth_rows(plan, W, N, plan->D, PQ_SR_PRE, smooth_w, codes_W, scales_W, nullptr, s);
      break;
  }
  return cuda_fail(e, "pq_pack_weights launch");
}

namespace {

// Size checks shared by the GEMM entry points and the launch-count query.
pq_status check_gemm_sizes(int64_t T, int64_t N, int64_t D) {
  if (T < 1 || N < 1 || D < kGroup) { set_error("T, N must be >= 1 and D >= 128"); return PQ_ERR_INVALID_ARG; }
  if (D % kGroup != 0) { set_error("D=%lld must be a multiple of 128", (long long)D); return PQ_ERR_INVALID_ARG; }
  if (N % 16 != 0) { set_error("N=%lld must be a multiple of 16", (long long)N); return PQ_ERR_INVALID_ARG; }
  if (T >= ((int64_t)1 << 31) || N >= ((int64_t)1 << 31) || D >= ((int64_t)1 << 24)) {
    set_error("T, N must be < 2^31 and D < 2^24");
    return PQ_ERR_INVALID_ARG;
  }
  return PQ_OK;
}

// Argument checks shared by the GEMM entry points; nothing here touches the device.
pq_status check_gemm_args(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W,
                          const float* scales_W, int64_t T, int64_t N, int64_t D, int g, void* Y,
                          pq_out_dtype out_dtype) {
  if (!codes_A || !scales_A || !codes_W || !scales_W || !Y) {
    set_error("all tensor pointers must be non-NULL");
    return PQ_ERR_INVALID_ARG;
  }
  if (g != 64 && g != 128 && g != 256) { set_error("g=%d: the GEMM supports g = 64, 128, 256", g); return PQ_ERR_UNSUPPORTED; }
  pq_status st = check_gemm_sizes(T, N, D);
  if (st != PQ_OK) return st;
  if (D % g != 0) { set_error("D=%lld must be a multiple of g=%d", (long long)D, g); return PQ_ERR_INVALID_ARG; }
  if (out_dtype != PQ_OUT_F32 && out_dtype != PQ_OUT_BF16) { set_error("bad out_dtype"); return PQ_ERR_INVALID_ARG; }
  if (!aligned16(codes_A) || !aligned16(scales_A) || !aligned16(codes_W) ||
      !aligned16(scales_W) || !aligned16(Y)) {
    set_error("device pointers must be 16-byte aligned");
    return PQ_ERR_INVALID_ARG;
  }
  return PQ_OK;
}

}  // namespace

extern "C" pq_status pq_w4a4_gemm(const uint8_t* codes_A, const float* scales_A,
                                  const uint8_t* codes_W, const float* scales_W, int64_t T,
                                  int64_t N, int64_t D, int g, void* Y, pq_out_dtype out_dtype,
                                  void* stream) {
  clear_error();
  pq_status st = check_gemm_args(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype);
  if (st != PQ_OK) return st;
  return gemm_run(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype,
                  reinterpret_cast<cudaStream_t>(stream));
}

extern "C" pq_status pq_w4a4_gemm_noalloc(const uint8_t* codes_A, const float* scales_A,
                                          const uint8_t* codes_W, const float* scales_W,
                                          int64_t T, int64_t N, int64_t D, int g, void* Y,
                                          pq_out_dtype out_dtype, void* stream) {
  clear_error();
  pq_status st = check_gemm_args(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype);
  if (st != PQ_OK) return st;
  return gemm_run_static_scratch(codes_A, scales_A, codes_W, scales_W, T, N, D, g, Y, out_dtype,
                                 reinterpret_cast<cudaStream_t>(stream));
}


extern "C" pq_status pq_w4a4_linear(const pq_plan* plan, const void* X, int64_t T, int64_t ldx, uint8_t* codes_A,
                                    float* scales_A, const uint8_t* codes_W, const float* scales_W, int64_t N,
                                    void* Y, pq_out_dtype out_dtype, void* stream) {
  clear_error();
  pq_status st = check_transform_args(plan, X, T, ldx, codes_A, scales_A, nullptr);
  if (st != PQ_OK) return st;
  // The GEMM's reduction length: D, or with 8-bit groups the Gx groups of their digit layout.
  const int64_t Dk = (int64_t)plan->Gx * plan->g;
  st = check_gemm_args(codes_A, scales_A, codes_W, scales_W, T, N, Dk, plan->g, Y, out_dtype);
  if (st != PQ_OK) return st;
  st = check_plan(plan);
  if (st != PQ_OK) return st;
  const TransformCall call{plan, X, T, ldx, codes_A, scales_A, reinterpret_cast<cudaStream_t>(stream)};
  return gemm_run_linear(&transform_thunk, &call, codes_A, scales_A, codes_W, scales_W, T, N, Dk, plan->g, Y,
                         out_dtype, reinterpret_cast<cudaStream_t>(stream));
}

// --------------------------------------- rotated runtime smoothing (RRS page, Fig. 4)
namespace {

pq_status check_rrs_plan(const pq_plan* plan) {
  if (!plan) { set_error("plan is NULL"); return PQ_ERR_INVALID_ARG; }
  if (plan->kind != PQ_HADAMARD || plan->g != kGroup || plan->n8 != 0) {
    set_error("rotated runtime smoothing needs a PQ_HADAMARD plan with g = 128 (no 8-bit groups)");
    return PQ_ERR_UNSUPPORTED;
  }
  if (plan->D > 16384 || rrs_rows_smem_bytes(plan->D) > 232448) {
    set_error("D=%d: rotated runtime smoothing supports D <= 16384", plan->D);
    return PQ_ERR_UNSUPPORTED;
  }
  return check_plan(plan);
}

pq_status check_rows_arg(const void* X, int64_t rows, int64_t ldx, int D, const char* what) {
  if (!X) { set_error("%s is NULL", what); return PQ_ERR_INVALID_ARG; }
  if (rows < 1 || rows >= ((int64_t)1 << 31)) { set_error("%s: rows=%lld out of range", what, (long long)rows); return PQ_ERR_INVALID_ARG; }
  if (ldx < D || ldx % 8 != 0) { set_error("ldx=%lld must be >= D=%d and a multiple of 8", (long long)ldx, D); return PQ_ERR_INVALID_ARG; }
  if (!aligned16(X)) { set_error("device pointers must be 16-byte aligned"); return PQ_ERR_INVALID_ARG; }
  return PQ_OK;
}

}  // namespace

extern "C" pq_status pq_rrs_prepare(const pq_plan* plan, const void* X, int64_t T, int64_t ldx, float* chan_max,
                                    int32_t* perm, int32_t* inv_perm, float* group_scale, void* stream) {
  clear_error();
  pq_status st = check_rrs_plan(plan);
  if (st != PQ_OK) return st;
  st = check_rows_arg(X, T, ldx, plan->D, "X");
  if (st != PQ_OK) return st;
  if (!chan_max || !perm || !inv_perm || !group_scale || !aligned16(chan_max) || !aligned16(perm) ||
      !aligned16(inv_perm) || !aligned16(group_scale)) {
    set_error("chan_max, perm, inv_perm and group_scale must be non-NULL and 16-byte aligned");
    return PQ_ERR_INVALID_ARG;
  }
  return cuda_fail(launch_rrs_prepare(plan, X, T, ldx, chan_max, perm, inv_perm, group_scale,
                                      reinterpret_cast<cudaStream_t>(stream)),
                   "pq_rrs_prepare launch");
}

extern "C" pq_status pq_rrs_transform_quant(const pq_plan* plan, const void* X, int64_t T, int64_t ldx,
                                            const int32_t* perm, const float* group_scale, uint8_t* codes,
                                            float* token_scales, void* stream) {
  clear_error();
  pq_status st = check_rrs_plan(plan);
  if (st != PQ_OK) return st;
  st = check_rows_arg(X, T, ldx, plan->D, "X");
  if (st != PQ_OK) return st;
  if (!perm || !group_scale || !codes || !token_scales || !aligned16(perm) || !aligned16(group_scale) ||
      !aligned16(codes) || !aligned16(token_scales)) {
    set_error("perm, group_scale, codes and token_scales must be non-NULL and 16-byte aligned");
    return PQ_ERR_INVALID_ARG;
  }
  return cuda_fail(launch_rrs_rows(plan, X, T, ldx, 0, perm, group_scale, codes, token_scales,
                                   reinterpret_cast<cudaStream_t>(stream)),
                   "pq_rrs_transform_quant launch");
}

extern "C" pq_status pq_rrs_pack_weights(const pq_plan* plan, const void* W, int64_t N, const int32_t* perm,
                                         const float* group_scale, uint8_t* codes_W, float* scales_W,
                                         void* stream) {
  clear_error();
  pq_status st = check_rrs_plan(plan);
  if (st != PQ_OK) return st;
  st = check_rows_arg(W, N, plan->D, plan->D, "W");
  if (st != PQ_OK) return st;
  if (!perm || !group_scale || !codes_W || !scales_W || !aligned16(perm) || !aligned16(group_scale) ||
      !aligned16(codes_W) || !aligned16(scales_W)) {
    set_error("perm, group_scale, codes_W and scales_W must be non-NULL and 16-byte aligned");
    return PQ_ERR_INVALID_ARG;
  }
  return cuda_fail(launch_rrs_rows(plan, W, N, plan->D, 1, perm, group_scale, codes_W, scales_W,
                                   reinterpret_cast<cudaStream_t>(stream)),
                   "pq_rrs_pack_weights launch");
}

extern "C" pq_status pq_rrs_gemm(const uint8_t* codes_A, const float* token_scales, const uint8_t* codes_W,
                                 const float* scales_W, int64_t T, int64_t N, int64_t D, int g, void* Y,
                                 pq_out_dtype out_dtype, void* stream) {
  clear_error();
  pq_status st = check_gemm_args(codes_A, token_scales, codes_W, scales_W, T, N, D, g, Y, out_dtype);
  if (st != PQ_OK) return st;
  if (g != kGroup) { set_error("g=%d: rotated runtime smoothing uses g = 128", g); return PQ_ERR_UNSUPPORTED; }
  return gemm_run(codes_A, token_scales, codes_W, scales_W, T, N, D, g, Y, out_dtype,
                  reinterpret_cast<cudaStream_t>(stream), /*row_scale=*/true);
}

extern "C" pq_status pq_w4a4_gemm_launch_count_g(int64_t T, int64_t N, int64_t D, int g, int* launches) {
  clear_error();
  if (!launches) {
    set_error("launches must be non-NULL");
    return PQ_ERR_INVALID_ARG;
  }
  if (g != 64 && g != 128 && g != 256) { set_error("g=%d: the GEMM supports g = 64, 128, 256", g); return PQ_ERR_UNSUPPORTED; }
  pq_status st = check_gemm_sizes(T, N, D);
  if (st != PQ_OK) return st;
  if (D % g != 0) { set_error("D=%lld must be a multiple of g=%d", (long long)D, g); return PQ_ERR_INVALID_ARG; }
  const int split = gemm_ksplit(T, N, D, g, nullptr) > 1 ? 1 : 0;
  *launches = (T <= kGemmSmallT ? 1 : 2) + split;
  return PQ_OK;
}

extern "C" pq_status pq_w4a4_gemm_launch_count(int64_t T, int64_t N, int64_t D, int* launches) {
  return pq_w4a4_gemm_launch_count_g(T, N, D, kGroup, launches);
}

extern "C" pq_status pq_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  clear_error();
  if (limit_ns < 1000 || limit_ns > 100000000) {
    set_error("limit_ns=%llu must be within [1 us, 100 ms]", (unsigned long long)limit_ns);
    return PQ_ERR_INVALID_ARG;
  }
  return gemm_wait_timeout_selftest(limit_ns, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" pq_status pq_check_status(const pq_plan* plan, void* stream) {
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  pq_status st = cuda_fail(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  if (st != PQ_OK) return st;
  unsigned int bits = 0;
  if (plan && plan->d_status) {
    unsigned int pb = 0;
    st = cuda_fail(cudaMemcpy(&pb, plan->d_status, sizeof(pb), cudaMemcpyDeviceToHost), "read plan status");
    if (st != PQ_OK) return st;
    if (pb) {
      st = cuda_fail(cudaMemset(plan->d_status, 0, sizeof(pb)), "clear plan status");
      if (st != PQ_OK) return st;
    }
    bits |= pb;
  }
  unsigned int gb = 0;
  st = gemm_read_and_clear_status(&gb);
  if (st != PQ_OK) return st;
  bits |= gb;
  if (bits & PQ_DEV_TIMEOUT) {
    set_error("a device-side bounded wait timed out (status bits 0x%x)", bits);
    return PQ_ERR_TIMEOUT;
  }
  return PQ_OK;
}
