/*
 * pq.h — C ABI of libpq: online rotation + INT4 quantisation of bf16 activations and the
 * W4A4 GEMM that consumes the codes, for NVIDIA B200 (sm_100a).
 *
 * Sources (pages, by title and section):
 *   ParoQuant page — codearts.csdn.net article on independent rotation and channel scaling:
 *       §2.2 (Algorithm A1, greedy disjoint channel pairs per 128-channel group; the three
 *       properties listed under it), §2.3 (W^ = diag(alpha) W with alpha = exp(beta); 128
 *       channels share the quantisation parameters), §3.2 (rotation, scaling and quantisation
 *       fused in one kernel; only the angles are stored), §6.4 (cloud: tensor cores).
 *   Hadamard page — "神经网络量化技术：Hadamard变换与格码本优化": §2.1 (Walsh–Hadamard matrix,
 *       entries (-1)^popcount(i&j), 1/sqrt(n)), §4.2 (butterflies; H(AB) = (HA)B), §6.1 (block
 *       Hadamard).
 *   RRS page — "Rotated Runtime Smooth: 训练无关的激活平滑器，用于精确的 INT4 推理": main equation
 *       (X_rot = XR, W_rot = R^-1 W, s_j = max|(X_rot)_j|, Quantize(X_rot diag(s)^-1),
 *       Y = sum_j (X'_q)_j (W'_q)_j^T s_j), R = (1/sqrt(K))[s_ij], alpha = max|X|/(2^(N-1)-1),
 *       the INT4 range -8..7, RTN rounding, Fig. 2(a) (Y = (XR)(R^-1 W^T) = XW^T) and Fig. 4
 *       (scales applied to the interim block results inside the GEMM).
 *
 * Conventions
 *   X  bf16 [T][D] row-major, row stride ldx elements (activations, one row per token).
 *   W  bf16 [N][D] row-major (Y = X W^T).
 *   g  group size: 128, 64 (Hadamard, Givens) or 256 (Hadamard); G = D / g groups per row.
 *   codes  uint8 [rows][D/2]: byte k holds element 2k in the low nibble and element 2k+1 in
 *          the high nibble, both two's complement in -8..7.
 *   scales float32 [rows][G]: per-group scale m/7, m = max |transformed value| in the group
 *          (0 for an all-zero group, whose codes are 0).
 *   Codes are q = round_half_even(y / scale) computed in float32 (|q| <= 7).
 *
 * Ownership and memory
 *   Every tensor pointer is a DEVICE pointer owned by the caller, on the current device,
 *   16-byte aligned.  The library allocates no user-visible buffer.  A plan owns a few small
 *   device tables and a status word, allocated by pq_make_plan and freed by pq_destroy_plan;
 *   it is immutable after creation and may be used from several streams at once.
 *   pq_w4a4_gemm takes (T + N) * D bytes (T > 128; more when split, see there) of temporary
 *   scratch per call from a library-owned, stream-ordered memory pool on the current device and
 *   returns it on the same stream; the pool keeps freed memory for reuse, so it holds about the
 *   largest single call's need.  Calls with T <= 128 take none unless they split.
 *
 * Errors
 *   Every call returns pq_status and never throws, aborts or exits.  Arguments are validated
 *   before anything is launched; a failed call launches nothing and pq_last_error() (thread
 *   local) describes why.  Launches are asynchronous on the given stream (NULL = legacy default
 *   stream); device-side faults surface at the caller's next synchronisation, and bounded-wait
 *   timeouts inside the GEMM are reported by pq_check_status.
 */
#ifndef PQ_H_
#define PQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pq_status {
  PQ_OK = 0,
  PQ_ERR_INVALID_ARG = 1,   /* bad pointer, size, stride, alignment or plan */
  PQ_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. a group size a kind lacks) */
  PQ_ERR_CUDA = 3,          /* a CUDA runtime call failed (message in pq_last_error) */
  PQ_ERR_ALLOC = 4,         /* a device allocation (plan tables, GEMM scratch) failed */
  PQ_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up (see pq_check_status) */
} pq_status;

typedef enum pq_kind {
  PQ_HADAMARD = 0,          /* block Walsh–Hadamard H_g / sqrt(g) per group */
  PQ_GIVENS = 1,            /* K layers of disjoint Givens pairs per group, then exp(-beta) */
  PQ_SMOOTH_HADAMARD = 2    /* runtime per-channel smoothing per 128-token block + Hadamard */
} pq_kind;

typedef enum pq_out_dtype {
  PQ_OUT_F32 = 0,
  PQ_OUT_BF16 = 1           /* round-to-nearest-even of the float32 result */
} pq_out_dtype;

/* pq_make_plan flags */
#define PQ_FLAG_SMOOTH_AFTER_ROTATE 0x1u  /* PQ_SMOOTH_HADAMARD: rotate first, then smooth the
                                             rotated channels (the RRS page's order).  Default:
                                             smooth the input channels, then rotate. */

/* Pair-slot marker for "no pair" in pair tables. */
#define PQ_NO_PAIR 0xFFu

typedef struct pq_plan pq_plan;

/*
 * pq_select_pairs — ParoQuant page §2.2, Algorithm A1, run once per group (host only, no GPU).
 *   For each group independently: all pairs (i, j), 0 <= i < j < g, in lexicographic order,
 *   Fisher–Yates shuffled (for i = n-1..1: swap a[i], a[r mod (i+1)], r = next SplitMix64
 *   output; one SplitMix64 stream seeded with `seed` serves the groups in order 0..G-1).
 *   Then K layers: scan the shuffled list, take a pair when both channels are still free in
 *   this layer and the pair was not taken by an earlier layer; stop a layer at N pairs.
 *   pairs_out: host uint8 [D/g][K][g/2][2], caller-owned; slots past a layer's last pair are
 *   PQ_NO_PAIR.  Requires g = 64 or 128, D % g = 0, 1 <= K <= 64, 1 <= N <= g/2.
 */
pq_status pq_select_pairs(uint64_t seed, int D, int g, int K, int N, uint8_t* pairs_out);

/*
 * pq_make_plan — build the device tables for one transform.
 *   kind    PQ_HADAMARD | PQ_GIVENS | PQ_SMOOTH_HADAMARD.
 *   D, g    channels and group size: D % 128 == 0, D % g == 0, and g = 128 for every kind,
 *           64 for PQ_HADAMARD and PQ_GIVENS (ParoQuant page §4.1: smaller groups for layers
 *           with many outliers), 256 for PQ_HADAMARD (§6: larger groups on mobile parts);
 *           other combinations return PQ_ERR_UNSUPPORTED.  (Givens at g = 256 would need
 *           256 x 256 matrices, which do not fit the rotation kernel's shared memory.)
 *   K       Givens layers (1..64); ignored otherwise.
 *   pairs   host uint8 [D/g][K][g/2][2] (Givens; NULL otherwise).  Within a layer of a group
 *           the valid pairs (i < j < g) must be disjoint; PQ_NO_PAIR slots are skipped.
 *   angles  host float32 [D/g][K][g/2] (Givens), radians.  Pair (i, j) with angle t maps the
 *           column (x_i, x_j) to (cos t x_i - sin t x_j, sin t x_i + cos t x_j); layer 0 first.
 *   beta    host float32 [D] or NULL (= 0): channel scale alpha = exp(beta) (ParoQuant page
 *           §2.3).  Activations are multiplied by exp(-beta) after the rotations and weights by
 *           exp(+beta), so that the product is unchanged before quantisation.
 *   flags   PQ_FLAG_* bits.
 *   Givens: per group the K layers and exp(-+beta) are composed on the host in double precision
 *   into one g x g matrix (one for activations, one for weights; at g = 64 two groups share a
 *   128 x 128 block-diagonal matrix), stored as a bf16 pair hi + lo (about 2^-17 relative);
 *   the transform is then a tensor-core product y = x R.
 *   The plan is created on the current device.  *out is set only on success.
 */
pq_status pq_make_plan(pq_plan** out, pq_kind kind, int D, int g, int K, const uint8_t* pairs,
                       const float* angles, const float* beta, uint32_t flags);

/*
 * pq_make_plan_outliers — pq_make_plan with 8-bit outlier groups (ParoQuant page §4.1: extreme
 * outliers keep an 8-bit representation).  PQ_HADAMARD or PQ_GIVENS with g = 128 only
 * (PQ_ERR_UNSUPPORTED otherwise).
 *   n8       number of 8-bit groups, 0 <= n8 <= D/g (0: the same plan as pq_make_plan).
 *   groups8  host int32 [n8]: distinct group indices.
 *   In those groups a row's codes are q = RNE(119 y / m) (|q| <= 119), scale s = m / 119 (with the
 *   Hadamard's 1/sqrt(g) folded in as for 4-bit groups).  Each 8-bit code is written as two signed
 *   4-bit digits, q = 16 q_hi + q_lo with q_hi, q_lo in -8..7 (119 is the largest symmetric range
 *   that splits so), and the group as four 4-bit groups of the ordinary layout, so that
 *   pq_w4a4_gemm computes the 8-bit product exactly from 4-bit codes:
 *     codes and scales hold Gx = D/g + 3 n8 groups per row ([T][Gx*g/2] bytes, [T][Gx] floats);
 *     8-bit group gi, the j-th listed, uses its own slot gi and the appended slots G + 3j,
 *     G + 3j + 1, G + 3j + 2 (G = D/g);
 *     activations: digits (hi, hi, lo, lo), scales (16 s, 16 s, s, s);
 *     weights:     digits (hi, lo, hi, lo), scales (16 s, s, 16 s, s);
 *   so the four digit-group products add up to s_a s_w sum(q_a q_w).  Multiply with
 *   pq_w4a4_gemm(..., D = Gx * g, g) (pq_w4a4_linear does this itself).  The plan is otherwise
 *   as from pq_make_plan; rotated runtime smoothing rejects it.
 */
pq_status pq_make_plan_outliers(pq_plan** out, pq_kind kind, int D, int g, int K, const uint8_t* pairs,
                                const float* angles, const float* beta, uint32_t flags, int n8,
                                const int32_t* groups8);

/* pq_destroy_plan — frees the plan's device tables (synchronous).  NULL is a no-op. */
void pq_destroy_plan(pq_plan* plan);

/*
 * pq_transform_quant — the online activation path, one fused kernel (ParoQuant page §3.2;
 * RRS page main equation, first and fourth lines):
 *   y = x M per row, M = H_g/sqrt(g) | R diag(exp(-beta)) | diag(1/s) H_g/sqrt(g) (smoothing
 *   first; or H_g/sqrt(g) diag(1/s) with PQ_FLAG_SMOOTH_AFTER_ROTATE), then per group
 *   scale = max|y|/7 and codes = round(y/scale), nibble-packed.
 *   X          device bf16 [T][ldx] (first D columns used), ldx >= D, ldx % 8 == 0.
 *   T          rows, T >= 1.
 *   codes      device uint8 [T][D/2] (dense).
 *   scales     device float32 [T][D/g] (dense).
 *   smooth_out PQ_SMOOTH_HADAMARD only: device float32 [ceil(T/128)][D] receiving s, the max
 *              |x| (or |rotated x|) of each channel over each 128-row block (0 -> 1); may be
 *              NULL.  Must be NULL for the other kinds.
 *   stream     cudaStream_t or NULL.
 */
pq_status pq_transform_quant(const pq_plan* plan, const void* X, int64_t T, int64_t ldx,
                             uint8_t* codes, float* scales, float* smooth_out, void* stream);

/*
 * pq_pack_weights — the offline weight path: w -> w M^{-T} per row (RRS page: W_rot = R^-1 W;
 * Hadamard page §4.2 H(AB) = (HA)B; OSTQuant page §3.2: the pair is merged into the weights),
 * then the same per-group quantisation and packing as the activations.
 *   Hadamard: same rotation.  Givens: same rotations, then exp(+beta).
 *   Smooth+Hadamard: multiply channel j by smooth_w[j], then rotate (with
 *   PQ_FLAG_SMOOTH_AFTER_ROTATE: rotate, then multiply by smooth_w); smooth_w NULL = ones.
 *   W        device bf16 [N][D] dense.   N >= 1.
 *   smooth_w device float32 [D] or NULL (PQ_SMOOTH_HADAMARD only; must be NULL otherwise).
 *   codes_W  device uint8 [N][D/2];  scales_W device float32 [N][D/g].
 */
pq_status pq_pack_weights(const pq_plan* plan, const void* W, int64_t N, const float* smooth_w,
                          uint8_t* codes_W, float* scales_W, void* stream);

/*
 * pq_w4a4_gemm — Y[t][n] = sum_G scales_A[t][G] * scales_W[n][G] * d_G[t][n], with
 * d_G = sum over the group's g channels of qa * qw, and the per-group scaling applied to
 * each group's interim result in float32, groups summed in ascending order (RRS page main
 * equation, last line, and Fig. 4 step (3) with block size = group size).
 *   How d_G is formed: the int4 codes are widened to E4M3 (every integer -8..7 is exact in
 *   E4M3) and multiplied on the tensor cores by tcgen05.mma kind::f8f6f4 into a float32
 *   accumulator in tensor memory, one accumulator per group.  Every product is an integer of
 *   magnitude <= 64 and every partial sum an integer of magnitude <= 256 * 64 = 2^14, so each
 *   is exact in float32 and d_G arrives exact (no int32 accumulator is involved).
 *   codes_A [T][D/2], scales_A [T][D/g], codes_W [N][D/2], scales_W [N][D/g]: device, dense.
 *   T >= 1, N >= 1 with N % 16 == 0, D % 128 == 0, g in {64, 128, 256} with D % g == 0
 *   (PQ_ERR_UNSUPPORTED for another g).  A group is g / 32 tensor-core K32 steps into its own
 *   accumulator: two groups per 128-code K-block at g = 64, two K-blocks per group at g = 256.
 *   Y device [T][N] float32 (PQ_OUT_F32) or bf16 (PQ_OUT_BF16, RNE of the float32 result).
 *   Scales must be finite.
 *   Returns PQ_ERR_ALLOC if the stream-ordered scratch cannot be allocated.
 *   T > 128: the codes are first widened to E4M3 into (T + N) * D bytes of scratch; output
 *   tiles are 256 channels x 256 tokens, one per pair of SMs.  Few tiles (at most half the SM
 *   pairs): the groups are split into ranges of a multiple of 4 handled by different SM pairs,
 *   and the float32 partial results are added in ascending range order (4 * ranges * T * N
 *   extra scratch bytes).
 *   4 < T <= 128 (decode batches): the packed codes are read directly (no operand scratch) and
 *   widened to int8 q * 16 inside the kernel; tcgen05.mma kind::i8 forms 256 d_G exactly in
 *   int32 and the epilogue applies sw / 256 (exact) and sa, giving the same per-group float32
 *   values.  One kernel writes Y, unless the 128-row weight tiles are too few to fill the
 *   device: then the groups are split into ranges and their float32 partial tiles
 *   (4 * ranges * T * N scratch bytes) are added in ascending range order by a second kernel.
 *   T <= 4 (single-token decode): one kernel on the CUDA cores, no scratch: the weights stream
 *   through registers, __dp4a on q * 16 operands forms 256 d_G exactly in int32, the same
 *   per-group term fl(d_G * sw) * sa is accumulated, and the groups' terms are added in an
 *   order of the kernel's own (ascending per lane, then a tree over lanes).
 *   A split or reordered sum differs from the ascending order only by float32 rounding.
 */
pq_status pq_w4a4_gemm(const uint8_t* codes_A, const float* scales_A, const uint8_t* codes_W,
                       const float* scales_W, int64_t T, int64_t N, int64_t D, int g, void* Y,
                       pq_out_dtype out_dtype, void* stream);

/*
 * pq_w4a4_linear — the activation transform and the GEMM in one call (ParoQuant page §3.2:
 * rotation, scaling and quantisation fused with the matrix multiply to save memory round trips;
 * §6, memory tips: transform first, then quantise):
 *   pq_transform_quant(plan, X, T, ldx, codes_A, scales_A, NULL) followed by
 *   pq_w4a4_gemm(codes_A, scales_A, codes_W, scales_W, T, N, plan->D, plan->g, Y, out_dtype).
 *   T <= 128: the GEMM is launched as a programmatic dependent of the transform: its prologue
 *   and its weight-side loads start while the transform runs (T <= 4: the first 2 KB of each
 *   weight row), and it reads codes_A and scales_A only after the transform has completed.
 *   T > 128: the two run one after the other.
 *   codes_A [T][D/2] and scales_A [T][D/g] are caller-owned device buffers and are written (the
 *   activation codes stay available; with 8-bit outlier groups D is the plan's Gx * g and D/g its
 *   Gx, for codes_W and scales_W too).  codes_W and scales_W must be complete when the call is
 *   made (written by work enqueued on `stream` before it, or earlier); Y must not overlap X,
 *   codes_A or scales_A.  Arguments as for the two calls (smoothing plans: no smooth_out).
 *   Launches: the transform's plus pq_w4a4_gemm_launch_count_g(T, N, D, g).
 */
pq_status pq_w4a4_linear(const pq_plan* plan, const void* X, int64_t T, int64_t ldx, uint8_t* codes_A,
                         float* scales_A, const uint8_t* codes_W, const float* scales_W, int64_t N, void* Y,
                         pq_out_dtype out_dtype, void* stream);

/*
 * Rotated runtime smoothing with channel reordering: the RRS page's main equation (X_rot = X R,
 * s_j = max |(X_rot)_j|, Quantize(X_rot diag(s)^-1), Y = sum_j (X'_q)_j (W'_q)_j^T s_j) carried
 * out as in its Fig. 4: (1) the channels are reordered by their maxima, (2) the reordered
 * channels are grouped by 128 (the GEMM's block) and each group's maximum is its smoothing scale,
 * (3) the GEMM applies each block's smoothing scale to the block's interim result.  Activations
 * are quantised per token over the whole row (the page's setup); weights per group of 128
 * reordered channels.  All four calls need a PQ_HADAMARD plan (R = block Hadamard H_128/sqrt(128))
 * with D <= 16384 (else PQ_ERR_UNSUPPORTED); pointers are device pointers owned by the caller,
 * 16-byte aligned; errors and launches behave as for the calls above.
 *
 * pq_rrs_prepare — from this call's activations X (bf16 [T][ldx], as pq_transform_quant):
 *   chan_max     float32 [D]: max over all T rows of |(X R)[:, j]| (original channel order).
 *   perm         int32 [D]: perm[k] = the original channel at reordered position k (descending
 *                maximum; equal maxima keep the lower channel first).
 *   inv_perm     int32 [D]: the inverse, inv_perm[perm[k]] = k.
 *   group_scale  float32 [D/128]: s_G, the largest maximum of reordered group G (0 -> 1).
 *   The four outputs are written in full (chan_max and inv_perm are cleared first on `stream`).
 */
pq_status pq_rrs_prepare(const pq_plan* plan, const void* X, int64_t T, int64_t ldx, float* chan_max,
                         int32_t* perm, int32_t* inv_perm, float* group_scale, void* stream);

/*
 * pq_rrs_transform_quant — per row t: v_k = (X R)[t, perm[k]] / s_(k / 128), then one symmetric
 * INT4 scale for the whole row, token_scales[t] = max_k |v_k| / 7, codes = RNE(v / scale) packed
 * as elsewhere (codes [T][D/2] are in the reordered channel order).  perm and group_scale as
 * written by pq_rrs_prepare (for the same or an earlier batch).
 */
pq_status pq_rrs_transform_quant(const pq_plan* plan, const void* X, int64_t T, int64_t ldx,
                                 const int32_t* perm, const float* group_scale, uint8_t* codes,
                                 float* token_scales, void* stream);

/*
 * pq_rrs_pack_weights — per weight row n (W bf16 [N][D] dense): v_k = (W R)[n, perm[k]] (the
 * same rotation; H is symmetric orthogonal, so R^-T = R), quantised per group of 128 reordered
 * channels; scales_W[n][G] = (max_(k in G) |v_k| / 7) * s_G, the group's weight scale with its
 * smoothing scale folded in, which is the factor pq_rrs_gemm applies per block.
 */
pq_status pq_rrs_pack_weights(const pq_plan* plan, const void* W, int64_t N, const int32_t* perm,
                              const float* group_scale, uint8_t* codes_W, float* scales_W, void* stream);

/*
 * pq_rrs_gemm — Y[t][n] = token_scales[t] * sum_G scales_W[n][G] * d_G[t][n], d_G the exact
 * integer dot of group G as in pq_w4a4_gemm: per block one multiply-add per output element with
 * the block's factor, then the token's scale once.  codes and scales as written by
 * pq_rrs_transform_quant (token_scales float32 [T]) and pq_rrs_pack_weights.  Sizes, output,
 * scratch, splitting and errors as for pq_w4a4_gemm.
 */
pq_status pq_rrs_gemm(const uint8_t* codes_A, const float* token_scales, const uint8_t* codes_W,
                      const float* scales_W, int64_t T, int64_t N, int64_t D, int g, void* Y,
                      pq_out_dtype out_dtype, void* stream);

/* Bytes of the fixed device-array scratch behind pq_w4a4_gemm_noalloc (32 MiB). */
#define PQ_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * pq_w4a4_gemm_noalloc — the same operation, arguments, layouts and results as pq_w4a4_gemm,
 * for callers that cannot let a library allocate device memory (for example an engine that has
 * reserved nearly all of it for its own caches, or a loop that needs a fixed footprint).  None
 * of the pages has a counterpart: it only changes where the GEMM's temporary int8 operands live.
 *   Scratch: a fixed device array of PQ_NOALLOC_SCRATCH_BYTES inside the library, one per
 *   device, reserved when the CUDA module holding it is loaded on that device and held by
 *   every process that loads the library until it exits.  With CUDA's lazy module loading (the
 *   default since CUDA 12.2) that happens at the first call of the library that touches the
 *   module on the device, which may be this entry's first call: a caller that reserves nearly
 *   all device memory for itself should make one call on each device before doing so, or run
 *   with CUDA_MODULE_LOADING=EAGER.  No call allocates or frees memory.  It needs no zeroing:
 *   each call writes every scratch byte it reads, and the tensor maps bound each operand to
 *   its own rows, so bytes left by an earlier, larger call are never read.
 *   Limit: (T + N) * D <= PQ_NOALLOC_SCRATCH_BYTES, else PQ_ERR_INVALID_ARG before anything is
 *   launched.
 *   First call on each device: looks up the scratch address with that device current; make it
 *   before any stream capture.
 *   Concurrency: calls on one device share the scratch.  Calls whose GPU work may overlap
 *   (different streams without an event between them) race and can give wrong results; issue
 *   them on one stream or order them with events.
 *   Errors and timeouts are reported as for pq_w4a4_gemm.
 */
pq_status pq_w4a4_gemm_noalloc(const uint8_t* codes_A, const float* scales_A,
                               const uint8_t* codes_W, const float* scales_W, int64_t T,
                               int64_t N, int64_t D, int g, void* Y, pq_out_dtype out_dtype,
                               void* stream);

/*
 * pq_w4a4_gemm_launch_count — host-only query, no counterpart in the pages.  Writes to
 * *launches the number of kernels one pq_w4a4_gemm call with these sizes and g = 128 launches
 * on the current device (pq_w4a4_gemm_launch_count_g: the same for group size g).  T > 128: 2 (operand expansion, contraction) or 3 (plus the split-K
 * reduction, chosen when the 256 x 256 output tiles fill at most half of the device's SM
 * pairs).  4 < T <= 128: 1, or 2 with the group-range reduction.  T <= 4: 1.  pq_w4a4_gemm_noalloc never
 * splits: it launches 2 for T > 128 and 1 otherwise.  Sizes are validated as for
 * pq_w4a4_gemm (PQ_ERR_INVALID_ARG otherwise).  Without a usable device the count assumes 148 SMs.
 */
pq_status pq_w4a4_gemm_launch_count(int64_t T, int64_t N, int64_t D, int* launches);
pq_status pq_w4a4_gemm_launch_count_g(int64_t T, int64_t N, int64_t D, int g, int* launches);

/*
 * pq_check_status — synchronises `stream`, then reads and clears the device status words
 * (the plan's, if plan != NULL, and the GEMM's).  Returns PQ_ERR_TIMEOUT if a bounded
 * device-side wait gave up since the last check (the affected output is incomplete),
 * PQ_ERR_CUDA if the stream reports an error, PQ_OK otherwise.
 */
pq_status pq_check_status(const pq_plan* plan, void* stream);

/*
 * pq_selftest_wait_timeout — diagnostic, no counterpart in the pages.  Launches on `stream` one
 * thread that waits on a shared-memory barrier nothing will complete, using the same bounded
 * wait as every pipeline barrier of the library's kernels; after limit_ns (1 us .. 100 ms,
 * else PQ_ERR_INVALID_ARG) it gives up and sets the GEMM status word, so the next
 * pq_check_status returns PQ_ERR_TIMEOUT (and clears it).  Nothing faults or traps; the
 * context stays usable.
 */
pq_status pq_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Static description of a status code. */
const char* pq_status_string(pq_status status);

/* Detail of the last failure on the calling thread ("" if none).  Valid until the next call. */
const char* pq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PQ_H_ */
