"""CPU oracle (float64 numpy) for the rotation + INT4 W4A4 hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or execute this
module; only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
use it.  It shares no code, table or constant generator with the CUDA path.

Sources (pages, by title and section):
  [ParoQuant page]   codearts.csdn.net article on independent rotation + channel scaling:
                     §2.2 "独立旋转的技术实现" (Algorithm A1, its three listed properties),
                     §2.3 "通道缩放的自适应机制" (W^ = diag(alpha) W, alpha = exp(beta),
                     128 channels share one set of quantisation parameters).
  [Hadamard page]    "神经网络量化技术：Hadamard变换与格码本优化" §2.1 (entries
                     (-1)^popcount(i&j), 1/sqrt(n) normalisation), §4.2 (butterflies,
                     H(AB) = (HA)B), §6.1 (block Hadamard).
  [RRS page]         "Rotated Runtime Smooth: 训练无关的激活平滑器" — main equation
                     (X_rot = XR, W_rot = R^-1 W, s_j = max|(X_rot)_j|, quantise
                     X_rot diag(s)^-1, Y = sum_j ...), the R = (1/sqrt(K))[s_ij] definition,
                     alpha = max|X| / (2^(N-1) - 1), INT4 range -8..7, RTN rounding, Fig. 2(a)
                     Y = (XR)(R^-1 W^T) = XW^T, Fig. 4 (per-block scales on interim results).

Readings where the pages are silent or garbled are listed in the repository's design notes;
each function below states the reading it implements.

Conventions: X is [T, D] (rows = tokens), W is [N, D] (Y = X W^T), group size g, G = D/g
groups per row.  bf16 inputs arrive as uint16 bit patterns and are decoded exactly.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

NONE = 0xFF      # pair slot with no pair (identity)


# ----------------------------------------------------------------------------- decoding
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns: the 16 bits are the top half of a float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32).astype(np.float64)


# ------------------------------------------------------------ pair selection (Alg. A1)
class SplitMix64:
    """SplitMix64 (Steele, Lea & Flood, OOPSLA 2014), written from its published definition.

    The pages shuffle the candidate pairs with Python's ``shuffle``; that stream is not
    reproducible, so the shuffle here is a Fisher-Yates (Durstenfeld) shuffle driven by this
    generator: for i = n-1 down to 1, draw r and swap a[i] with a[r mod (i+1)].
    """
    _MASK = (1 << 64) - 1

    def __init__(self, seed: int):
        self.state = seed & self._MASK

    def next(self) -> int:
        self.state = (self.state + 0x9E3779B97F4A7C15) & self._MASK
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & self._MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & self._MASK
        return z ^ (z >> 31)


def shuffled_candidates(rng: SplitMix64, g: int) -> list[tuple[int, int]]:
    """All pairs (i, j), i < j < g, in lexicographic order, then Fisher-Yates shuffled."""
    cand = [(i, j) for i in range(g) for j in range(i + 1, g)]
    for i in range(len(cand) - 1, 0, -1):
        k = rng.next() % (i + 1)
        cand[i], cand[k] = cand[k], cand[i]
    return cand


def select_pairs_group(rng: SplitMix64, g: int, K: int, N: int) -> list[list[tuple[int, int]]]:
    """[ParoQuant page] §2.2 Algorithm A1 for one group of g channels.

    One shuffled candidate list serves all K layers.  Within a layer a pair is taken when
    neither channel is used yet in that layer; a taken pair is also struck from a global
    availability table so no later layer repeats it.  A layer stops at N pairs.
    """
    cand = shuffled_candidates(rng, g)
    avail = np.ones((g, g), dtype=bool)
    np.fill_diagonal(avail, False)
    layers = []
    for _ in range(K):
        layer: list[tuple[int, int]] = []
        local = avail.copy()
        for i, j in cand:
            if len(layer) >= N:
                break
            if local[i, j]:
                layer.append((i, j))
                local[i, :] = False
                local[:, i] = False
                local[j, :] = False
                local[:, j] = False
                avail[i, j] = False
                avail[j, i] = False
        layers.append(layer)
    return layers


def select_pairs(seed: int, D: int, g: int, K: int, N: int) -> np.ndarray:
    """Pairs for every group: uint8 [D/g, K, g/2, 2], unused slots = 0xFF.

    Groups are processed in order 0..D/g-1, each drawing its own shuffle from one
    SplitMix64 stream seeded with ``seed``.
    """
    G = D // g
    out = np.full((G, K, g // 2, 2), NONE, dtype=np.uint8)
    rng = SplitMix64(seed)
    for gi in range(G):
        for l, layer in enumerate(select_pairs_group(rng, g, K, N)):
            for p, (i, j) in enumerate(layer):
                out[gi, l, p] = (i, j)
    return out


# ------------------------------------------------------------------------ Hadamard
def hadamard_matrix(n: int) -> np.ndarray:
    """[Hadamard page] §2.1: H[i, j] = (-1)^popcount(i & j), Sylvester (natural) order."""
    i = np.arange(n)
    bits = np.bitwise_and.outer(i, i)
    pc = np.zeros_like(bits)
    while bits.any():
        pc += bits & 1
        bits = bits >> 1
    return np.where(pc % 2 == 0, 1.0, -1.0)


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform along the last axis ([Hadamard page] §4.2
    butterflies): log2(n) radix-2 stages, each (a, b) -> (a + b, a - b)."""
    y = np.array(x, dtype=np.float64, copy=True)
    n = y.shape[-1]
    h = 1
    while h < n:
        v = y.reshape(y.shape[:-1] + (n // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        h *= 2
    return y


def hadamard_rotate(x: np.ndarray, g: int) -> np.ndarray:
    """Block Hadamard rotation x -> x (H_g / sqrt(g)) per group of g channels.

    [RRS page] R = (1/sqrt(K)) [s_ij], s_ij = +-1; [Hadamard page] §6.1 block Hadamard.
    H_g is symmetric, so the row-vector product x H equals the FWHT of x.
    """
    rows, D = x.shape
    y = fwht(x.reshape(rows, D // g, g)) / math.sqrt(g)
    return y.reshape(rows, D)


def hadamard_rotate_explicit(x: np.ndarray, g: int) -> np.ndarray:
    """Same rotation by an explicit matrix product (cross-check of :func:`hadamard_rotate`)."""
    rows, D = x.shape
    H = hadamard_matrix(g) / math.sqrt(g)
    return (x.reshape(rows, D // g, g) @ H).reshape(rows, D)


# --------------------------------------------------------------------------- Givens
def givens_rotate(x: np.ndarray, pairs: np.ndarray, angles: np.ndarray, g: int,
                  inverse: bool = False) -> np.ndarray:
    """[ParoQuant page] §2.2: K layers of disjoint pair rotations inside each group.

    Reading: layer 0 first; pair (i, j) with angle theta maps the column (x_i, x_j) to
    (cos t * x_i - sin t * x_j, sin t * x_i + cos t * x_j).  ``inverse`` applies the
    transposed rotations in reverse layer order.  cos/sin are taken in float64 of the
    float32 angle.
    """
    rows, D = x.shape
    G, K = pairs.shape[0], pairs.shape[1]
    y = np.array(x, dtype=np.float64, copy=True).reshape(rows, G, g)
    order = range(K - 1, -1, -1) if inverse else range(K)
    for l in order:
        for gi in range(G):
            pl = pairs[gi, l]
            valid = pl[:, 0] != NONE
            i = pl[valid, 0].astype(np.int64)
            j = pl[valid, 1].astype(np.int64)
            th = angles[gi, l][valid].astype(np.float64)
            c, s = np.cos(th), np.sin(th)
            if inverse:
                s = -s
            xi = y[:, gi, i].copy()
            xj = y[:, gi, j].copy()
            y[:, gi, i] = c * xi - s * xj
            y[:, gi, j] = s * xi + c * xj
    return y.reshape(rows, D)


def givens_matrix(pairs_g: np.ndarray, angles_g: np.ndarray, g: int) -> np.ndarray:
    """Explicit g x g matrix R = G_0 G_1 ... G_{K-1} of one group's layers (row-vector
    convention x' = x R), each G_l built from the identity; a cross-check only."""
    R = np.eye(g)
    for l in range(pairs_g.shape[0]):
        Gl = np.eye(g)
        for (i, j), th in zip(pairs_g[l], angles_g[l]):
            if i == NONE:
                continue
            c, s = math.cos(float(th)), math.sin(float(th))
            # x'_i = c x_i - s x_j ; x'_j = s x_i + c x_j  (x' = x Gl)
            Gl[i, i] = c
            Gl[j, i] = -s
            Gl[i, j] = s
            Gl[j, j] = c
        R = R @ Gl
    return R


# ------------------------------------------------------------------------ smoothing
def smooth_scales(x: np.ndarray, block: int = 128) -> np.ndarray:
    """Runtime smoothing scales ([RRS page] main equation, s_j = max |(X)_j|), taken per
    channel over each block of ``block`` consecutive rows (the last block may be short).
    Reading: a channel whose block maximum is 0 gets s = 1.  Returns float64 [nb, D]."""
    rows, D = x.shape
    nb = (rows + block - 1) // block
    s = np.empty((nb, D), dtype=np.float64)
    for b in range(nb):
        s[b] = np.max(np.abs(x[b * block:(b + 1) * block]), axis=0)
    s[s == 0.0] = 1.0
    return s


def apply_smoothing(x: np.ndarray, s: np.ndarray, block: int = 128) -> np.ndarray:
    """x[t, j] / s[t // block, j] ([RRS page]: X diag(s)^-1)."""
    return x / np.repeat(s, block, axis=0)[: x.shape[0]]


# ----------------------------------------------------------------------- quantisation
@dataclasses.dataclass
class Quantized:
    codes: np.ndarray        # int8 [rows, D], values in -8..7
    scales: np.ndarray       # float32 [rows, G]
    ratio: np.ndarray        # float64 [rows, D]: y / (m / 7), the value that was rounded
    near_tie: np.ndarray     # bool [rows, D]: |frac(ratio) - 0.5| < 1e-3


def quantize(y: np.ndarray, g: int, tie_band: float = 1e-3) -> Quantized:
    """Symmetric per-group INT4: scale = max|y| / 7 ([RRS page]: alpha = max|X| / (2^(N-1)-1)
    with N = 4; [ParoQuant page] §2.3: 128 channels share the parameters), codes =
    clamp(round(y / scale), -8, 7) ([RRS page]: range -8..7, RTN).

    Readings: rounding is half-to-even; an all-zero group gets scale 0 and codes 0; the
    rounded value is computed in float64 as 7 y / m and the stored scale is float32(m / 7).
    """
    rows, D = y.shape
    G = D // g
    yg = y.reshape(rows, G, g)
    if not np.all(np.isfinite(yg)):
        raise ValueError("non-finite input is outside the contract")
    m = np.max(np.abs(yg), axis=2, keepdims=True)
    safe = np.where(m > 0.0, m, 1.0)
    ratio = np.where(m > 0.0, 7.0 * yg / safe, 0.0)
    codes = np.clip(np.rint(ratio), -8, 7).astype(np.int8)
    scales = (m[..., 0] / 7.0).astype(np.float32)
    frac = ratio - np.floor(ratio)
    near = np.abs(frac - 0.5) < tie_band
    return Quantized(codes.reshape(rows, D), scales, ratio.reshape(rows, D), near.reshape(rows, D))


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Reading: byte k = (q[2k] & 0xF) | (q[2k+1] & 0xF) << 4, two's-complement nibbles."""
    c = np.asarray(codes, dtype=np.int16) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_nibbles` -> int8 codes in -8..7."""
    p = np.asarray(packed, dtype=np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# ----------------------------------------------------------------------------- plans
@dataclasses.dataclass
class Plan:
    """What the transform needs: kind in {"hadamard", "givens", "smooth_hadamard"}."""
    kind: str
    D: int
    g: int = 128
    K: int = 0
    pairs: np.ndarray | None = None     # uint8 [G, K, g/2, 2]
    angles: np.ndarray | None = None    # float32 [G, K, g/2]
    beta: np.ndarray | None = None      # float32 [D] or None (= 0)
    smooth_after_rotate: bool = False
    smooth_block: int = 128


def activation_transform(x: np.ndarray, plan: Plan):
    """x -> x M (before quantisation).  Returns (y, smoothing scales or None).

    hadamard:         y = x H/sqrt(g) per group.
    givens:           y = ((x G_0) ... G_{K-1}) diag(exp(-beta))  — [ParoQuant page] §2.3
                      puts alpha = exp(beta) on the weights (W^ = diag(alpha) W), so the
                      activations carry exp(-beta).  Reading: the scale follows the rotations.
    smooth_hadamard:  y = (x diag(s)^-1) H/sqrt(g), s per channel per row block (default), or
                      the [RRS page] order y = (x H/sqrt(g)) diag(s)^-1 with s taken on the
                      rotated values when ``smooth_after_rotate``.
    """
    if plan.kind == "hadamard":
        return hadamard_rotate(x, plan.g), None
    if plan.kind == "givens":
        y = givens_rotate(x, plan.pairs, plan.angles, plan.g)
        if plan.beta is not None:
            y = y * np.exp(-plan.beta.astype(np.float64))
        return y, None
    if plan.kind == "smooth_hadamard":
        if plan.smooth_after_rotate:
            r = hadamard_rotate(x, plan.g)
            s = smooth_scales(r, plan.smooth_block)
            return apply_smoothing(r, s, plan.smooth_block), s
        s = smooth_scales(x, plan.smooth_block)
        return hadamard_rotate(apply_smoothing(x, s, plan.smooth_block), plan.g), s
    raise ValueError(plan.kind)


def weight_transform(w: np.ndarray, plan: Plan, smooth_w: np.ndarray | None = None) -> np.ndarray:
    """w -> w M^{-T}, so that (x M)(w M^{-T})^T = x w^T ([RRS page] Fig. 2(a) and
    W_rot = R^-1 W; [Hadamard page] §4.2 H(AB) = (HA)B; [OSTQuant page] §3.2: the
    transform pair is merged into the weights).

    hadamard:         M = H/sqrt(g) is symmetric orthogonal: same rotation.
    givens:           M = R diag(e^-beta)  ->  M^{-T} = R diag(e^+beta): same rotations,
                      then x exp(+beta).
    smooth_hadamard:  M = diag(1/s) H/sqrt(g)  ->  M^{-T} = diag(s) H/sqrt(g): scale the
                      channels by ``smooth_w`` then rotate (the weight side has one s).
    """
    if plan.kind == "hadamard":
        return hadamard_rotate(w, plan.g)
    if plan.kind == "givens":
        y = givens_rotate(w, plan.pairs, plan.angles, plan.g)
        if plan.beta is not None:
            y = y * np.exp(plan.beta.astype(np.float64))
        return y
    if plan.kind == "smooth_hadamard":
        s = np.ones(w.shape[1]) if smooth_w is None else np.asarray(smooth_w, np.float64)
        if plan.smooth_after_rotate:
            return hadamard_rotate(w, plan.g) * s
        return hadamard_rotate(w * s, plan.g)
    raise ValueError(plan.kind)


@dataclasses.dataclass
class TQResult:
    codes: np.ndarray          # uint8 [rows, D/2] packed
    scales: np.ndarray         # float32 [rows, G]
    smooth: np.ndarray | None  # float32 [nb, D] or None
    q: Quantized               # unpacked codes, ratios, near-tie mask
    y: np.ndarray              # float64 transformed values before quantisation


def transform_quant(x_bits: np.ndarray, plan: Plan) -> TQResult:
    """The activation path: decode bf16, transform, quantise per group, pack."""
    x = bf16_to_f64(x_bits)
    y, s = activation_transform(x, plan)
    q = quantize(y, plan.g)
    return TQResult(pack_nibbles(q.codes), q.scales,
                    None if s is None else s.astype(np.float32), q, y)


def pack_weights(w_bits: np.ndarray, plan: Plan, smooth_w: np.ndarray | None = None) -> TQResult:
    """The weight path: decode bf16, apply M^{-T} per row, quantise per group, pack."""
    w = bf16_to_f64(w_bits)
    y = weight_transform(w, plan, smooth_w)
    q = quantize(y, plan.g)
    return TQResult(pack_nibbles(q.codes), q.scales, None, q, y)


# ------------------------------------------------------------------------------ GEMM
@dataclasses.dataclass
class GemmResult:
    y32: np.ndarray   # float32 [T, N], fp32 accumulation over groups in ascending order
    y64: np.ndarray   # float64 [T, N], exact sum of the same terms


def group_dots(codes_a: np.ndarray, codes_w: np.ndarray, g: int) -> np.ndarray:
    """Integer dot products per group: d[G, T, N] = sum_{k in group} qa[t,k] qw[n,k].
    Exact: the float64 matmul of integers with |d| <= 128*64 has no rounding."""
    qa = unpack_nibbles(codes_a).astype(np.float64)
    qw = unpack_nibbles(codes_w).astype(np.float64)
    T, D = qa.shape
    N = qw.shape[0]
    G = D // g
    d = np.empty((G, T, N), dtype=np.float64)
    for gi in range(G):
        d[gi] = qa[:, gi * g:(gi + 1) * g] @ qw[:, gi * g:(gi + 1) * g].T
    return d.astype(np.int64)


def gemm(codes_a, scales_a, codes_w, scales_w, g: int = 128) -> GemmResult:
    """W4A4 GEMM ([RRS page] main equation, last line, and Fig. 4 step (3): the integer
    product is formed per K-block = quantisation group and the block's scales are applied
    to the interim result):  Y[t,n] = sum_G sa[t,G] sw[n,G] d_G[t,n].

    Reading: fp32 accumulation over G in ascending order, each term fl32(fl32(sa*sw) * d);
    the float64 shadow is the exact sum of sa*sw*d.
    """
    d = group_dots(codes_a, codes_w, g)
    G, T, N = d.shape
    sa = np.asarray(scales_a, dtype=np.float32)
    sw = np.asarray(scales_w, dtype=np.float32)
    acc = np.zeros((T, N), dtype=np.float32)
    acc64 = np.zeros((T, N), dtype=np.float64)
    for gi in range(G):
        s = sa[:, gi][:, None] * sw[:, gi][None, :]                 # float32 product
        term = s * d[gi].astype(np.float32)                         # float32 product
        acc = (acc + term).astype(np.float32)
        acc64 += sa[:, gi].astype(np.float64)[:, None] * sw[:, gi].astype(np.float64)[None, :] \
            * d[gi].astype(np.float64)
    return GemmResult(acc, acc64)


def bf16_round(y32: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of float32 values to bfloat16, returned as float32 values."""
    b = np.ascontiguousarray(y32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (r.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ------------------------------------------------ rotated runtime smoothing (RRS Fig. 4)
@dataclasses.dataclass
class RRSPrep:
    chan_max: np.ndarray     # float64 [D]: max over all rows of |X_rot[:, j]| (original channel j)
    perm: np.ndarray         # int64 [D]: reordered position k holds original channel perm[k]
    group_scale: np.ndarray  # float64 [G]: s_G, the maximum over reordered group G (0 -> 1)


def rrs_prepare(x_bits: np.ndarray, g: int = 128) -> RRSPrep:
    """[RRS page] main equation: X_rot = X R and s_j = max |(X_rot)_j| over every row of the
    column; Fig. 4 (1): the channels are reordered by their maxima; Fig. 4 (2): the reordered
    channels are grouped by the GEMM's block size and each group's maximum is its runtime
    smoothing scale.

    Readings: R is the block Hadamard H_g / sqrt(g) (the page's R = (1/sqrt(K))[s_ij]); the order
    is descending, ties broken by the lower original index; a group whose maximum is 0 gets 1.
    """
    xr = hadamard_rotate(bf16_to_f64(x_bits), g)
    D = xr.shape[1]
    m = np.max(np.abs(xr), axis=0)
    perm = np.lexsort((np.arange(D), -m))          # primary key: -m ascending; then the index
    s = m[perm].reshape(D // g, g).max(axis=1)
    s[s == 0.0] = 1.0
    return RRSPrep(m, perm.astype(np.int64), s)


def rrs_transform_quant(x_bits: np.ndarray, prep: RRSPrep, g: int = 128) -> TQResult:
    """The smoothed activations X_rot[:, perm] / s_G ([RRS page] main equation, fourth line:
    Quantize(X_rot diag(s)^-1), with s constant over each reordered group as in Fig. 4 (2)),
    quantised symmetrically per row over all D channels (the RRS page's setup quantises
    activations per token): scale = max|.| / 7, codes = RNE(value / scale).  Returns codes
    [rows, D/2] and the per-row scales [rows] (TQResult.scales)."""
    xr = hadamard_rotate(bf16_to_f64(x_bits), g)
    D = xr.shape[1]
    xs = xr[:, prep.perm] / np.repeat(prep.group_scale, g)
    q = quantize(xs, D)
    return TQResult(pack_nibbles(q.codes), q.scales[:, 0].copy(), None, q, xs)


def rrs_pack_weights(w_bits: np.ndarray, prep: RRSPrep, g: int = 128) -> TQResult:
    """W_rot = W R^-T (the same block Hadamard, symmetric orthogonal) with its channels reordered
    like the activations, quantised per group of g reordered channels.  The group's smoothing
    scale is folded into the stored weight scale ([RRS page] Fig. 4 (3): the runtime smoothing
    scales are applied to the interim block results):  F[n, G] = fl32(fl32(m / 7) * fl32(s_G))."""
    wr = hadamard_rotate(bf16_to_f64(w_bits), g)[:, prep.perm]
    q = quantize(wr, g)
    F = (q.scales.astype(np.float32) * prep.group_scale.astype(np.float32)[None, :]).astype(np.float32)
    return TQResult(pack_nibbles(q.codes), F, None, q, wr)


def rrs_gemm(codes_a, token_scales, codes_w, F, g: int = 128) -> GemmResult:
    """[RRS page] main equation, last line (Y = sum_j (X'_q)_j (W'_q)_j^T s_j) with Fig. 4 (3):
    per block (= quantisation group) the interim integer product is scaled by the block's factor
    F[n, G] (weight scale x smoothing scale), and the token's scale is applied once:
    Y[t, n] = sa[t] * sum_G F[n, G] d_G[t, n].

    Reading: float32 accumulation over G in ascending order, acc = fl(acc + fl(F d)), then
    Y = fl(acc * sa); the float64 shadow is the exact sum."""
    d = group_dots(codes_a, codes_w, g)
    G, T, N = d.shape
    sa = np.asarray(token_scales, dtype=np.float32)
    Fw = np.asarray(F, dtype=np.float32)
    acc = np.zeros((T, N), dtype=np.float32)
    acc64 = np.zeros((T, N), dtype=np.float64)
    for gi in range(G):
        acc = (acc + (Fw[:, gi][None, :] * d[gi].astype(np.float32)).astype(np.float32)).astype(np.float32)
        acc64 += Fw[:, gi].astype(np.float64)[None, :] * d[gi].astype(np.float64)
    return GemmResult((acc * sa[:, None]).astype(np.float32), acc64 * sa.astype(np.float64)[:, None])


# ------------------------------------ 8-bit outlier groups ([ParoQuant page] §4.1, third remedy)
LEVELS8 = 119   # symmetric range of an 8-bit code made of two signed 4-bit digits (reading below)


def quantize_mixed(y: np.ndarray, g: int, groups8, tie_band: float = 1e-3) -> Quantized:
    """Mixed precision ([ParoQuant page] §4.1: extreme outliers keep an 8-bit representation):
    the listed groups are quantised with an 8-bit code, the others as :func:`quantize` (INT4).
    Per group: L = 119 for an 8-bit group, 7 otherwise; scale = max|y| / L (float32),
    codes = clamp(round_half_even(L y / max|y|), -L, L) (INT4: -8..7).

    Reading: the page does not fix the 8-bit format.  An 8-bit code here is one byte made of two
    signed 4-bit digits, q = 16 q_hi + q_lo with q_hi, q_lo in -8..7 (so that an 8-bit group can
    be multiplied as four 4-bit groups); the largest symmetric range of such bytes is +-119.
    Returns int16 codes [rows, D] (not packed)."""
    rows, D = y.shape
    G = D // g
    L = np.full(G, 7.0)
    L[np.asarray(list(groups8), dtype=np.int64)] = float(LEVELS8)
    yg = y.reshape(rows, G, g)
    if not np.all(np.isfinite(yg)):
        raise ValueError("non-finite input is outside the contract")
    m = np.max(np.abs(yg), axis=2, keepdims=True)
    safe = np.where(m > 0.0, m, 1.0)
    ratio = np.where(m > 0.0, L[None, :, None] * yg / safe, 0.0)
    low = np.where(L == 7.0, -8.0, -float(LEVELS8))[None, :, None]
    codes = np.clip(np.rint(ratio), low, L[None, :, None]).astype(np.int16)
    scales = (m[..., 0] / L[None, :]).astype(np.float32)
    frac = ratio - np.floor(ratio)
    near = np.abs(frac - 0.5) < tie_band
    return Quantized(codes.reshape(rows, D), scales, ratio.reshape(rows, D), near.reshape(rows, D))


def transform_quant_mixed(x_bits: np.ndarray, plan: Plan, groups8) -> TQResult:
    """The activation path with 8-bit outlier groups (codes unpacked, int16 [rows, D])."""
    y, s = activation_transform(bf16_to_f64(x_bits), plan)
    q = quantize_mixed(y, plan.g, groups8)
    return TQResult(q.codes, q.scales, None if s is None else s.astype(np.float32), q, y)


def pack_weights_mixed(w_bits: np.ndarray, plan: Plan, groups8, smooth_w: np.ndarray | None = None) -> TQResult:
    """The weight path with the same 8-bit groups (codes unpacked, int16 [rows, D])."""
    y = weight_transform(bf16_to_f64(w_bits), plan, smooth_w)
    q = quantize_mixed(y, plan.g, groups8)
    return TQResult(q.codes, q.scales, None, q, y)


def gemm_mixed(qa: np.ndarray, scales_a, qw: np.ndarray, scales_w, g: int = 128) -> GemmResult:
    """The W4A4 GEMM of :func:`gemm` on integer codes of either width (unpacked):
    Y[t,n] = sum_G fl32(fl32(sa sw) d_G), d_G the exact integer dot (|d| <= 128 * 119^2 < 2^21,
    exact in float32), float32 accumulation over G ascending; float64 shadow of the exact sum."""
    qa = np.asarray(qa, dtype=np.float64)
    qw = np.asarray(qw, dtype=np.float64)
    T, D = qa.shape
    N = qw.shape[0]
    sa = np.asarray(scales_a, dtype=np.float32)
    sw = np.asarray(scales_w, dtype=np.float32)
    acc = np.zeros((T, N), dtype=np.float32)
    acc64 = np.zeros((T, N), dtype=np.float64)
    for gi in range(D // g):
        d = qa[:, gi * g:(gi + 1) * g] @ qw[:, gi * g:(gi + 1) * g].T
        s = sa[:, gi][:, None] * sw[:, gi][None, :]
        acc = (acc + (s * d.astype(np.float32)).astype(np.float32)).astype(np.float32)
        acc64 += sa[:, gi].astype(np.float64)[:, None] * sw[:, gi].astype(np.float64)[None, :] * d
    return GemmResult(acc, acc64)
