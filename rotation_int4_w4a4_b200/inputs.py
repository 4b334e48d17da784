"""Seeded synthetic inputs shared by the tests, the oracle checks and the benchmark.

This module holds none of the method's arithmetic: it only draws numbers.  It is the one
module that both the CPU oracle's tests and the CUDA path's tests/benchmark use, so that
both sides see bit-identical inputs.

Generator
---------
Every stream is counter based: element ``i`` of the stream with seed ``s`` is
``mix(s + (i + 1) * GAMMA)`` where ``mix`` is the SplitMix64 output function
(Steele, Lea & Flood, "Fast Splittable Pseudorandom Number Generators", OOPSLA 2014;
the constants are those of Vigna's public-domain ``splitmix64.c``).  Uniforms use the top
53 bits; normals use Box-Muller on consecutive pairs; Laplace uses the inverse CDF.
Floating values are rounded to bfloat16 with round-to-nearest-even on the float32 bit
pattern and returned as raw ``uint16`` bit patterns (numpy has no bfloat16 dtype).

Workloads
---------
The shapes follow LLaMA-3-8B projections (hidden 4096, FFN 14336, group 128).  The five
named workloads and their outlier recipes are defined in :func:`workload`.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
BASE_SEED = 0x5EED0000

# Sub-stream tags (added to a workload's seed) so that X, W, angles, ... never overlap.
TAG_X, TAG_W, TAG_X_OUT, TAG_X_POS, TAG_ANGLES, TAG_BETA, TAG_PAIRS, TAG_CODES = (
    0x0100, 0x0200, 0x0300, 0x0400, 0x0500, 0x0600, 0x0700, 0x0800)


def _mix(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def u64_stream(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Elements ``start .. start+n-1`` of the counter-based SplitMix64 stream ``seed``."""
    idx = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * GAMMA
    return _mix(z)


def uniform01(seed: int, n: int) -> np.ndarray:
    """float64 uniforms in [0, 1) from the top 53 bits."""
    return (u64_stream(seed, n) >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(seed: int, n: int, std: float = 1.0) -> np.ndarray:
    """Box-Muller normals, float64."""
    m = (n + 1) // 2
    u = uniform01(seed, 2 * m)
    u1 = 1.0 - u[0::2]           # (0, 1]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    z = np.empty(2 * m, dtype=np.float64)
    z[0::2] = r * np.cos(2.0 * math.pi * u2)
    z[1::2] = r * np.sin(2.0 * math.pi * u2)
    return z[:n] * std


def laplace(seed: int, n: int, b: float = 1.0) -> np.ndarray:
    """Laplace(0, b) by the inverse CDF, float64."""
    u = uniform01(seed, n) - 0.5                     # [-0.5, 0.5)
    a = np.minimum(np.abs(u) * 2.0, 1.0 - 2.0 ** -53)
    return -b * np.sign(u) * np.log1p(-a)


def distinct_indices(seed: int, count: int, limit: int) -> np.ndarray:
    """``count`` distinct indices in [0, limit), in draw order (first occurrences win)."""
    if count > limit:
        raise ValueError("count > limit")
    out: list[int] = []
    seen: set[int] = set()
    start = 0
    while len(out) < count:
        batch = u64_stream(seed, max(64, 2 * (count - len(out))), start)
        start += batch.size
        for v in (batch % np.uint64(limit)).tolist():
            if v not in seen:
                seen.add(v)
                out.append(v)
                if len(out) == count:
                    break
    return np.asarray(out, dtype=np.int64)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to bfloat16 (RNE on the float32 pattern) -> uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    with np.errstate(over="ignore"):
        r = b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact decode of bfloat16 bit patterns (used only to build float inputs such as beta)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Workload:
    """One synthetic workload: bf16 activations/weights plus the transform's parameters."""
    name: str
    kind: str                 # "hadamard" | "givens" | "smooth_hadamard"
    T: int
    D: int
    N: int
    g: int
    K: int
    seed: int
    X: np.ndarray             # uint16 bf16 bits [T, D]
    W: np.ndarray | None      # uint16 bf16 bits [N, D] (None when not materialised)
    angles: np.ndarray | None  # float32 [D/g, K, g/2]
    beta: np.ndarray | None    # float32 [D]
    pair_seed: int | None      # seed for the greedy pair selection (pairs are drawn by the method)
    description: str = ""


def _x_gauss_outlier_channels(seed, T, D, n_ch, mult):
    x = normal(seed + TAG_X, T * D).reshape(T, D)
    ch = distinct_indices(seed + TAG_X_OUT, n_ch, D)
    x[:, ch] *= mult
    return x


def workload(name: str, T: int | None = None, N: int | None = None, kind: str | None = None,
             with_weights: bool = True) -> Workload:
    """Build a named workload.

    ``tiny``     T16 D256 N256, Givens K=8; N(0,1) with channels 3 and 200 x50 and
                 round(0.001*T*D) seeded entries x100.
    ``q_proj``   T2048 D4096 N4096, block Hadamard; N(0,1) with 8 seeded channels x30.
    ``up_proj``  T4096 D4096 N14336, Givens K=16; N(0,1) with round(0.0005*T*D) spikes x200.
    ``down_proj`` T8192 D14336 N4096, runtime smoothing + Hadamard; Laplace(0,1) with 16
                 seeded channels x100.
    ``sweep``    T in {1..16384} D4096, N 4096 or 14336, Hadamard or Givens K=8; N(0,1)
                 with 8 seeded channels x30.
    Weights are N(0, 0.02) (0.02 is the standard deviation).  Angles are U(-pi, pi) and
    beta ~ N(0, 0.1), both rounded to float32.
    """
    g = 128
    if name == "tiny":
        seed = BASE_SEED + 0
        T, D, N, K, kind = 16, 256, 256, 8, "givens"
        x = normal(seed + TAG_X, T * D).reshape(T, D)
        x[:, [3, 200]] *= 50.0
        pos = distinct_indices(seed + TAG_X_POS, int(round(0.001 * T * D)), T * D)
        x.reshape(-1)[pos] *= 100.0
        desc = "X[16,256] N(0,1), ch 3,200 x50, 4 entries x100; Givens K=8"
    elif name == "q_proj":
        seed = BASE_SEED + 1
        T = 2048 if T is None else T
        D, N, K, kind = 4096, 4096, 0, "hadamard"
        x = _x_gauss_outlier_channels(seed, T, D, 8, 30.0)
        desc = f"X[{T},4096] N(0,1), 8 ch x30; block Hadamard"
    elif name == "up_proj":
        seed = BASE_SEED + 2
        T = 4096 if T is None else T
        D, N, K, kind = 4096, 14336, 16, "givens"
        x = normal(seed + TAG_X, T * D).reshape(T, D)
        pos = distinct_indices(seed + TAG_X_POS, int(round(0.0005 * T * D)), T * D)
        x.reshape(-1)[pos] *= 200.0
        desc = f"X[{T},4096] N(0,1), 0.05% spikes x200; Givens K=16"
    elif name == "down_proj":
        seed = BASE_SEED + 3
        T = 8192 if T is None else T
        D, N, K, kind = 14336, 4096, 0, "smooth_hadamard"
        x = laplace(seed + TAG_X, T * D).reshape(T, D)
        ch = distinct_indices(seed + TAG_X_OUT, 16, D)
        x[:, ch] *= 100.0
        desc = f"X[{T},14336] Laplace(0,1), 16 ch x100; smooth + Hadamard"
    elif name == "sweep":
        seed = BASE_SEED + 4 + 100 * (T or 0)
        T = 1 if T is None else T
        D = 4096
        N = 4096 if N is None else N
        kind = "hadamard" if kind is None else kind
        K = 8 if kind == "givens" else 0
        x = _x_gauss_outlier_channels(seed, T, D, 8, 30.0)
        desc = f"X[{T},4096] N(0,1), 8 ch x30; {kind}"
    else:
        raise KeyError(name)
    if T is not None and name in ("tiny",):
        pass
    X = to_bf16_bits(x)
    W = to_bf16_bits(normal(seed + TAG_W, N * D, 0.02).reshape(N, D)) if with_weights else None
    angles = beta = None
    pair_seed = None
    if kind == "givens":
        G = D // g
        angles = ((uniform01(seed + TAG_ANGLES, G * K * (g // 2)) * 2.0 - 1.0) * math.pi
                  ).astype(np.float32).reshape(G, K, g // 2)
        beta = normal(seed + TAG_BETA, D, 0.1).astype(np.float32)
        pair_seed = seed + TAG_PAIRS
    return Workload(name, kind, T, D, N, g, K, seed, X, W, angles, beta, pair_seed, desc)


def random_codes(seed: int, rows: int, D: int, g: int = 128):
    """Random packed int4 codes (all 16 nibble values) and positive float32 scales.

    Used to drive the GEMM with inputs that exercise every code, independent of any
    transform.  Returns (codes u8 [rows, D/2], scales f32 [rows, D/g]).
    """
    codes = (u64_stream(seed + TAG_CODES, rows * D // 2) & np.uint64(0xFF)).astype(np.uint8)
    sc = np.exp(normal(seed + TAG_CODES + 1, rows * (D // g), 0.5)) * 0.01
    return codes.reshape(rows, D // 2), sc.astype(np.float32).reshape(rows, D // g)
