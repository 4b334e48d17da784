"""Pins for the CPU oracle: closed forms, invariants, textbook constructions, published
generator vectors and brute force.  None of these re-types the oracle's own formula; each
checks it against something the pages or the mathematics fix.  The last section plants
plausible mistakes in the oracle (on the CPU) and shows that a pin catches each one.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import oracle as O
from rotation_int4_w4a4_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=1):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- generator vectors
def test_splitmix64_published_vectors():
    with open(os.path.join(GOLD, "splitmix64.txt")) as f:
        rows = [l for l in f if l.strip() and not l.startswith("#")]
    for row in rows:
        seed, outs = row.split(":")
        want = [int(v) for v in outs.split()]
        g = oracle.SplitMix64(int(seed))
        assert [g.next() for _ in want] == want
        # The input generator's counter-based form yields the same stream.
        assert inputs.u64_stream(int(seed), len(want)).tolist() == want


def test_bf16_decode_exact():
    vals = np.array([0.0, 1.0, -2.5, 3.140625, 2.0 ** -100, -65280.0], dtype=np.float32)
    bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.bf16_to_f64(bits), vals.astype(np.float64))


# ------------------------------------------------------------------------- Hadamard
def sylvester(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def test_hadamard_golden_h8():
    with open(os.path.join(GOLD, "sylvester_h8.txt")) as f:
        M = np.array([[float(v) for v in l.split()] for l in f if l.strip() and not l.startswith("#")])
    assert np.array_equal(oracle.hadamard_matrix(8), M)
    assert np.array_equal(oracle.fwht(np.eye(8)), M)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128])
def test_hadamard_three_constructions_agree(n):
    H = oracle.hadamard_matrix(n)
    assert np.array_equal(H, sylvester(n))                     # recursive definition
    assert np.array_equal(oracle.fwht(np.eye(n)), H)           # butterflies on e_k
    assert np.array_equal(H @ H.T, n * np.eye(n))              # H H^T = n I exactly


def test_hadamard_rotation_orthonormal_and_involutive():
    x = rng().standard_normal((7, 512))
    y = oracle.hadamard_rotate(x, 128)
    assert np.allclose(y, oracle.hadamard_rotate_explicit(x, 128), rtol=0, atol=1e-12)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # H/sqrt(g) is symmetric orthogonal, so applying it twice is the identity.
    back = oracle.hadamard_rotate(y, 128)
    assert np.max(np.abs(back - x)) < 1e-12
    # Block structure: groups do not mix.
    x2 = x.copy()
    x2[:, 128:] = 0
    assert np.all(oracle.hadamard_rotate(x2, 128)[:, 128:] == 0)


def test_hadamard_closed_forms():
    x = np.zeros((2, 128))
    x[0, 0] = 1.0
    x[1, 0] = x[1, 1] = 1.0
    y = oracle.hadamard_rotate(x, 128)
    assert np.allclose(y[0], 1 / math.sqrt(128), atol=1e-15)
    assert np.allclose(y[1, 0::2], 2 / math.sqrt(128), atol=1e-15)
    assert np.allclose(y[1, 1::2], 0.0, atol=1e-15)
    q = oracle.quantize(y, 128)
    assert np.all(q.codes[0] == 7)
    assert np.all(q.codes[1, 0::2] == 7) and np.all(q.codes[1, 1::2] == 0)
    assert q.scales[0, 0] == np.float32(1 / math.sqrt(128) / 7)


# --------------------------------------------------------------------------- Givens
def one_pair_plan(i, j, theta, g=128, K=1):
    pairs = np.full((1, K, g // 2, 2), oracle.NONE, dtype=np.uint8)
    angles = np.zeros((1, K, g // 2), dtype=np.float32)
    pairs[0, 0, 0] = (i, j)
    angles[0, 0, 0] = theta
    return pairs, angles


def test_givens_closed_forms():
    th = np.float32(0.7)
    c, s = math.cos(float(th)), math.sin(float(th))
    pairs, angles = one_pair_plan(5, 77, th)
    e = np.zeros((3, 128))
    e[0, 5] = 1.0
    e[1, 77] = 1.0
    e[2, 9] = 3.0                       # a channel outside the pair
    y = oracle.givens_rotate(e, pairs, angles, 128)
    assert y[0, 5] == pytest.approx(c, abs=1e-15) and y[0, 77] == pytest.approx(s, abs=1e-15)
    assert y[1, 5] == pytest.approx(-s, abs=1e-15) and y[1, 77] == pytest.approx(c, abs=1e-15)
    assert np.array_equal(y[2], e[2])
    assert np.count_nonzero(y[0]) == 2 and np.count_nonzero(y[1]) == 2
    # theta = 0 is the identity; theta = pi negates the pair.
    p0, a0 = one_pair_plan(5, 77, 0.0)
    x = rng().standard_normal((4, 128))
    assert np.array_equal(oracle.givens_rotate(x, p0, a0, 128), x)
    pp, ap = one_pair_plan(5, 77, np.float32(np.pi))
    ypi = oracle.givens_rotate(x, pp, ap, 128)
    assert np.allclose(ypi[:, [5, 77]], -x[:, [5, 77]], atol=1e-6)


def random_givens(seed, G=2, K=8, g=128):
    pairs = oracle.select_pairs(seed, G * g, g, K, g // 2)
    a = (rng(seed).uniform(-np.pi, np.pi, size=(G, K, g // 2))).astype(np.float32)
    return pairs, a


def test_givens_layers_match_explicit_product_and_are_orthogonal():
    pairs, angles = random_givens(11)
    x = rng(2).standard_normal((5, 256))
    y = oracle.givens_rotate(x, pairs, angles, 128)
    for gi in range(2):
        R = oracle.givens_matrix(pairs[gi], angles[gi], 128)
        assert np.allclose(R @ R.T, np.eye(128), atol=1e-12)
        assert np.allclose(y[:, gi * 128:(gi + 1) * 128], x[:, gi * 128:(gi + 1) * 128] @ R,
                           rtol=0, atol=1e-12)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    back = oracle.givens_rotate(y, pairs, angles, 128, inverse=True)
    assert np.max(np.abs(back - x)) < 1e-12


# ----------------------------------------------------- channel scale (ParoQuant §2.3)
def _identity_pairs_plan(beta, K=2, G=2, g=128):
    """A Givens plan whose every slot is empty: the rotations are the identity, so only the
    channel scale acts."""
    pairs = np.full((G, K, g // 2, 2), oracle.NONE, dtype=np.uint8)
    angles = np.zeros((G, K, g // 2), dtype=np.float32)
    return oracle.Plan("givens", G * g, g, K, pairs, angles, beta)


def test_channel_scale_direction_closed_form():
    """ParoQuant page §2.3 fixes W^ = diag(alpha) W with alpha = exp(beta), alpha one factor
    per input channel: the weights are multiplied by exp(+beta) and, for the product to be
    unchanged, the activations by exp(-beta).  With no rotation this is the whole transform."""
    beta = (rng(12).standard_normal(256) * 0.7).astype(np.float32)
    plan = _identity_pairs_plan(beta)
    x = rng(13).standard_normal((5, 256))
    w = rng(14).standard_normal((7, 256))
    e = np.exp(beta.astype(np.float64))
    y, s = oracle.activation_transform(x, plan)
    assert s is None
    assert np.allclose(y, x / e, rtol=1e-15, atol=0)
    assert np.allclose(oracle.weight_transform(w, plan), w * e, rtol=1e-15, atol=0)
    # A channel with beta = ln 2 exactly halves the activation and doubles the weight.
    b2 = np.zeros(256, dtype=np.float32)
    b2[9] = np.float32(math.log(2.0))
    p2 = _identity_pairs_plan(b2)
    one = np.ones((1, 256))
    ya, _ = oracle.activation_transform(one, p2)
    yw = oracle.weight_transform(one, p2)
    assert ya[0, 9] == pytest.approx(0.5, rel=1e-7) and yw[0, 9] == pytest.approx(2.0, rel=1e-7)
    assert np.all(np.delete(ya[0], 9) == 1.0) and np.all(np.delete(yw[0], 9) == 1.0)


def test_channel_scale_follows_the_rotations():
    """Reading: the channel scale is applied after the K layers (y = (x G_0 ... G_{K-1})
    diag(exp(-beta))).  One pair (5, 77) rotated by theta and a scale on channel 77 only:
    e_5 goes to (cos, sin) on (5, 77) and then channel 77 alone is divided by exp(beta_77)."""
    g = 128
    th = np.float32(0.9)
    pairs, angles = one_pair_plan(5, 77, th)
    beta = np.zeros(g, dtype=np.float32)
    beta[77] = np.float32(0.5)
    plan = oracle.Plan("givens", g, g, 1, pairs, angles, beta)
    e5 = np.zeros((1, g))
    e5[0, 5] = 1.0
    y, _ = oracle.activation_transform(e5, plan)
    c, s = math.cos(float(th)), math.sin(float(th))
    assert y[0, 5] == pytest.approx(c, abs=1e-15)
    assert y[0, 77] == pytest.approx(s * math.exp(-0.5), abs=1e-15)
    # scale-then-rotate would have mixed the scaled channel 77 back into channel 5
    e77 = np.zeros((1, g))
    e77[0, 77] = 1.0
    y77, _ = oracle.activation_transform(e77, plan)
    assert y77[0, 5] == pytest.approx(-s, abs=1e-15)
    assert y77[0, 77] == pytest.approx(c * math.exp(-0.5), abs=1e-15)


# -------------------------------------------------------------- pair selection (A1)
@pytest.mark.parametrize("K,N", [(8, 64), (16, 64), (4, 20)])
def test_select_pairs_properties(K, N):
    g = 128
    P = oracle.select_pairs(1234 + K, 2 * g, g, K, N)
    assert P.shape == (2, K, g // 2, 2)
    for gi in range(2):
        used = set()
        for l in range(K):
            sl = [tuple(p) for p in P[gi, l] if p[0] != oracle.NONE]
            # slots after the first empty one are empty
            n = len(sl)
            assert all(P[gi, l, k, 0] == oracle.NONE for k in range(n, g // 2))
            assert n <= N
            chans = [c for p in sl for c in p]
            assert len(chans) == len(set(chans))                   # disjoint in the layer
            assert all(0 <= i < j < g for i, j in sl)              # inside the group, i < j
            assert not (set(sl) & used)                            # never reused
            if l == 0:
                assert n == min(N, g // 2)
            if n < N:
                # Greedy scan of the whole candidate list: no still-unused pair joins two
                # channels this layer left unmatched.
                free = sorted(set(range(g)) - set(chans))
                for a in range(len(free)):
                    for b in range(a + 1, len(free)):
                        assert (free[a], free[b]) in used
            used |= set(sl)


def test_select_pairs_tiny_bruteforce():
    # g = 4 has 6 pairs and 3 perfect matchings; with K = 3 and N = 2 the greedy layers
    # must be exactly the 3 perfect matchings (each pair used once), in some order.
    P = oracle.select_pairs(7, 4, 4, 3, 2)
    layers = [frozenset(tuple(p) for p in P[0, l] if p[0] != oracle.NONE) for l in range(3)]
    assert set(layers) == {frozenset({(0, 1), (2, 3)}), frozenset({(0, 2), (1, 3)}),
                           frozenset({(0, 3), (1, 2)})}


def test_select_pairs_deterministic():
    a = oracle.select_pairs(99, 256, 128, 4, 64)
    assert np.array_equal(a, oracle.select_pairs(99, 256, 128, 4, 64))
    assert not np.array_equal(a, oracle.select_pairs(100, 256, 128, 4, 64))


# ------------------------------------------------------- equivalence (Fig. 2(a))
def _plans():
    pairs, angles = random_givens(5)
    beta = (rng(3).standard_normal(256) * 0.1).astype(np.float32)
    return [oracle.Plan("hadamard", 256),
            oracle.Plan("givens", 256, 128, 8, pairs, angles, beta),
            oracle.Plan("smooth_hadamard", 256),
            oracle.Plan("smooth_hadamard", 256, smooth_after_rotate=True)]


@pytest.mark.parametrize("pi", range(4))
def test_equivalence_before_quantisation(pi):
    plan = _plans()[pi]
    x = rng(4).standard_normal((100, 256)) * np.where(np.arange(256) % 37 == 0, 30.0, 1.0)
    w = rng(5).standard_normal((64, 256)) * 0.02
    y, s = oracle.activation_transform(x, plan)
    sw = None if s is None else s[0]
    wt = oracle.weight_transform(w, plan, sw)
    ref = x @ w.T
    err = np.linalg.norm(y @ wt.T - ref) / np.linalg.norm(ref)
    assert err < 1e-6
    if plan.kind == "smooth_hadamard":
        # the smoothing actually bounds every channel of the (rotated) operand by 1
        z = y if plan.smooth_after_rotate else oracle.hadamard_rotate(y, 128)
        assert np.max(np.abs(z)) <= 1.0 + 1e-12


# --------------------------------------------------------------------- quantisation
def brute_quantize(y, g):
    """Per element with Python floats and Python's round (half to even)."""
    rows, D = y.shape
    codes = np.zeros((rows, D), dtype=np.int64)
    scales = np.zeros((rows, D // g))
    for r in range(rows):
        for G in range(D // g):
            grp = [float(v) for v in y[r, G * g:(G + 1) * g]]
            m = max(abs(v) for v in grp)
            scales[r, G] = m / 7
            for k, v in enumerate(grp):
                codes[r, G * g + k] = 0 if m == 0 else max(-8, min(7, round(7 * v / m)))
    return codes, scales


def test_quantize_bruteforce_and_bounds():
    y = rng(6).standard_normal((6, 256)) * np.array([1, 10, 1e-3, 100, 1, 1])[:, None]
    y[5, :128] = 0.0                                      # a zero group
    q = oracle.quantize(y, 128)
    bc, bs = brute_quantize(y, 128)
    assert np.array_equal(q.codes, bc)
    assert np.array_equal(q.scales, bs.astype(np.float32))
    assert q.codes.min() >= -8 and q.codes.max() <= 7
    for r in range(6):
        for G in range(2):
            grp = y[r, G * 128:(G + 1) * 128]
            c = q.codes[r, G * 128:(G + 1) * 128]
            s = float(q.scales[r, G])
            if s == 0:
                assert np.all(c == 0)
                continue
            k = np.argmax(np.abs(grp))
            assert c[k] == (7 if grp[k] > 0 else -7)             # absmax -> +-7
            # dequantisation error <= scale/2 (plus the float32 rounding of the scale)
            assert np.max(np.abs(grp - c * s)) <= s / 2 * (1 + 1e-6) + 7 * s * 2 ** -24


def test_quantize_special_cases():
    y = np.zeros((3, 128))
    y[0, 17] = -3.5                                       # single non-zero
    y[1] = 2.0                                            # all equal
    y[2, 0] = 7.0
    y[2, 1] = 2.5                                         # exact tie 2.5 -> 2 (half even)
    y[2, 2] = 3.5                                         # exact tie 3.5 -> 4
    q = oracle.quantize(y, 128)
    assert q.codes[0, 17] == -7 and np.count_nonzero(q.codes[0]) == 1
    assert np.all(q.codes[1] == 7)
    assert q.codes[2, 1] == 2 and q.codes[2, 2] == 4
    assert q.near_tie[2, 1] and q.near_tie[2, 2] and not q.near_tie[2, 0]
    # codes are invariant under a power-of-two rescale; the scale follows it exactly
    x = rng(7).standard_normal((4, 256))
    a, b = oracle.quantize(x, 128), oracle.quantize(x * 2.0 ** -7, 128)
    assert np.array_equal(a.codes, b.codes)
    assert np.array_equal(a.scales * np.float32(2.0 ** -7), b.scales)


def test_pack_golden_and_roundtrip():
    with open(os.path.join(GOLD, "nibbles.txt")) as f:
        for l in f:
            if not l.strip() or l.startswith("#"):
                continue
            c, b = l.split("|")
            codes = np.array([int(v) for v in c.split()], dtype=np.int8)
            want = np.array([int(v, 16) for v in b.split()], dtype=np.uint8)
            assert np.array_equal(oracle.pack_nibbles(codes), want)
            assert np.array_equal(oracle.unpack_nibbles(want), codes)
    allb = np.arange(256, dtype=np.uint8)
    assert np.array_equal(oracle.pack_nibbles(oracle.unpack_nibbles(allb)), allb)


# ------------------------------------------------------------------------ smoothing
def test_smoothing_bruteforce():
    x = rng(8).laplace(size=(300, 16))
    x[:, 3] = 0.0
    s = oracle.smooth_scales(x, 128)
    assert s.shape == (3, 16)
    for b in range(3):
        for j in range(16):
            m = 0.0
            for t in range(b * 128, min(300, (b + 1) * 128)):
                m = max(m, abs(float(x[t, j])))
            assert s[b, j] == (m if m > 0 else 1.0)
    z = oracle.apply_smoothing(x, s, 128)
    for b in range(3):
        blk = np.abs(z[b * 128:(b + 1) * 128])
        assert np.all(np.max(blk, axis=0)[[j for j in range(16) if j != 3]] == 1.0)
        assert np.all(blk[:, 3] == 0.0)


# ------------------------------------------------------------------------------ GEMM
def test_gemm_bruteforce_tiny():
    T, N, D, g = 3, 5, 256, 128
    ca, sa = inputs.random_codes(21, T, D)
    cw, sw = inputs.random_codes(22, N, D)
    res = oracle.gemm(ca, sa, cw, sw, g)
    qa, qw = oracle.unpack_nibbles(ca), oracle.unpack_nibbles(cw)
    for t in range(T):
        for n in range(N):
            acc = np.float32(0.0)
            exact = []
            for G in range(D // g):
                d = 0
                for k in range(G * g, (G + 1) * g):
                    d += int(qa[t, k]) * int(qw[n, k])        # Python ints: exact
                s = np.float32(sa[t, G]) * np.float32(sw[n, G])
                acc = np.float32(acc + np.float32(s * np.float32(d)))
                exact.append(float(sa[t, G]) * float(sw[n, G]) * d)
            assert res.y32[t, n] == acc
            assert res.y64[t, n] == pytest.approx(math.fsum(exact), rel=1e-15, abs=1e-300)


def test_gemm_closed_forms_and_dequant_product():
    D, g = 512, 128
    ones = oracle.pack_nibbles(np.ones((4, D), dtype=np.int8))
    unit = np.ones((4, D // g), dtype=np.float32)
    r = oracle.gemm(ones, unit, ones, unit, g)
    assert np.all(r.y32 == D) and np.all(r.y64 == D)
    ca, sa = inputs.random_codes(31, 40, D)
    cw, sw = inputs.random_codes(32, 24, D)
    r = oracle.gemm(ca, sa, cw, sw, g)
    deq_a = oracle.unpack_nibbles(ca) * np.repeat(sa.astype(np.float64), g, axis=1)
    deq_w = oracle.unpack_nibbles(cw) * np.repeat(sw.astype(np.float64), g, axis=1)
    ref = deq_a @ deq_w.T
    assert np.allclose(r.y64, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # fp32 accumulation stays within its rounding bound of the exact sum
    bound = (D // g + 2) * 2.0 ** -24 * (np.abs(deq_a) @ np.abs(deq_w).T)
    assert np.all(np.abs(r.y32 - r.y64) <= bound + 1e-30)


def test_bf16_round():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -3.0 - 2 ** -7], dtype=np.float32)
    assert oracle.bf16_round(v).tolist() == [1.0, 1.0, 1.0 + 2 ** -7, -3.0]


# -------------------------------------------------------------- planted mistakes
def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def _q8(orig):
    """Mutant: rounds y / (m / 8) instead of y / (m / 7)."""
    def f(y, g, tie_band=1e-3):
        q = orig(y, g, tie_band)
        codes = np.clip(np.rint(q.ratio * 8 / 7), -8, 7).astype(np.int8)
        return O.Quantized(codes, q.scales, q.ratio, q.near_tie)
    return f


def _negated_beta(orig):
    """Mutant: the same transform with beta replaced by -beta (flips the side that carries
    exp(+beta); applied to both sides the product x w^T is unchanged)."""
    def f(a, plan, *rest):
        flipped = oracle.Plan(plan.kind, plan.D, plan.g, plan.K, plan.pairs, plan.angles,
                              None if plan.beta is None else -plan.beta, plan.smooth_after_rotate)
        return orig(a, flipped, *rest)
    return f


def _scale_first(orig, sign):
    """Mutant: Givens applies exp(sign * beta) before the rotations instead of after them
    (on both sides the product x w^T is again unchanged)."""
    def f(a, plan, *rest):
        if plan.kind != "givens" or plan.beta is None:
            return orig(a, plan, *rest)
        y = O.givens_rotate(a * np.exp(sign * plan.beta.astype(np.float64)), plan.pairs, plan.angles, plan.g)
        return (y, None) if sign < 0 else y
    return f


MUTANTS = {
    "givens_sign_swapped": (
        "givens_rotate",
        lambda orig: (lambda x, p, a, g, inverse=False: orig(x, p, -a, g, inverse)),
        test_givens_closed_forms),
    "hadamard_unnormalised": (
        "hadamard_rotate",
        lambda orig: (lambda x, g: orig(x, g) * math.sqrt(g)),
        test_hadamard_rotation_orthonormal_and_involutive),
    "quantise_by_8": ("quantize", lambda orig: _q8(orig), test_quantize_bruteforce_and_bounds),
    "weight_scale_wrong_direction": (
        "weight_transform",
        lambda orig: (lambda w, plan, sw=None: orig(w, oracle.Plan(
            plan.kind, plan.D, plan.g, plan.K, plan.pairs, plan.angles,
            None if plan.beta is None else -plan.beta, plan.smooth_after_rotate), sw)),
        lambda: test_equivalence_before_quantisation(1)),
    # exp(+beta) on the activations and exp(-beta) on the weights: the product is unchanged,
    # so only the closed form of the page's W^ = diag(exp(beta)) W can catch it.
    "channel_scale_both_sides_flipped": (
        ("activation_transform", "weight_transform"),
        (lambda orig: _negated_beta(orig), lambda orig: _negated_beta(orig)),
        test_channel_scale_direction_closed_form),
    "channel_scale_before_rotation": (
        ("activation_transform", "weight_transform"),
        (lambda orig: _scale_first(orig, -1.0), lambda orig: _scale_first(orig, +1.0)),
        test_channel_scale_follows_the_rotations),
    "weight_rotation_transposed": (
        "weight_transform",
        lambda orig: (lambda w, plan, sw=None: orig(w, plan, sw) if plan.kind != "givens" else
                      O.givens_rotate(w, plan.pairs, plan.angles, plan.g, inverse=True)
                      * np.exp(plan.beta.astype(np.float64))),
        lambda: test_equivalence_before_quantisation(1)),
    "nibbles_swapped": (
        "pack_nibbles",
        lambda orig: (lambda c: orig(np.asarray(c).reshape(-1, 2)[:, ::-1].reshape(np.shape(c)))),
        test_pack_golden_and_roundtrip),
    "gemm_drops_last_group": (
        "group_dots",
        lambda orig: (lambda a, w, g: np.concatenate([orig(a, w, g)[:-1],
                                                      0 * orig(a, w, g)[-1:]])),
        test_gemm_bruteforce_tiny),
    "smoothing_ignores_sign": (
        "smooth_scales",
        lambda orig: (lambda x, block=128: orig(np.maximum(x, 0), block)),
        test_smoothing_bruteforce),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    attrs, makes, pin = MUTANTS[name]
    if isinstance(attrs, str):
        attrs, makes = (attrs,), (makes,)
    for attr, make in zip(attrs, makes):
        orig = getattr(O, attr)
        monkeypatch.setattr(O, attr, make(orig))
        monkeypatch.setattr(oracle, attr, getattr(O, attr))
    assert _fails(pin), f"pin did not catch mutant {name}"


@pytest.mark.parametrize("name", ["channel_scale_both_sides_flipped", "channel_scale_before_rotation"])
def test_two_sided_mutants_keep_the_product(name, monkeypatch):
    """The two-sided channel-scale mutants leave (x M)(w M^-T)^T = x w^T intact, so the
    equivalence pin alone cannot see them: only the closed forms above can."""
    attrs, makes, _ = MUTANTS[name]
    for attr, make in zip(attrs, makes):
        orig = getattr(O, attr)
        monkeypatch.setattr(O, attr, make(orig))
        monkeypatch.setattr(oracle, attr, getattr(O, attr))
    test_equivalence_before_quantisation(1)
