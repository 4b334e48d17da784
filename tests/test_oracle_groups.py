"""Pins for the oracle at group sizes 64 and 256 (ParoQuant page §4.1: a smaller group, g = 64,
for layers with many outliers; §6, cross-platform advice: g = 256 on mobile parts).

Every check builds its expectation independently of the oracle's own code: the Walsh-Hadamard
matrix from its entry definition (-1)^popcount(i & j), Givens layers as explicit products of
2 x 2 plane rotations, quantisation and group dot products by brute force in Python.  The last
section plants g-handling mistakes in the oracle and shows that a pin catches each.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import oracle as O


def rng(seed=1):
    return np.random.default_rng(seed)


def hadamard_by_entries(n):
    """H[i][j] = (-1)^popcount(i & j) (Hadamard page §2.1, the entry definition)."""
    return np.array([[(-1.0) ** bin(i & j).count("1") for j in range(n)] for i in range(n)])


def block_rotation(D, g):
    """x -> x M with M = diag(H_g / sqrt(g), ..., H_g / sqrt(g)) (Hadamard page §6.1: blocks)."""
    M = np.zeros((D, D))
    H = hadamard_by_entries(g) / math.sqrt(g)
    for b in range(D // g):
        M[b * g:(b + 1) * g, b * g:(b + 1) * g] = H
    return M


@pytest.mark.parametrize("g", [64, 256])
def test_hadamard_rotation_matches_entry_definition(g):
    D = 512
    x = rng(g).standard_normal((5, D))
    M = block_rotation(D, g)
    assert np.allclose(M @ M.T, np.eye(D), atol=1e-12)           # orthonormal blocks
    assert np.allclose(oracle.hadamard_rotate(x, g), x @ M, rtol=0, atol=1e-12)
    # groups do not mix: a row confined to one group stays in it
    x1 = np.zeros((1, D))
    x1[0, g:2 * g] = rng(3).standard_normal(g)
    y1 = oracle.hadamard_rotate(x1, g)
    assert np.all(y1[0, :g] == 0) and np.all(y1[0, 2 * g:] == 0)


@pytest.mark.parametrize("g", [64, 256])
def test_hadamard_closed_form_first_channel(g):
    """e_0 of each group rotates to the constant 1/sqrt(g) over the group; quantised, every code
    is 7 and the scale is 1/(7 sqrt(g))."""
    x = np.zeros((1, 2 * g))
    x[0, 0] = 1.0
    x[0, g] = -1.0
    y = oracle.hadamard_rotate(x, g)
    assert np.allclose(y[0, :g], 1 / math.sqrt(g), atol=1e-15)
    assert np.allclose(y[0, g:], -1 / math.sqrt(g), atol=1e-15)
    q = oracle.quantize(y, g)
    assert np.all(q.codes[0, :g] == 7) and np.all(q.codes[0, g:] == -7)
    assert q.scales[0, 0] == np.float32(1 / math.sqrt(g) / 7)


@pytest.mark.parametrize("g", [64, 256])
def test_quantize_bruteforce(g):
    y = rng(10 + g).standard_normal((3, 512)) * np.array([1.0, 1e3, 1e-3])[:, None]
    y[1, 5] = 0.0
    y[2, g:2 * g] = 0.0                                        # an all-zero group
    q = oracle.quantize(y, g)
    for t in range(3):
        for G in range(512 // g):
            seg = [float(v) for v in y[t, G * g:(G + 1) * g]]
            m = max(abs(v) for v in seg)
            assert q.scales[t, G] == np.float32(m / 7)
            want = [0] * g if m == 0 else [max(-8, min(7, round(7 * v / m))) for v in seg]
            assert q.codes[t, G * g:(G + 1) * g].tolist() == want


def test_select_pairs_g64_properties():
    """ParoQuant page §2.2: within a layer the pairs are disjoint; across layers no pair repeats;
    every index lies in its 64-channel group."""
    K, N = 6, 32
    p = oracle.select_pairs(7, 256, 64, K, N)
    assert p.shape == (4, K, 32, 2)
    for gi in range(4):
        seen_pairs = set()
        for l in range(K):
            used = set()
            for i, j in p[gi, l]:
                if i == oracle.NONE:
                    continue
                assert i < j < 64
                assert i not in used and j not in used
                used |= {int(i), int(j)}
                assert (int(i), int(j)) not in seen_pairs
                seen_pairs.add((int(i), int(j)))


def explicit_givens(pairs_g, angles_g, g):
    """Product of the layers' 2 x 2 plane rotations for the row-vector convention y = x R:
    each pair (i, j, theta) contributes the identity except R[i,i] = R[j,j] = cos theta,
    R[i,j] = sin theta, R[j,i] = -sin theta; layers multiply in order."""
    R = np.eye(g)
    for l in range(pairs_g.shape[0]):
        L = np.eye(g)
        for (i, j), th in zip(pairs_g[l], angles_g[l]):
            if i == oracle.NONE:
                continue
            c, s = math.cos(float(th)), math.sin(float(th))
            L[i, i] = L[j, j] = c
            L[i, j] = s
            L[j, i] = -s
        R = R @ L
    return R


def test_givens_g64_matches_explicit_product():
    g, G, K = 64, 3, 5
    pairs = oracle.select_pairs(21, G * g, g, K, g // 2)
    angles = rng(22).uniform(-np.pi, np.pi, size=(G, K, g // 2)).astype(np.float32)
    x = rng(23).standard_normal((4, G * g))
    y = oracle.givens_rotate(x, pairs, angles, g)
    for gi in range(G):
        R = explicit_givens(pairs[gi], angles[gi], g)
        assert np.allclose(R @ R.T, np.eye(g), atol=1e-12)
        assert np.allclose(y[:, gi * g:(gi + 1) * g], x[:, gi * g:(gi + 1) * g] @ R, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind,g", [("givens", 64), ("hadamard", 64), ("hadamard", 256)])
def test_transform_pair_keeps_the_product(kind, g):
    """Before quantisation (x M)(w M^-T)^T = x w^T (RRS page, Fig. 2(a); OSTQuant page §3.2)."""
    D = 512
    if kind == "givens":
        pairs = oracle.select_pairs(31, D, g, 4, g // 2)
        angles = rng(32).uniform(-np.pi, np.pi, size=(D // g, 4, g // 2)).astype(np.float32)
        beta = (rng(33).standard_normal(D) * 0.3).astype(np.float32)
        plan = oracle.Plan("givens", D, g, 4, pairs, angles, beta)
    else:
        plan = oracle.Plan("hadamard", D, g)
    x = rng(34).standard_normal((6, D))
    w = rng(35).standard_normal((9, D))
    a, _ = oracle.activation_transform(x, plan)
    b = oracle.weight_transform(w, plan)
    ref = x @ w.T
    assert np.linalg.norm(a @ b.T - ref) / np.linalg.norm(ref) < 1e-12


@pytest.mark.parametrize("g", [64, 256])
def test_gemm_bruteforce(g):
    """Integer dots per group and the float32 sum over groups in ascending order, element by
    element in Python."""
    T, N, D = 2, 3, 512
    r = rng(40 + g)
    qa = r.integers(-8, 8, size=(T, D))
    qw = r.integers(-8, 8, size=(N, D))
    sa = (r.uniform(0.01, 1.0, size=(T, D // g))).astype(np.float32)
    sw = (r.uniform(0.01, 1.0, size=(N, D // g))).astype(np.float32)
    ca, cw = oracle.pack_nibbles(qa), oracle.pack_nibbles(qw)
    d = oracle.group_dots(ca, cw, g)
    res = oracle.gemm(ca, sa, cw, sw, g)
    for t in range(T):
        for n in range(N):
            acc = np.float32(0.0)
            for G in range(D // g):
                dd = sum(int(qa[t, k]) * int(qw[n, k]) for k in range(G * g, (G + 1) * g))
                assert d[G, t, n] == dd
                acc = np.float32(acc + np.float32(np.float32(sa[t, G] * sw[n, G]) * np.float32(dd)))
            assert res.y32[t, n] == acc


# -------------------------------------------------------------- planted mistakes
def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def _quantize_fixed_128(orig):
    return lambda y, g, tie_band=1e-3: orig(y, 128, tie_band)


def _hadamard_fixed_128(orig):
    return lambda x, g: orig(x, 128)


def _dots_fixed_128(orig):
    return lambda ca, cw, g: orig(ca, cw, 128)


MUTANTS = {
    "quantize_ignores_g": ("quantize", _quantize_fixed_128, test_quantize_bruteforce, 64),
    "hadamard_ignores_g": ("hadamard_rotate", _hadamard_fixed_128, test_hadamard_rotation_matches_entry_definition, 256),
    "dots_ignore_g": ("group_dots", _dots_fixed_128, test_gemm_bruteforce, 64),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    attr, make, pin, g = MUTANTS[name]
    monkeypatch.setattr(O, attr, make(getattr(O, attr)))
    monkeypatch.setattr(oracle, attr, getattr(O, attr))
    assert _fails(pin, g), f"pin did not catch mutant {name}"
