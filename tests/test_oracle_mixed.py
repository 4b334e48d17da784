"""Pins for the oracle's 8-bit outlier groups (ParoQuant page §4.1, third remedy: extreme
outliers keep an 8-bit representation).

The 8-bit code is read as one byte of two signed 4-bit digits, q = 16 q_hi + q_lo; the digit
split is checked exhaustively, and with it the largest symmetric range, 119.  Quantisation and
the mixed GEMM are checked element by element in Python, the INT4-only case against the plain
functions, and the four-digit-group form of an 8-bit group (what the library's GEMM computes)
against the mixed GEMM.  Planted mistakes must each fail a pin.
"""
import numpy as np
import pytest

import oracle
from oracle import oracle as O


def rng(seed=1):
    return np.random.default_rng(seed)


def split(q):
    """Balanced base-16 digits: q_hi = floor((q + 8) / 16), q_lo = q - 16 q_hi."""
    hi = (q + 8) // 16
    return hi, q - 16 * hi


def test_digit_split_exhaustive_and_range():
    for q in range(-oracle.LEVELS8, oracle.LEVELS8 + 1):
        hi, lo = split(q)
        assert -8 <= hi <= 7 and -8 <= lo <= 7 and 16 * hi + lo == q
    # 119 is the largest symmetric range: +120 needs a high digit of 8
    assert split(120)[0] == 8
    assert oracle.LEVELS8 == 119


def sample(rows=5, D=512, seed=2):
    y = rng(seed).standard_normal((rows, D))
    y[:, 130] *= 200.0                  # group 1 holds an extreme outlier channel
    y[2, 300] = -500.0                  # one spike in group 2
    y[3, 384:] = 0.0                    # an all-zero group
    return y


@pytest.mark.parametrize("groups8", [[1], [1, 2], [0, 3]])
def test_quantize_mixed_bruteforce(groups8):
    y = sample()
    q = oracle.quantize_mixed(y, 128, groups8)
    for t in range(y.shape[0]):
        for G in range(4):
            L = 119 if G in groups8 else 7
            seg = [float(v) for v in y[t, G * 128:(G + 1) * 128]]
            m = max(abs(v) for v in seg)
            assert q.scales[t, G] == np.float32(m / L)
            lo = -L if L == 119 else -8
            want = [0] * 128 if m == 0 else [max(lo, min(L, round(L * v / m))) for v in seg]
            assert q.codes[t, G * 128:(G + 1) * 128].tolist() == want


def test_no_8bit_groups_is_plain_int4():
    y = sample()
    a = oracle.quantize_mixed(y, 128, [])
    b = oracle.quantize(y, 128)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.scales, b.scales)


def test_mixed_reduces_the_outlier_groups_error():
    """In the 8-bit group every dequantisation error is at most half its scale, max|y| / 238
    (17 times below the INT4 bound max|y| / 14), and the RMS error falls; the other groups are
    unchanged."""
    y = sample()
    q4 = oracle.quantize(y, 128)
    q8 = oracle.quantize_mixed(y, 128, [1])
    deq = lambda q: q.codes.astype(np.float64) * np.repeat(q.scales.astype(np.float64), 128, axis=1)
    e4 = np.abs(deq(q4) - y)
    e8 = np.abs(deq(q8) - y)
    g1 = slice(128, 256)
    m = np.abs(y[:, g1]).max(axis=1, keepdims=True)
    assert np.all(e8[:, g1] <= m / 238 * (1 + 1e-6))
    assert np.sqrt((e8[:, g1] ** 2).mean()) < np.sqrt((e4[:, g1] ** 2).mean())
    assert np.array_equal(e8[:, 256:], e4[:, 256:])


def test_gemm_mixed_bruteforce():
    r = rng(7)
    T, N, D = 3, 4, 384
    groups8 = [2]
    qa = r.integers(-8, 8, size=(T, D)).astype(np.int16)
    qw = r.integers(-8, 8, size=(N, D)).astype(np.int16)
    qa[:, 256:] = r.integers(-119, 120, size=(T, 128))
    qw[:, 256:] = r.integers(-119, 120, size=(N, 128))
    sa = r.uniform(0.01, 1, size=(T, 3)).astype(np.float32)
    sw = r.uniform(0.01, 1, size=(N, 3)).astype(np.float32)
    res = oracle.gemm_mixed(qa, sa, qw, sw, 128)
    for t in range(T):
        for n in range(N):
            acc = np.float32(0.0)
            for G in range(3):
                d = sum(int(qa[t, k]) * int(qw[n, k]) for k in range(G * 128, (G + 1) * 128))
                acc = np.float32(acc + np.float32(np.float32(sa[t, G] * sw[n, G]) * np.float32(d)))
            assert res.y32[t, n] == acc


def four_digit_groups(q, s, g8, weights):
    """An 8-bit group as four 4-bit groups: activations (hi, hi, lo, lo) with scales
    (16 s, 16 s, s, s); weights (hi, lo, hi, lo) with (16 s, s, 16 s, s)."""
    hi, lo = split(q.astype(np.int64))
    cols = [hi, lo, hi, lo] if weights else [hi, hi, lo, lo]
    sc = [16 * s, s, 16 * s, s] if weights else [16 * s, 16 * s, s, s]
    return np.concatenate(cols, axis=1), np.stack(sc, axis=1).astype(np.float32)


def test_four_digit_groups_give_the_mixed_product():
    """sum over the four 4-bit groups of (scale products x digit dots) = sa sw d8 exactly."""
    r = rng(9)
    T, N = 5, 6
    qa = r.integers(-119, 120, size=(T, 128))
    qw = r.integers(-119, 120, size=(N, 128))
    sa = r.uniform(0.01, 1, size=T).astype(np.float32)
    sw = r.uniform(0.01, 1, size=N).astype(np.float32)
    A, SA = four_digit_groups(qa, sa, 0, False)
    W, SW = four_digit_groups(qw, sw, 0, True)
    via_digits = oracle.gemm(oracle.pack_nibbles(A), SA, oracle.pack_nibbles(W), SW, 128).y64
    direct = oracle.gemm_mixed(qa, sa[:, None], qw, sw[:, None], 128).y64
    assert np.allclose(via_digits, direct, rtol=1e-13, atol=0)
    assert np.abs(A).max() <= 8 and np.abs(W).max() <= 8


# ------------------------------------------------------------------ planted mistakes
def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def _full_int8_range(orig):
    def f(y, g, groups8, tie_band=1e-3):
        old = O.LEVELS8
        O.LEVELS8 = 127
        try:
            return orig(y, g, groups8, tie_band)
        finally:
            O.LEVELS8 = old
    return f


def _ignores_groups(orig):
    return lambda y, g, groups8, tie_band=1e-3: orig(y, g, [], tie_band)


def _drops_8bit_dots(orig):
    def f(qa, sa, qw, sw, g=128):
        qa = np.where(np.abs(qa) > 8, 0, qa)
        return orig(qa, sa, qw, sw, g)
    return f


MUTANTS = {
    "127_levels": ("quantize_mixed", _full_int8_range, test_quantize_mixed_bruteforce, [1]),
    "groups_ignored": ("quantize_mixed", _ignores_groups, test_quantize_mixed_bruteforce, [1]),
    "8bit_dots_dropped": ("gemm_mixed", _drops_8bit_dots, test_gemm_mixed_bruteforce, None),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    attr, make, pin, arg = MUTANTS[name]
    monkeypatch.setattr(O, attr, make(getattr(O, attr)))
    monkeypatch.setattr(oracle, attr, getattr(O, attr))
    args = () if arg is None else (arg,)
    assert _fails(pin, *args), f"pin did not catch mutant {name}"
