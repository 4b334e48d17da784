"""Pins for the oracle's rotated runtime smoothing pipeline (RRS page, main equation and Fig. 4):
brute force on small inputs, the page's own invariance (reordering leaves Y unchanged), the
exact product before quantisation, a one-group closed form, and planted mistakes that must
each fail a pin."""
import math

import numpy as np
import pytest

import oracle
from oracle import oracle as O
from rotation_int4_w4a4_b200 import inputs


def bits(x):
    return inputs.to_bf16_bits(x)


def sample(T=40, D=384, N=24, seed=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, D)) * np.where(np.arange(D) % 41 == 0, 25.0, 1.0)
    w = rng.standard_normal((N, D)) * 0.02
    return bits(x), bits(w)


def test_prepare_bruteforce():
    """Channel maxima of the rotated activations over all rows, the descending order (ties by
    index) and the per-group maxima, computed element by element in Python."""
    xb, _ = sample(T=9, D=256)
    p = oracle.rrs_prepare(xb, 128)
    xr = oracle.hadamard_rotate_explicit(oracle.bf16_to_f64(xb), 128)
    D = 256
    m = [max(abs(float(xr[t, j])) for t in range(9)) for j in range(D)]
    assert np.allclose(p.chan_max, m, rtol=1e-13, atol=0)
    order = sorted(range(D), key=lambda j: (-p.chan_max[j], j))
    assert p.perm.tolist() == order
    for G in range(2):
        assert p.group_scale[G] == max(p.chan_max[order[G * 128:(G + 1) * 128]])
    # descending: every group's scale is its first member's maximum and the scales fall
    assert p.group_scale[0] >= p.group_scale[1]
    assert sorted(p.perm.tolist()) == list(range(D))


def test_prepare_ties_and_zero_group():
    """Equal maxima keep index order; an all-zero group gets scale 1."""
    x = np.zeros((4, 256))
    x[:, :128] = 1.0                               # group 0 rotates to (sqrt(128), 0, ...)
    p = oracle.rrs_prepare(bits(x), 128)
    assert p.perm[0] == 0                           # the single non-zero channel comes first
    assert p.perm[1:].tolist() == list(range(1, 256))   # then every zero channel, by index
    assert p.group_scale[1] == 1.0
    assert p.group_scale[0] == pytest.approx(math.sqrt(128.0), rel=1e-15)


def test_reordering_and_smoothing_leave_the_product_unchanged():
    """Before quantisation: sum_k (X_rot[:, perm] / s)_k (W_rot[:, perm])_k s_G(k) = X W^T
    (Fig. 4 (1): the order of the channels does not change Y; the smoothing scale is undone)."""
    xb, wb = sample()
    p = oracle.rrs_prepare(xb, 128)
    a = oracle.rrs_transform_quant(xb, p, 128).y
    w = oracle.rrs_pack_weights(wb, p, 128).y
    y = (a * np.repeat(p.group_scale, 128)) @ w.T
    ref = oracle.bf16_to_f64(xb) @ oracle.bf16_to_f64(wb).T
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 1e-12


def test_one_group_closed_form():
    """D = g: one group, so the smoothing divides every channel by the same s and per-token
    quantisation is scale invariant: the codes equal those of X_rot quantised per row, and
    token scale x s equals that row's plain scale."""
    xb, _ = sample(T=11, D=128)
    p = oracle.rrs_prepare(xb, 128)
    r = oracle.rrs_transform_quant(xb, p, 128)
    xr = oracle.hadamard_rotate(oracle.bf16_to_f64(xb), 128)[:, p.perm]
    plain = oracle.quantize(xr, 128)
    assert np.array_equal(r.q.codes, plain.codes)
    assert np.allclose(r.scales.astype(np.float64) * p.group_scale[0], plain.scales[:, 0], rtol=1e-6)
    assert p.group_scale[0] == np.max(np.abs(xr))


def test_per_token_quantisation_bruteforce():
    xb, _ = sample(T=5, D=256)
    p = oracle.rrs_prepare(xb, 128)
    r = oracle.rrs_transform_quant(xb, p, 128)
    for t in range(5):
        row = [float(v) for v in r.y[t]]
        m = max(abs(v) for v in row)
        assert r.scales[t] == np.float32(m / 7)
        assert [int(c) for c in r.q.codes[t]] == [max(-8, min(7, round(7 * v / m))) for v in row]
    assert np.max(np.abs(r.y)) <= 1.0 + 1e-12        # smoothing bounds every channel by 1


def test_gemm_bruteforce_and_folded_scales():
    xb, wb = sample(T=3, D=256, N=5)
    p = oracle.rrs_prepare(xb, 128)
    a = oracle.rrs_transform_quant(xb, p, 128)
    w = oracle.rrs_pack_weights(wb, p, 128)
    # folded weight scale = plain group scale x smoothing scale
    plain = oracle.quantize(w.y, 128).scales
    assert np.array_equal(w.scales, (plain * p.group_scale.astype(np.float32)[None, :]).astype(np.float32))
    res = oracle.rrs_gemm(a.codes, a.scales, w.codes, w.scales, 128)
    qa, qw = oracle.unpack_nibbles(a.codes), oracle.unpack_nibbles(w.codes)
    for t in range(3):
        for n in range(5):
            acc = np.float32(0.0)
            for G in range(2):
                d = sum(int(qa[t, k]) * int(qw[n, k]) for k in range(G * 128, (G + 1) * 128))
                acc = np.float32(acc + np.float32(np.float32(w.scales[n, G]) * np.float32(d)))
            assert res.y32[t, n] == np.float32(acc * np.float32(a.scales[t]))


def test_quantised_product_tracks_xw():
    """After quantisation the pipeline still approximates X W^T: the error is bounded by the
    per-element dequantisation errors (half a scale each side), summed over the channels."""
    xb, wb = sample(T=16, D=384, N=32)
    p = oracle.rrs_prepare(xb, 128)
    a = oracle.rrs_transform_quant(xb, p, 128)
    w = oracle.rrs_pack_weights(wb, p, 128)
    y = oracle.rrs_gemm(a.codes, a.scales, w.codes, w.scales, 128).y64
    x = oracle.bf16_to_f64(xb)
    ref = x @ oracle.bf16_to_f64(wb).T
    s = np.repeat(p.group_scale, 128)
    ea = a.scales.astype(np.float64)[:, None] / 2 * s[None, :]          # |error| per activation element
    ew = np.repeat(oracle.quantize(w.y, 128).scales.astype(np.float64), 128, axis=1) / 2
    bound = np.abs(a.y * s) @ ew.T + ea @ (np.abs(w.y) + ew).T
    assert np.all(np.abs(y - ref) <= bound * (1 + 1e-6) + 1e-12)


# -------------------------------------------------------------- planted mistakes
def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def _ascending(orig):
    def f(x_bits, g=128):
        p = orig(x_bits, g)
        D = p.chan_max.size
        perm = np.lexsort((np.arange(D), p.chan_max))
        s = p.chan_max[perm].reshape(D // g, g).max(axis=1)
        s[s == 0] = 1
        return O.RRSPrep(p.chan_max, perm, s)
    return f


def _unsorted_groups(orig):
    def f(x_bits, g=128):
        p = orig(x_bits, g)
        D = p.chan_max.size
        s = p.chan_max.reshape(D // g, g).max(axis=1)   # scales of the original channel order
        s[s == 0] = 1
        return O.RRSPrep(p.chan_max, p.perm, s)
    return f


def _unfolded(orig):
    def f(w_bits, prep, g=128):
        r = orig(w_bits, prep, g)
        return O.TQResult(r.codes, oracle.quantize(r.y, g).scales, None, r.q, r.y)
    return f


def _per_group_act(orig):
    def f(x_bits, prep, g=128):
        r = orig(x_bits, prep, g)
        q = oracle.quantize(r.y, g)
        return O.TQResult(oracle.pack_nibbles(q.codes), q.scales[:, 0].copy(), None, q, r.y)
    return f


MUTANTS = {
    "order_ascending": ("rrs_prepare", _ascending, test_prepare_bruteforce),
    "group_scales_before_reordering": ("rrs_prepare", _unsorted_groups, test_prepare_bruteforce),
    "smoothing_not_folded_into_weights": ("rrs_pack_weights", _unfolded, test_gemm_bruteforce_and_folded_scales),
    "per_group_activation_quantisation": ("rrs_transform_quant", _per_group_act, test_per_token_quantisation_bruteforce),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    attr, make, pin = MUTANTS[name]
    monkeypatch.setattr(O, attr, make(getattr(O, attr)))
    monkeypatch.setattr(oracle, attr, getattr(O, attr))
    assert _fails(pin), f"pin did not catch mutant {name}"

