"""GPU parity of the tcgen05 W4A4 GEMM against the CPU oracle on identical codes and scales.

Acceptance: per-group integer dots bit-exact (D = 128, unit scales: Y is the dot itself);
float32 Y within 1e-5 relative Frobenius error of the oracle; bf16 Y within one bf16 ulp of
the round-to-nearest-even of the oracle's float32 result.
"""
import numpy as np
import pytest

import oracle
from rotation_int4_w4a4_b200 import inputs
from tests.helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def run_gemm(pq, ca, sa, cw, sw, out="f32"):
    import torch
    T, N = ca.shape[0], cw.shape[0]
    Y = torch.empty((T, N), dtype=torch.float32 if out == "f32" else torch.bfloat16, device="cuda")
    pq.pq_w4a4_gemm(to_dev(ca), to_dev(sa), to_dev(cw), to_dev(sw), Y)
    pq.pq_check_status()
    return Y.float().cpu().numpy()


def rel_fro(a, b):
    return float(np.linalg.norm(a.astype(np.float64) - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("T,N", [(1, 256), (128, 256), (130, 512), (257, 768), (64, 16)])
def test_dots_bit_exact(pq, T, N):
    """D = 128 (one group) and unit scales: Y[t][n] is the integer dot product itself."""
    ca, _ = inputs.random_codes(101 + T, T, 128)
    cw, _ = inputs.random_codes(202 + N, N, 128)
    ones_a = np.ones((T, 1), np.float32)
    ones_w = np.ones((N, 1), np.float32)
    Y = run_gemm(pq, ca, ones_a, cw, ones_w)
    d = oracle.group_dots(ca, cw, 128)[0]
    assert np.array_equal(Y, d.astype(np.float32))


def test_extreme_codes_bit_exact(pq):
    # all -8 x all -8 gives the largest dot, 128 * 64 = 8192; mixed signs the most negative.
    T, N = 128, 256
    m8 = oracle.pack_nibbles(np.full((T, 128), -8, np.int8))
    p7 = oracle.pack_nibbles(np.full((N, 128), 7, np.int8))
    n8 = oracle.pack_nibbles(np.full((N, 128), -8, np.int8))
    one_a, one_w = np.ones((T, 1), np.float32), np.ones((N, 1), np.float32)
    assert np.all(run_gemm(pq, m8, one_a, n8, one_w) == 8192.0)
    assert np.all(run_gemm(pq, m8, one_a, p7, one_w) == -7168.0)


def adversarial_codes(rows, seed):
    """Codes for one 128-element group whose dot products stress an accumulator of limited
    alignment precision.  The contraction sees each group as four K32 slices: the low nibbles
    of packed bytes 0..31 (even elements 0..62), of bytes 32..63 (even elements 64..126), then
    the high nibbles of bytes 0..31 (odd elements 1..63) and of bytes 32..63 (odd 65..127).
    Row pattern r % 7 puts large equal-sign codes (-8 or 7) in some slices, so that the running
    sum reaches several thousand, and small codes (-5..5, odd and even) elsewhere, so that odd
    products and odd slice sums meet a large partial sum at every slice boundary, in both
    orders."""
    rng = np.random.default_rng(seed)
    slices = [np.arange(0, 64, 2), np.arange(64, 128, 2), np.arange(1, 64, 2), np.arange(65, 128, 2)]
    big_sets = [(0, 1, 2), (1, 2, 3), (0, 2, 3), (0, 1, 3), (3,), (0,), (0, 1, 2, 3)]
    q = np.zeros((rows, 128), dtype=np.int8)
    for r in range(rows):
        big = big_sets[r % len(big_sets)]
        sign_big = -8 if (r // len(big_sets)) % 2 == 0 else 7
        for k, idx in enumerate(slices):
            if k in big:
                q[r, idx] = sign_big
            else:
                q[r, idx] = rng.integers(-5, 6, idx.size).astype(np.int8)
    return oracle.pack_nibbles(q)


def test_adversarial_dots_bit_exact(pq):
    """D = 128, unit scales: every output is one group's integer dot.  Row and column patterns
    combine large slices (|partial sums| up to 96 * 64 = 6144 after three slices and up to
    8192 in total) with odd products in the other slices; all results must be exact."""
    T, N = 192, 384
    ca = adversarial_codes(T, 71)
    cw = adversarial_codes(N, 72)
    Y = run_gemm(pq, ca, np.ones((T, 1), np.float32), cw, np.ones((N, 1), np.float32))
    d = oracle.group_dots(ca, cw, 128)[0]
    assert np.abs(d).max() == 8192 and np.any((d % 2) != 0) and np.any((np.abs(d) > 5000) & (d % 2 != 0))
    assert np.array_equal(Y, d.astype(np.float32))


@pytest.mark.parametrize("T,N,D", [(3, 16, 256), (200, 272, 384), (128, 256, 1024), (333, 1024, 512)])
def test_random_codes_f32(pq, T, N, D):
    ca, sa = inputs.random_codes(7 + T, T, D)
    cw, sw = inputs.random_codes(9 + N, N, D)
    Y = run_gemm(pq, ca, sa, cw, sw)
    ref = oracle.gemm(ca, sa, cw, sw)
    assert rel_fro(Y, ref.y64) < 1e-5
    assert rel_fro(Y, ref.y32) < 1e-5


def test_random_codes_bf16(pq):
    T, N, D = 150, 512, 512
    ca, sa = inputs.random_codes(31, T, D)
    cw, sw = inputs.random_codes(32, N, D)
    Y = run_gemm(pq, ca, sa, cw, sw, out="bf16")
    ref = oracle.bf16_round(oracle.gemm(ca, sa, cw, sw).y32)
    # one bf16 ulp of the reference value
    ulp = np.maximum(np.abs(ref), 2.0 ** -126) * 2.0 ** -7
    assert np.all(np.abs(Y - ref) <= ulp)


@pytest.mark.parametrize("T,N,D,out", [(1, 4096, 4096, "f32"), (16, 512, 2048, "bf16"),
                                       (256, 1024, 4096, "f32"), (3, 4096, 1024, "bf16"),
                                       (1, 272, 4096, "f32"), (5, 16, 1024, "bf16")])
def test_split_k_small_T(pq, T, N, D, out):
    """Few output tiles: the groups are split across CTA pairs and the float32 partial tiles are
    reduced in ascending order; same tolerances as the unsplit path.  N = 272 and N = 16 leave
    the odd CTA of the last pair with no channel inside N."""
    ca, sa = inputs.random_codes(41 + T, T, D)
    cw, sw = inputs.random_codes(43 + N, N, D)
    Y = run_gemm(pq, ca, sa, cw, sw, out=out)
    r = oracle.gemm(ca, sa, cw, sw)
    if out == "f32":
        assert rel_fro(Y, r.y64) < 1e-5
    else:
        ref = oracle.bf16_round(r.y32)
        ulp = np.maximum(np.abs(ref), 2.0 ** -126) * 2.0 ** -7
        assert np.all(np.abs(Y - ref) <= ulp)


def test_oracle_codes_end_to_end_tiny(pq):
    """The tiny Givens workload: the oracle's own activation and weight codes through the GPU GEMM."""
    wl = inputs.workload("tiny")
    pairs = oracle.select_pairs(wl.pair_seed, wl.D, wl.g, wl.K, 64)
    plan = oracle.Plan("givens", wl.D, 128, wl.K, pairs, wl.angles, wl.beta)
    a = oracle.transform_quant(wl.X, plan)
    w = oracle.pack_weights(wl.W, plan)
    Y = run_gemm(pq, a.codes, a.scales, w.codes, w.scales)
    ref = oracle.gemm(a.codes, a.scales, w.codes, w.scales)
    assert rel_fro(Y, ref.y64) < 1e-5


@pytest.mark.parametrize("T,N", [(1, 14336), (16, 4096), (4096, 14336)])
def test_sweep_shapes_sampled(pq, T, N):
    """Decode/prefill sweep shapes at D = 4096 (split and unsplit launches), sampled rows."""
    import torch
    D = 4096
    ca, sa = inputs.random_codes(3000 + T, T, D)
    cw, sw = inputs.random_codes(4000 + N, N, D)
    Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    pq.pq_w4a4_gemm(to_dev(ca), to_dev(sa), to_dev(cw), to_dev(sw), Y)
    pq.pq_check_status()
    rows = np.unique(np.array([0, T // 2, T - 1]))
    Ys = Y[torch.from_numpy(rows).cuda()].cpu().numpy()
    ref = oracle.gemm(ca[rows], sa[rows], cw, sw)
    assert rel_fro(Ys, ref.y64) < 1e-5


@pytest.mark.parametrize("name", ["q_proj", "up_proj", "down_proj"])
def test_full_size_sampled_rows(pq, name):
    """The full workload shapes in the launch configuration the benchmark uses, checked on a
    few sampled rows (first, middle, last tile) against the oracle."""
    import torch
    wl = inputs.workload(name, with_weights=False)
    T, N, D = wl.T, wl.N, wl.D
    ca, sa = inputs.random_codes(1000 + T, T, D)
    cw, sw = inputs.random_codes(2000 + N, N, D)
    Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    pq.pq_w4a4_gemm(to_dev(ca), to_dev(sa), to_dev(cw), to_dev(sw), Y)
    pq.pq_check_status()
    rows = np.array([0, 1, 127, T // 2, T // 2 + 77, T - 1])
    Ys = Y[torch.from_numpy(rows).cuda()].cpu().numpy()
    ref = oracle.gemm(ca[rows], sa[rows], cw, sw)
    assert rel_fro(Ys, ref.y64) < 1e-5


# ------------------------------------------------------- few-token kernel (T <= 128)
@pytest.mark.parametrize("T,N,D,out", [(1, 16, 128, "f32"), (2, 272, 384, "f32"), (15, 512, 1024, "bf16"),
                                       (16, 4096, 4096, "f32"), (17, 144, 256, "f32"), (33, 1024, 512, "bf16"),
                                       (64, 4096, 4096, "f32"), (65, 400, 640, "f32"), (100, 272, 1280, "bf16"),
                                       (128, 1024, 2048, "f32"), (129, 256, 512, "f32")])
def test_few_tokens(pq, T, N, D, out):
    """T <= 128 runs the few-token kernel (packed codes widened in the kernel, int8 MMAs, N = T
    rounded up to 16/32/64/128): token counts on both sides of each width, ragged N (past the
    last 128-row weight tile), group-range splits (small T) and single launches (T = 64, 128).
    T = 129 is the first call on the CTA-pair kernel."""
    ca, sa = inputs.random_codes(5000 + T, T, D)
    cw, sw = inputs.random_codes(6000 + N, N, D)
    Y = run_gemm(pq, ca, sa, cw, sw, out=out)
    r = oracle.gemm(ca, sa, cw, sw)
    if out == "f32":
        assert rel_fro(Y, r.y64) < 1e-5
    else:
        ref = oracle.bf16_round(r.y32)
        ulp = np.maximum(np.abs(ref), 2.0 ** -126) * 2.0 ** -7
        assert np.all(np.abs(Y - ref) <= ulp)


def test_few_tokens_adversarial_dots_bit_exact(pq):
    """Unit scales and D = 128 through the int8 path: each output is 256 d / 256, exact."""
    T, N = 96, 384
    ca = adversarial_codes(T, 81)
    cw = adversarial_codes(N, 82)
    Y = run_gemm(pq, ca, np.ones((T, 1), np.float32), cw, np.ones((N, 1), np.float32))
    assert np.array_equal(Y, oracle.group_dots(ca, cw, 128)[0].astype(np.float32))


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_few_tokens_match_unsplit_order(pq, T):
    """The split group ranges (summed in ascending order) agree with the oracle's ascending
    float32 accumulation to within float32 rounding, at the sweep's decode sizes."""
    D, N = 4096, 14336
    ca, sa = inputs.random_codes(7000 + T, T, D)
    cw, sw = inputs.random_codes(7100, N, D)
    Y = run_gemm(pq, ca, sa, cw, sw)
    r = oracle.gemm(ca, sa, cw, sw)
    assert rel_fro(Y, r.y64) < 1e-5
    assert rel_fro(Y, r.y32) < 1e-5
