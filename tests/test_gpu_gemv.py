"""GPU parity of the CUDA-core W4A4 kernel (at most 4 tokens: decode) against the oracle; the
same checks run at 5 to 16 tokens, on the tensor-core few-token kernel that takes over there.

The kernel computes each group's integer dot product with __dp4a on q * 16 operands (256 d,
exact in int32) and sums the scaled group terms in an order of its own (ascending per lane,
then a shuffle tree over the warp's group slots).  Acceptance: with unit scales Y is the integer
sum of the dots, exactly (every partial sum is an integer below 2^24); with random scales every
element lies within the float32 summation bound (G + 2) u sum_G |d sw sa| (u = 2^-24) of the
exact value, which is also what fixes the 1e-5 relative Frobenius bound of the other GEMM tests.
Shapes cover every token bucket (1, 2, 4 with tokens past T masked), ragged K (the
last 512-byte K-step partly past the row), one-group rows, the three group sizes, both
outputs, the row-scale mode and the fused call.
"""
import numpy as np
import pytest

import oracle
from rotation_int4_w4a4_b200 import inputs
from tests.helpers import to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def run(pq, ca, sa, cw, sw, g=128, out="f32", rrs=False):
    import torch
    T, N = ca.shape[0], cw.shape[0]
    Y = torch.full((T, N), float("nan"), dtype=torch.float32 if out == "f32" else torch.bfloat16, device="cuda")
    if rrs:
        pq.pq_rrs_gemm(to_dev(ca), to_dev(sa), to_dev(cw), to_dev(sw), Y)
    else:
        pq.pq_w4a4_gemm(to_dev(ca), to_dev(sa), to_dev(cw), to_dev(sw), Y, g=g)
    pq.pq_check_status()
    return Y.float().cpu().numpy()


def summation_bound(ca, sa, cw, sw, g):
    d = np.abs(oracle.group_dots(ca, cw, g).astype(np.float64))
    G = d.shape[0]
    return (G + 2) * U * np.einsum("gtn,tg,ng->tn", d, sa.astype(np.float64), sw.astype(np.float64))


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 7, 8, 9, 12, 15, 16])
@pytest.mark.parametrize("N,D", [(16, 128), (272, 640), (96, 4224)])
def test_random_codes_every_token_count(pq, T, N, D):
    """D = 640 and 4224: the last K-step is partly past the row (320 and 2112 packed bytes)."""
    ca, sa = inputs.random_codes(9100 + T, T, D)
    cw, sw = inputs.random_codes(9200 + N + D, N, D)
    Y = run(pq, ca, sa, cw, sw)
    r = oracle.gemm(ca, sa, cw, sw)
    assert np.all(np.abs(Y - r.y64) <= summation_bound(ca, sa, cw, sw, 128))


@pytest.mark.parametrize("g", [64, 128, 256])
@pytest.mark.parametrize("T", [1, 6, 16])
def test_unit_scales_exact(pq, g, T):
    """Unit scales: Y = sum over groups of the integer dots, bit for bit, including the extremes
    (all -8 against all -8: 64 g per group) and codes with mixed signs."""
    D, N = 2048, 144
    ca, _ = inputs.random_codes(9300 + T + g, T, D, g)
    cw, _ = inputs.random_codes(9400 + g, N, D, g)
    ca[0] = 0x88
    cw[0] = 0x88
    cw[1] = 0x77
    cw[2] = 0x78                                      # alternating 8 and 7 nibbles: -8, 7
    ones_a = np.ones((T, D // g), np.float32)
    ones_w = np.ones((N, D // g), np.float32)
    Y = run(pq, ca, ones_a, cw, ones_w, g)
    d = oracle.group_dots(ca, cw, g).sum(axis=0)
    assert Y[0, 0] == 64 * D
    assert np.array_equal(Y.astype(np.int64), d)


@pytest.mark.parametrize("g", [64, 256])
@pytest.mark.parametrize("T,N,D", [(1, 4096, 4096), (3, 272, 1280), (11, 512, 2048)])
def test_group_sizes(pq, g, T, N, D):
    ca, sa = inputs.random_codes(9500 + T, T, D, g)
    cw, sw = inputs.random_codes(9600 + N, N, D, g)
    Y = run(pq, ca, sa, cw, sw, g)
    r = oracle.gemm(ca, sa, cw, sw, g)
    assert np.all(np.abs(Y - r.y64) <= summation_bound(ca, sa, cw, sw, g))


@pytest.mark.parametrize("T", [2, 13])
def test_bf16_output(pq, T):
    """bf16 Y: the float32 result rounded once (one bf16 ulp of the oracle away from heavy
    cancellation, the summation bound plus half an ulp everywhere)."""
    D, N = 1024, 400
    ca, sa = inputs.random_codes(9700 + T, T, D)
    cw, sw = inputs.random_codes(9701, N, D)
    Y = run(pq, ca, sa, cw, sw, out="bf16")
    r = oracle.gemm(ca, sa, cw, sw)
    S = summation_bound(ca, sa, cw, sw, 128)
    assert np.all(np.abs(Y - r.y64) <= 2.0 ** -8 * np.abs(Y) + S)
    ref = oracle.bf16_round(r.y32)
    ulp = np.maximum(np.abs(ref), 2.0 ** -126) * 2.0 ** -7
    clear = np.abs(r.y64) > S / ((D // 128 + 2) * U) * 2.0 ** -7
    assert np.all((np.abs(Y - ref) <= ulp)[clear])


@pytest.mark.parametrize("T", [1, 5, 16])
def test_row_scale_mode(pq, T):
    """Rotated runtime smoothing's GEMM: per-(row, group) factors and one scale per token."""
    D, N = 1024, 272
    ca, _ = inputs.random_codes(9800 + T, T, D)
    cw, sw = inputs.random_codes(9801, N, D)
    ts = (np.exp(inputs.normal(9802 + T, T, 0.5)) * 0.05).astype(np.float32)
    Y = run(pq, ca, ts, cw, sw, rrs=True)
    r = oracle.rrs_gemm(ca, ts, cw, sw, 128)
    d = np.abs(oracle.group_dots(ca, cw, 128).astype(np.float64))
    S = (D // 128 + 2) * U * ts.astype(np.float64)[:, None] * np.einsum("gtn,ng->tn", d, sw.astype(np.float64))
    assert np.all(np.abs(Y - r.y64) <= S + U * np.abs(r.y64))


@pytest.mark.parametrize("kind,g", [("hadamard", 64), ("givens", 128), ("hadamard", 256)])
@pytest.mark.parametrize("T", [3, 16])
def test_fused_call_matches_two_calls(pq, kind, g, T):
    """pq_w4a4_linear launches the kernel as the transform's programmatic dependent (weight
    loads before the wait): Y equals transform + GEMM as two calls, bit for bit."""
    import torch
    D, N = 1024, 528
    X = np.ascontiguousarray(inputs.workload("sweep", T=T).X[:, :D])
    W = inputs.to_bf16_bits(inputs.normal(9900 + N, N * D, 0.02).reshape(N, D))
    if kind == "givens":
        pairs = oracle.select_pairs(97, D, g, 8, g // 2)
        angles = ((inputs.uniform01(98, (D // g) * 8 * (g // 2)) * 2 - 1) * np.pi).astype(np.float32)
        plan = pq.Plan("givens", D, g=g, K=8, pairs=pairs, angles=angles.reshape(D // g, 8, g // 2),
                       beta=inputs.normal(99, D, 0.1).astype(np.float32))
    else:
        plan = pq.Plan(kind, D, g=g)
    G = D // g
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device="cuda")
    sw = torch.empty((N, G), dtype=torch.float32, device="cuda")
    pq.pq_pack_weights(plan, to_dev_bf16(W), cw, sw)
    Xd = to_dev_bf16(X)
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device="cuda")
    sa = torch.empty((T, G), dtype=torch.float32, device="cuda")
    Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    pq.pq_transform_quant(plan, Xd, ca, sa)
    pq.pq_w4a4_gemm(ca, sa, cw, sw, Y, g=g)
    Y2 = torch.full((T, N), float("nan"), dtype=torch.float32, device="cuda")
    ca2 = torch.zeros_like(ca)
    sa2 = torch.full_like(sa, 2.0)
    pq.pq_w4a4_linear(plan, Xd, ca2, sa2, cw, sw, Y2)
    pq.pq_check_status(plan)
    assert np.array_equal(Y2.cpu().numpy(), Y.cpu().numpy())
    r = oracle.gemm(ca.cpu().numpy(), sa.cpu().numpy(), cw.cpu().numpy(), sw.cpu().numpy(), g)
    assert float(np.linalg.norm(Y.cpu().numpy() - r.y64) / np.linalg.norm(r.y64)) < 1e-5
