"""GPU parity of 8-bit outlier groups (ParoQuant page §4.1: extreme outliers keep an 8-bit
representation) against the oracle.

The library writes an 8-bit group as four 4-bit groups of digits (q = 16 q_hi + q_lo) with
power-of-two scale factors.  The tests decode that layout back into 8-bit codes and one scale,
check every redundant digit copy and scale factor, and compare with the oracle's mixed
quantisation: codes bit-exact outside the 1e-3 tie band (within 1 inside it), scales within the
float32 error of each transform.  The W4A4 GEMM on the digit layout must give the oracle's mixed
GEMM of the same codes (1e-5 relative Frobenius), the fused call the same result as the two
calls, and the mixed plan must track X W^T better than the INT4 plan on outlier groups.
"""
import numpy as np
import pytest

import oracle
from rotation_int4_w4a4_b200 import inputs
from tests.helpers import to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

RTOL = {"hadamard": 1e-5, "givens": 2e-4}


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def rel_fro(a, b):
    return float(np.linalg.norm(a.astype(np.float64) - b) / max(np.linalg.norm(b), 1e-300))


def plans(pq, kind, D, groups8, K=8):
    if kind == "givens":
        pairs = oracle.select_pairs(41, D, 128, K, 64)
        angles = ((inputs.uniform01(42, (D // 128) * K * 64) * 2 - 1) * np.pi).astype(np.float32)
        angles = angles.reshape(D // 128, K, 64)
        beta = inputs.normal(43, D, 0.1).astype(np.float32)
        return (pq.Plan("givens", D, K=K, pairs=pairs, angles=angles, beta=beta, groups8=groups8),
                oracle.Plan("givens", D, 128, K, pairs, angles, beta))
    return pq.Plan("hadamard", D, groups8=groups8), oracle.Plan("hadamard", D)


def decode(codes, scales, D, groups8, weights):
    """The digit layout -> (int codes [rows, D], scales [rows, D/128]), checking the copies."""
    G = D // 128
    q = oracle.unpack_nibbles(codes).astype(np.int64)
    s = scales.astype(np.float64)
    out_q = q[:, :D].copy()
    out_s = s[:, :G].copy()
    for j, gi in enumerate(groups8):
        slot = lambda k: q[:, k * 128:(k + 1) * 128]
        a, b, c = G + 3 * j, G + 3 * j + 1, G + 3 * j + 2
        hi = slot(gi)
        lo = slot(a) if weights else slot(b)
        assert np.array_equal(slot(b) if weights else slot(a), hi)
        assert np.array_equal(slot(c), lo)
        out_q[:, gi * 128:(gi + 1) * 128] = 16 * hi + lo
        s8 = s[:, c]
        assert np.array_equal(s[:, gi], 16 * s8)
        assert np.array_equal(s[:, a], s8 if weights else 16 * s8)
        assert np.array_equal(s[:, b], 16 * s8 if weights else s8)
        out_s[:, gi] = s8
    return out_q, out_s


def assert_close_codes(q, ref):
    diff = np.abs(q - ref.q.codes.astype(np.int64))
    bad = (diff != 0) & ~ref.q.near_tie
    assert not bad.any(), f"{bad.sum()} codes differ away from ties"
    assert diff.max(initial=0) <= 1


def assert_scales(s, ref_s, rtol):
    ref_s = ref_s.astype(np.float64)
    zero = ref_s == 0
    assert np.all(s[zero] == 0)
    assert np.max(np.abs(s[~zero] - ref_s[~zero]) / ref_s[~zero], initial=0) <= rtol


def run(pq, plan, bits, weights):
    import torch
    rows = bits.shape[0]
    codes = torch.empty((rows, plan.Dx // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((rows, plan.Gx), dtype=torch.float32, device="cuda")
    (pq.pq_pack_weights if weights else pq.pq_transform_quant)(plan, to_dev_bf16(bits), codes, scales)
    pq.pq_check_status(plan)
    return codes, scales


CASES = [("hadamard", [1]), ("hadamard", [0, 5, 7]), ("givens", [3]), ("givens", [0, 1, 2, 3, 4, 5, 6, 7])]


@pytest.mark.parametrize("kind,groups8", CASES)
@pytest.mark.parametrize("T", [1, 130])
def test_transform_quant(pq, kind, groups8, T):
    D = 1024
    xb = np.ascontiguousarray(inputs.workload("sweep", T=T).X[:, :D])
    plan, oplan = plans(pq, kind, D, groups8)
    codes, scales = run(pq, plan, xb, False)
    q, s = decode(codes.cpu().numpy(), scales.cpu().numpy(), D, groups8, False)
    ref = oracle.transform_quant_mixed(xb, oplan, groups8)
    assert_close_codes(q, ref)
    assert_scales(s, ref.scales, RTOL[kind])
    assert np.abs(q).max() <= 119


@pytest.mark.parametrize("kind,groups8", CASES)
def test_pack_weights(pq, kind, groups8):
    D, N = 1024, 272
    W = inputs.to_bf16_bits(inputs.normal(300, N * D, 0.02).reshape(N, D))
    plan, oplan = plans(pq, kind, D, groups8)
    codes, scales = run(pq, plan, W, True)
    q, s = decode(codes.cpu().numpy(), scales.cpu().numpy(), D, groups8, True)
    ref = oracle.pack_weights_mixed(W, oplan, groups8)
    assert_close_codes(q, ref)
    assert_scales(s, ref.scales, RTOL[kind])


@pytest.mark.parametrize("kind,groups8", CASES)
@pytest.mark.parametrize("T,N", [(16, 512), (300, 768)])
def test_gemm_and_fused_call(pq, kind, groups8, T, N):
    """GEMM on the digit layout = the oracle's mixed GEMM on the decoded codes; the fused call
    gives the same Y as transform + GEMM."""
    import torch
    D = 1024
    xb = np.ascontiguousarray(inputs.workload("sweep", T=T).X[:, :D])
    W = inputs.to_bf16_bits(inputs.normal(301 + N, N * D, 0.02).reshape(N, D))
    plan, oplan = plans(pq, kind, D, groups8)
    ca, sa = run(pq, plan, xb, False)
    cw, sw = run(pq, plan, W, True)
    Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    pq.pq_w4a4_gemm(ca, sa, cw, sw, Y)
    pq.pq_check_status()
    qa, sa_d = decode(ca.cpu().numpy(), sa.cpu().numpy(), D, groups8, False)
    qw, sw_d = decode(cw.cpu().numpy(), sw.cpu().numpy(), D, groups8, True)
    ref = oracle.gemm_mixed(qa, sa_d.astype(np.float32), qw, sw_d.astype(np.float32), 128)
    assert rel_fro(Y.cpu().numpy(), ref.y64) < 1e-5
    Y2 = torch.full((T, N), float("nan"), dtype=torch.float32, device="cuda")
    ca2 = torch.zeros_like(ca)
    sa2 = torch.full_like(sa, 2.0)
    pq.pq_w4a4_linear(plan, to_dev_bf16(xb), ca2, sa2, cw, sw, Y2)
    pq.pq_check_status(plan)
    assert np.array_equal(Y2.cpu().numpy(), Y.cpu().numpy())


def test_outlier_groups_track_xw_better(pq):
    """On activations with outlier channels, keeping their groups at 8 bits brings Y closer to
    X W^T than the all-INT4 plan (the point of the page's remedy)."""
    import torch
    T, D, N = 256, 4096, 512
    xb = np.ascontiguousarray(inputs.workload("sweep", T=T).X)          # 8 channels x30
    W = inputs.to_bf16_bits(inputs.normal(302, N * D, 0.02).reshape(N, D))
    x = oracle.bf16_to_f64(xb)
    outl = np.argsort(-np.abs(x).max(axis=0))[:8]
    groups8 = sorted(set(int(c) // 128 for c in outl))
    exact = x @ oracle.bf16_to_f64(W).T
    errs = []
    for g8 in ([], groups8):
        plan = pq.Plan("hadamard", D, groups8=g8 or None)
        ca, sa = run(pq, plan, xb, False)
        cw, sw = run(pq, plan, W, True)
        Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
        pq.pq_w4a4_gemm(ca, sa, cw, sw, Y)
        pq.pq_check_status(plan)
        errs.append(rel_fro(Y.cpu().numpy(), exact))
    assert errs[1] < errs[0]
