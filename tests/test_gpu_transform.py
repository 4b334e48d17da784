"""GPU parity of the fused transform + quantisation kernels against the CPU oracle.

Acceptance: codes bit-exact wherever the oracle's y/scale is more than 1e-3 from a
half-integer, within 1 there; scales within the float32 error bound of each transform;
smoothing scales exact (max of bf16 values) or within float32 error (rotated order).
"""
import numpy as np
import pytest

import oracle
from rotation_int4_w4a4_b200 import inputs
from tests.helpers import (assert_codes_match, assert_scales_close, empty_outputs, oracle_plan,
                           to_dev, to_dev_bf16)

pytestmark = pytest.mark.gpu

# Scale tolerances (relative), from the float32 error of each transform (see design notes):
# Hadamard: 7 pairwise stages -> |dm|/m <= 7u*sqrt(128) + 2u < 5e-6.  Givens: K layers of
# 2-term rotations + channel scale -> about (3K+2)u*sqrt(128)*max(e^beta) < 1e-4 for K<=16.
RTOL_H = 1e-5
RTOL_G = 2e-4


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def run_tq(pq, plan, X_bits, D, smooth=False, ldx=None):
    import torch
    T = X_bits.shape[0]
    if ldx is not None and ldx != D:
        padded = np.zeros((T, ldx), dtype=np.uint16)
        padded[:, :D] = X_bits
        X = to_dev_bf16(padded)
    else:
        X = to_dev_bf16(X_bits)
    codes, scales = empty_outputs(T, D)
    sm = torch.empty(((T + 127) // 128, D), dtype=torch.float32, device="cuda") if smooth else None
    pq.pq_transform_quant(plan, X, codes, scales, sm, T=T, ldx=ldx or D)
    pq.pq_check_status(plan)
    return codes.cpu().numpy(), scales.cpu().numpy(), (sm.cpu().numpy() if smooth else None)


def givens_inputs(wl):
    pairs = oracle.select_pairs(wl.pair_seed, wl.D, wl.g, wl.K, wl.g // 2)
    return pairs, wl.angles, wl.beta


# ------------------------------------------------------------------ Hadamard
@pytest.mark.parametrize("T", [1, 3, 8, 129, 300])
def test_hadamard_small(pq, T):
    wl = inputs.workload("q_proj", T=T)
    plan = pq.Plan("hadamard", wl.D)
    codes, scales, _ = run_tq(pq, plan, wl.X, wl.D)
    ref = oracle.transform_quant(wl.X, oracle_plan("hadamard", wl.D))
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_H)


def test_hadamard_padded_rows(pq):
    wl = inputs.workload("q_proj", T=70)
    plan = pq.Plan("hadamard", wl.D)
    codes, scales, _ = run_tq(pq, plan, wl.X, wl.D, ldx=wl.D + 64)
    ref = oracle.transform_quant(wl.X, oracle_plan("hadamard", wl.D))
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_H)


def edge_rows(D):
    """Zero groups, single non-zero, all-equal, a huge outlier, tiny values, negatives."""
    x = np.random.default_rng(5).standard_normal((8, D)).astype(np.float32)
    x[0] = 0.0
    x[1] = 0.0
    x[1, 5] = -3.0
    x[2] = 1.5
    x[3, 7] = 1e30
    x[4] *= 1e-30
    x[5] = -np.abs(x[5])
    x[6, :128] = 0.0
    return inputs.to_bf16_bits(x)


@pytest.mark.parametrize("kind", ["hadamard", "smooth_hadamard", "givens"])
def test_edge_cases(pq, kind):
    D = 256
    X = edge_rows(D)
    if kind == "givens":
        wl = inputs.workload("tiny")
        pairs, angles, beta = givens_inputs(wl)
        plan = pq.Plan("givens", D, K=wl.K, pairs=pairs, angles=angles, beta=beta)
        oplan = oracle_plan("givens", D, wl.K, pairs, angles, beta)
    else:
        plan = pq.Plan(kind, D)
        oplan = oracle_plan(kind, D)
    codes, scales, sm = run_tq(pq, plan, X, D, smooth=(kind == "smooth_hadamard"))
    ref = oracle.transform_quant(X, oplan)
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_G if kind == "givens" else RTOL_H)
    assert np.all(scales[0] == 0) and np.all(oracle.unpack_nibbles(codes[0]) == 0)
    if sm is not None:
        assert np.array_equal(sm, ref.smooth)


# ------------------------------------------------------------------ Givens
@pytest.mark.parametrize("name,T", [("tiny", None), ("up_proj", 200), ("sweep", 33)])
def test_givens(pq, name, T):
    wl = inputs.workload(name, T=T, kind="givens") if name == "sweep" else inputs.workload(name, T=T)
    pairs, angles, beta = givens_inputs(wl)
    plan = pq.Plan("givens", wl.D, K=wl.K, pairs=pairs, angles=angles, beta=beta)
    codes, scales, _ = run_tq(pq, plan, wl.X, wl.D)
    ref = oracle.transform_quant(wl.X, oracle_plan("givens", wl.D, wl.K, pairs, angles, beta))
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_G)


def test_givens_partial_layers_and_no_beta(pq):
    # Fewer than 64 pairs in some layers (N = 20) and beta absent.
    D, K = 256, 6
    pairs = oracle.select_pairs(77, D, 128, K, 20)
    angles = np.random.default_rng(1).uniform(-np.pi, np.pi, (2, K, 64)).astype(np.float32)
    X = inputs.workload("tiny").X
    plan = pq.Plan("givens", D, K=K, pairs=pairs, angles=angles, beta=None)
    codes, scales, _ = run_tq(pq, plan, X, D)
    ref = oracle.transform_quant(X, oracle_plan("givens", D, K, pairs, angles, None))
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_G)


# ------------------------------------------------------------- smoothing
@pytest.mark.parametrize("after", [False, True])
@pytest.mark.parametrize("T", [5, 128, 300])
def test_smooth_hadamard(pq, after, T):
    wl = inputs.workload("down_proj", T=T)
    X = wl.X[:, :1024]            # 8 groups keeps the oracle fast
    D = 1024
    plan = pq.Plan("smooth_hadamard", D, flags=pq.PQ_FLAG_SMOOTH_AFTER_ROTATE if after else 0)
    codes, scales, sm = run_tq(pq, plan, X, D, smooth=True)
    ref = oracle.transform_quant(X, oracle_plan("smooth_hadamard", D, after=after))
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_H)
    if after:
        assert_scales_close(sm, ref.smooth, RTOL_H)
    else:
        assert np.array_equal(sm, ref.smooth)


# -------------------------------------------------------------- weights
@pytest.mark.parametrize("kind", ["hadamard", "givens", "smooth_hadamard", "smooth_after"])
def test_pack_weights(pq, kind):
    import torch
    wl = inputs.workload("tiny")
    D = wl.D
    W = wl.W[:100]
    smooth_w = None
    if kind == "givens":
        pairs, angles, beta = givens_inputs(wl)
        plan = pq.Plan("givens", D, K=wl.K, pairs=pairs, angles=angles, beta=beta)
        oplan = oracle_plan("givens", D, wl.K, pairs, angles, beta)
    elif kind.startswith("smooth"):
        after = kind == "smooth_after"
        plan = pq.Plan("smooth_hadamard", D, flags=pq.PQ_FLAG_SMOOTH_AFTER_ROTATE if after else 0)
        oplan = oracle_plan("smooth_hadamard", D, after=after)
        smooth_w = np.abs(np.random.default_rng(3).standard_normal(D)).astype(np.float32) + 0.5
    else:
        plan = pq.Plan("hadamard", D)
        oplan = oracle_plan("hadamard", D)
    Wd = to_dev_bf16(W)
    codes, scales = empty_outputs(W.shape[0], D)
    sw = to_dev(smooth_w) if smooth_w is not None else None
    pq.pq_pack_weights(plan, Wd, codes, scales, sw)
    pq.pq_check_status(plan)
    ref = oracle.pack_weights(W, oplan, smooth_w)
    assert_codes_match(codes.cpu().numpy(), ref)
    assert_scales_close(scales.cpu().numpy(), ref.scales, RTOL_G if kind == "givens" else 2 * RTOL_H)


# ----------------------------------------------- full-size, sampled rows
@pytest.mark.parametrize("name", ["q_proj", "up_proj", "down_proj"])
def test_full_size_sampled(pq, name):
    """The launch configuration of the full workloads, checked on sampled row blocks."""
    import torch
    wl = inputs.workload(name, with_weights=False)
    D = wl.D
    if wl.kind == "givens":
        pairs, angles, beta = givens_inputs(wl)
        plan = pq.Plan("givens", D, K=wl.K, pairs=pairs, angles=angles, beta=beta)
        oplan = oracle_plan("givens", D, wl.K, pairs, angles, beta)
    else:
        plan = pq.Plan(wl.kind, D)
        oplan = oracle_plan(wl.kind, D)
    smooth = wl.kind == "smooth_hadamard"
    codes, scales, sm = run_tq(pq, plan, wl.X, D, smooth=smooth)
    nb = (wl.T + 127) // 128
    blocks = sorted({0, nb // 2, nb - 1})
    for b in blocks:
        rows = np.arange(b * 128, min(wl.T, (b + 1) * 128))
        ref = oracle.transform_quant(wl.X[rows], oplan)
        assert_codes_match(codes[rows], ref)
        assert_scales_close(scales[rows], ref.scales, RTOL_G if wl.kind == "givens" else RTOL_H)
        if smooth:
            assert np.array_equal(sm[b], ref.smooth[0])


# ------------------------------------- weights at the workloads' full sizes, sampled rows
@pytest.mark.parametrize("name", ["q_proj", "up_proj", "down_proj"])
def test_pack_weights_full_size_sampled(pq, name):
    """pq_pack_weights on the whole W of each workload, in the launch configuration the
    benchmark uses, compared with the oracle on sampled rows.

    q_proj    Hadamard, W [4096, 4096] on the tensor cores.
    up_proj   Givens K=16 (32 groups of weight-side matrices, exp(+beta)), W [14336, 4096].
    down_proj smoothing + Hadamard, W [4096, 14336] with the register kernel's multi-task loop;
              the channel multiplier is the oracle's own smoothing scale of X's first 128-row
              block (the workload's pre-scaled weights), as float32.
    """
    import torch
    wl = inputs.workload(name)
    D, N = wl.D, wl.N
    smooth_w = None
    if wl.kind == "givens":
        pairs, angles, beta = givens_inputs(wl)
        plan = pq.Plan("givens", D, K=wl.K, pairs=pairs, angles=angles, beta=beta)
        oplan = oracle_plan("givens", D, wl.K, pairs, angles, beta)
    else:
        plan = pq.Plan(wl.kind, D)
        oplan = oracle_plan(wl.kind, D)
        if wl.kind == "smooth_hadamard":
            smooth_w = oracle.smooth_scales(oracle.bf16_to_f64(wl.X[:128]), 128)[0].astype(np.float32)
    codes, scales = empty_outputs(N, D)
    pq.pq_pack_weights(plan, to_dev_bf16(wl.W), codes, scales,
                       to_dev(smooth_w) if smooth_w is not None else None)
    pq.pq_check_status(plan)
    rng = np.random.default_rng(17)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, N // 2, N // 2 + 77, N - 1],
                                     rng.integers(0, N, 9)]))
    rt = torch.from_numpy(rows).cuda()
    ref = oracle.pack_weights(wl.W[rows], oplan, smooth_w)
    assert_codes_match(codes[rt].cpu().numpy(), ref)
    assert_scales_close(scales[rt].cpu().numpy(), ref.scales,
                        RTOL_G if wl.kind == "givens" else 2 * RTOL_H)


# ------------------------------------------------------------ few rows (CUDA-core path)
@pytest.mark.parametrize("kind", ["hadamard", "givens"])
@pytest.mark.parametrize("T", [1, 2, 7, 16, 17])
def test_few_rows(pq, kind, T):
    """Up to 16 rows take the warp-per-tile kernel (shuffle butterflies for Hadamard, the composed
    matrix from L2 for Givens); 17 rows the tensor-core kernel.  Both against the oracle, with the
    up_proj Givens plan (K = 16) and the q_proj Hadamard plan."""
    name = "up_proj" if kind == "givens" else "q_proj"
    wl = inputs.workload(name, T=T)
    if kind == "givens":
        pairs, angles, beta = givens_inputs(wl)
        plan = pq.Plan("givens", wl.D, K=wl.K, pairs=pairs, angles=angles, beta=beta)
        oplan = oracle_plan("givens", wl.D, wl.K, pairs, angles, beta)
        rtol = RTOL_G
    else:
        plan = pq.Plan("hadamard", wl.D)
        oplan = oracle_plan("hadamard", wl.D)
        rtol = RTOL_H
    codes, scales, _ = run_tq(pq, plan, wl.X, wl.D, ldx=wl.D + 64)
    ref = oracle.transform_quant(wl.X, oplan)
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, rtol)
