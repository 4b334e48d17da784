"""GPU parity of rotated runtime smoothing with channel reordering (RRS page, main equation and
Fig. 4) against the oracle.

- pq_rrs_prepare: channel maxima within float32 error of the oracle's float64 ones; the order
  is a permutation that sorts the library's own maxima (descending, ties by index) and equals
  the oracle's wherever neighbouring maxima differ by more than that error; each group's scale
  is its first member's maximum.
- pq_rrs_transform_quant / pq_rrs_pack_weights, given the oracle's order and scales: codes
  bit-exact outside the 1e-3 tie band (within 1 inside it), scales within float32 error.
- pq_rrs_gemm: the oracle's GEMM on the same codes and scales within 1e-5 relative Frobenius
  (bf16: one ulp), on both the few-token and the CTA-pair kernels, split and unsplit.
- The whole chain on the GPU tracks X W^T as closely as the oracle's chain does.
"""
import numpy as np
import pytest

import oracle
from rotation_int4_w4a4_b200 import inputs
from tests.helpers import assert_codes_match, assert_scales_close, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

RTOL_MAX = 2e-5      # float32 tensor-core rotation vs float64: a few ulps of |y|
RTOL_SCALE = 2e-5


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def rel_fro(a, b):
    return float(np.linalg.norm(a.astype(np.float64) - b) / max(np.linalg.norm(b), 1e-300))


def prepare_gpu(pq, plan, X_bits, D):
    import torch
    G = D // 128
    cm = torch.empty(D, dtype=torch.float32, device="cuda")
    perm = torch.empty(D, dtype=torch.int32, device="cuda")
    inv = torch.empty(D, dtype=torch.int32, device="cuda")
    gs = torch.empty(G, dtype=torch.float32, device="cuda")
    pq.pq_rrs_prepare(plan, to_dev_bf16(X_bits), cm, perm, inv, gs)
    pq.pq_check_status(plan)
    return cm.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy(), gs.cpu().numpy()


def workload_x(name, T=None, D=None):
    wl = inputs.workload(name, T=T, with_weights=False)
    X = wl.X if D is None else wl.X[:, :D]
    return np.ascontiguousarray(X)


@pytest.mark.parametrize("name,T,D", [("down_proj", 5, 1024), ("down_proj", 300, 2048), ("q_proj", 129, 4096),
                                      ("down_proj", 1000, 14336)])
def test_prepare(pq, name, T, D):
    X = workload_x(name, T, D)
    plan = pq.Plan("hadamard", D)
    cm, perm, inv, gs = prepare_gpu(pq, plan, X, D)
    ref = oracle.rrs_prepare(X, 128)
    assert np.allclose(cm, ref.chan_max, rtol=RTOL_MAX, atol=0)
    assert sorted(perm.tolist()) == list(range(D))
    assert np.array_equal(inv[perm], np.arange(D))
    # the library's order sorts its own maxima: descending, equal maxima by index
    c = cm[perm]
    assert np.all((c[:-1] > c[1:]) | ((c[:-1] == c[1:]) & (perm[:-1] < perm[1:])))
    # and agrees with the oracle's wherever the oracle's neighbours are well separated
    rm = ref.chan_max[ref.perm]
    gap = np.minimum(np.append(np.inf, rm[:-1] - rm[1:]), np.append(rm[:-1] - rm[1:], np.inf))
    sure = gap > 4 * RTOL_MAX * np.maximum(rm, 1e-30)
    assert np.array_equal(perm[sure], ref.perm[sure])
    assert np.array_equal(gs, np.where(cm[perm[::128]] > 0, cm[perm[::128]], 1.0).astype(np.float32))


def test_prepare_zero_channels(pq):
    """All-zero groups: every maximum 0, order by index, scales 1."""
    D = 384
    X = inputs.to_bf16_bits(np.zeros((7, D)))
    X[:, 0] = inputs.to_bf16_bits(np.full(7, 2.0))   # one non-zero input channel (group 0)
    plan = pq.Plan("hadamard", D)
    cm, perm, _, gs = prepare_gpu(pq, plan, X, D)
    ref = oracle.rrs_prepare(X, 128)
    assert np.allclose(cm, ref.chan_max, rtol=RTOL_MAX, atol=0)
    assert np.array_equal(perm, ref.perm)
    assert gs[1] == 1.0 and gs[2] == 1.0


@pytest.mark.parametrize("name,T,D", [("down_proj", 3, 1024), ("down_proj", 130, 2048), ("q_proj", 64, 4096),
                                      ("down_proj", 257, 14336)])
def test_transform_quant(pq, name, T, D):
    import torch
    X = workload_x(name, T, D)
    ref_p = oracle.rrs_prepare(X, 128)
    plan = pq.Plan("hadamard", D)
    codes = torch.empty((T, D // 2), dtype=torch.uint8, device="cuda")
    ts = torch.empty(T, dtype=torch.float32, device="cuda")
    pq.pq_rrs_transform_quant(plan, to_dev_bf16(X), to_dev(ref_p.perm.astype(np.int32)),
                              to_dev(ref_p.group_scale.astype(np.float32)), codes, ts)
    pq.pq_check_status(plan)
    ref = oracle.rrs_transform_quant(X, ref_p, 128)
    assert_codes_match(codes.cpu().numpy(), ref)
    assert_scales_close(ts.cpu().numpy(), ref.scales, RTOL_SCALE)


@pytest.mark.parametrize("N,D", [(100, 1024), (272, 4096), (48, 14336)])
def test_pack_weights(pq, N, D):
    import torch
    X = workload_x("down_proj", 200, D)
    W = inputs.to_bf16_bits(inputs.normal(77 + N, N * D, 0.02).reshape(N, D))
    ref_p = oracle.rrs_prepare(X, 128)
    plan = pq.Plan("hadamard", D)
    codes = torch.empty((N, D // 2), dtype=torch.uint8, device="cuda")
    sw = torch.empty((N, D // 128), dtype=torch.float32, device="cuda")
    pq.pq_rrs_pack_weights(plan, to_dev_bf16(W), to_dev(ref_p.perm.astype(np.int32)),
                           to_dev(ref_p.group_scale.astype(np.float32)), codes, sw)
    pq.pq_check_status(plan)
    ref = oracle.rrs_pack_weights(W, ref_p, 128)
    assert_codes_match(codes.cpu().numpy(), ref)
    assert_scales_close(sw.cpu().numpy(), ref.scales, RTOL_SCALE)


@pytest.mark.parametrize("T,N,D,out", [(1, 4096, 4096, "f32"), (16, 272, 1024, "bf16"), (100, 512, 2048, "f32"),
                                       (129, 256, 512, "f32"), (300, 768, 1024, "bf16"), (256, 4096, 4096, "f32")])
def test_gemm(pq, T, N, D, out):
    import torch
    ca, _ = inputs.random_codes(8100 + T, T, D)
    cw, sw = inputs.random_codes(8200 + N, N, D)
    ts = (np.exp(inputs.normal(8300 + T, T, 0.5)) * 0.05).astype(np.float32)
    Y = torch.empty((T, N), dtype=torch.float32 if out == "f32" else torch.bfloat16, device="cuda")
    pq.pq_rrs_gemm(to_dev(ca), to_dev(ts), to_dev(cw), to_dev(sw), Y)
    pq.pq_check_status()
    r = oracle.rrs_gemm(ca, ts, cw, sw, 128)
    got = Y.float().cpu().numpy()
    if out == "f32":
        assert rel_fro(got, r.y64) < 1e-5
    else:
        # The float32 sum over G groups may round differently from the oracle's order (fused
        # multiply-adds), so where the groups cancel, one bf16 ulp of the result is too tight: each
        # element must lie within the float32 summation bound (G + 2) u sum_G |F d| sa (u = 2^-24)
        # of the exact value, plus half a bf16 ulp; away from cancellation, within one bf16 ulp
        # of the rounded oracle value.
        d = oracle.group_dots(ca, cw, 128).astype(np.float64)
        S = ts.astype(np.float64)[:, None] * np.einsum("gtn,ng->tn", np.abs(d), sw.astype(np.float64))
        G = D // 128
        assert np.all(np.abs(got - r.y64) <= 2.0 ** -8 * np.abs(got) + (G + 2) * 2.0 ** -24 * S)
        ref = oracle.bf16_round(r.y32)
        ulp = np.maximum(np.abs(ref), 2.0 ** -126) * 2.0 ** -7
        clear = np.abs(r.y64) > 2.0 ** -7 * S          # no heavy cancellation
        assert np.all((np.abs(got - ref) <= ulp)[clear])


def test_pipeline_tracks_xw(pq):
    """prepare -> transform -> pack -> GEMM on the GPU approximates X W^T as well as the oracle's
    chain (a few near-tie codes may differ; the error to X W^T must not grow)."""
    import torch
    T, D, N = 256, 2048, 512
    X = workload_x("down_proj", T, D)
    W = inputs.to_bf16_bits(inputs.normal(991, N * D, 0.02).reshape(N, D))
    plan = pq.Plan("hadamard", D)
    G = D // 128
    cm = torch.empty(D, dtype=torch.float32, device="cuda")
    perm = torch.empty(D, dtype=torch.int32, device="cuda")
    inv = torch.empty(D, dtype=torch.int32, device="cuda")
    gsc = torch.empty(G, dtype=torch.float32, device="cuda")
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device="cuda")
    ts = torch.empty(T, dtype=torch.float32, device="cuda")
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device="cuda")
    sw = torch.empty((N, G), dtype=torch.float32, device="cuda")
    Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    Xd, Wd = to_dev_bf16(X), to_dev_bf16(W)
    pq.pq_rrs_prepare(plan, Xd, cm, perm, inv, gsc)
    pq.pq_rrs_transform_quant(plan, Xd, perm, gsc, ca, ts)
    pq.pq_rrs_pack_weights(plan, Wd, perm, gsc, cw, sw)
    pq.pq_rrs_gemm(ca, ts, cw, sw, Y)
    pq.pq_check_status(plan)
    ref_xw = oracle.bf16_to_f64(X) @ oracle.bf16_to_f64(W).T
    p = oracle.rrs_prepare(X, 128)
    a = oracle.rrs_transform_quant(X, p, 128)
    w = oracle.rrs_pack_weights(W, p, 128)
    y_or = oracle.rrs_gemm(a.codes, a.scales, w.codes, w.scales, 128).y64
    e_gpu = rel_fro(Y.cpu().numpy(), ref_xw)
    e_or = rel_fro(y_or, ref_xw)
    assert e_gpu <= e_or * 1.01 + 1e-6
    assert rel_fro(Y.cpu().numpy(), y_or) < 1e-2
