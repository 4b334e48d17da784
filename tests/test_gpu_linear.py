"""pq_w4a4_linear (transform + GEMM in one call; for T <= 128 the GEMM is the transform's
programmatic dependent) against the two separate calls and the oracle.

The activation buffers are filled with other codes and scales before every call, so a GEMM that
read them before the transform had written them would give a different Y.  Codes and Y must
equal those of pq_transform_quant followed by pq_w4a4_gemm bit for bit (the same kernels in the
same order), and the whole chain must track the oracle's.
"""
import numpy as np
import pytest

import oracle
from rotation_int4_w4a4_b200 import inputs
from tests.helpers import to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def make_plan(pq, kind, D, g):
    if kind == "givens":
        pairs = oracle.select_pairs(77, D, g, 16, g // 2)
        angles = ((inputs.uniform01(78, (D // g) * 16 * (g // 2)) * 2 - 1) * np.pi).astype(np.float32)
        beta = inputs.normal(79, D, 0.1).astype(np.float32)
        return pq.Plan("givens", D, g=g, K=16, pairs=pairs, angles=angles.reshape(D // g, 16, g // 2), beta=beta)
    return pq.Plan(kind, D, g=g)


@pytest.mark.parametrize("kind,g", [("hadamard", 128), ("givens", 128), ("smooth_hadamard", 128), ("hadamard", 64),
                                    ("hadamard", 256), ("givens", 64)])
@pytest.mark.parametrize("T,N", [(1, 4096), (16, 1024), (100, 272), (128, 512), (129, 256), (300, 512)])
def test_linear_equals_separate_calls(pq, kind, g, T, N):
    import torch
    D = 2048
    X = np.ascontiguousarray(inputs.workload("sweep", T=T).X[:, :D])
    W = inputs.to_bf16_bits(inputs.normal(123 + N, N * D, 0.02).reshape(N, D))
    plan = make_plan(pq, kind, D, g)
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
    pq.pq_check_status(plan)
    ca_ref, sa_ref, y_ref = ca.cpu().numpy(), sa.cpu().numpy(), Y.cpu().numpy()
    for rep in range(3):
        ca2 = torch.full((T, D // 2), 0x77 - rep, dtype=torch.uint8, device="cuda")   # other codes
        sa2 = torch.full((T, G), 3.0 + rep, dtype=torch.float32, device="cuda")
        Y2 = torch.full((T, N), float("nan"), dtype=torch.float32, device="cuda")
        pq.pq_w4a4_linear(plan, Xd, ca2, sa2, cw, sw, Y2)
        pq.pq_check_status(plan)
        assert np.array_equal(ca2.cpu().numpy(), ca_ref)
        assert np.array_equal(sa2.cpu().numpy(), sa_ref)
        assert np.array_equal(Y2.cpu().numpy(), y_ref)


def test_linear_tracks_oracle_chain(pq):
    import torch
    T, N, D = 8, 512, 1024
    X = np.ascontiguousarray(inputs.workload("sweep", T=T).X[:, :D])
    W = inputs.to_bf16_bits(inputs.normal(5, N * D, 0.02).reshape(N, D))
    plan = pq.Plan("hadamard", D)
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device="cuda")
    sw = torch.empty((N, D // 128), dtype=torch.float32, device="cuda")
    pq.pq_pack_weights(plan, to_dev_bf16(W), cw, sw)
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device="cuda")
    sa = torch.empty((T, D // 128), dtype=torch.float32, device="cuda")
    Y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    pq.pq_w4a4_linear(plan, to_dev_bf16(X), ca, sa, cw, sw, Y)
    pq.pq_check_status(plan)
    op = oracle.Plan("hadamard", D)
    a = oracle.transform_quant(X, op)
    w = oracle.pack_weights(W, op)
    ref = oracle.gemm(a.codes, a.scales, w.codes, w.scales).y64
    got = Y.float().cpu().numpy()
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-2
    own = oracle.gemm(ca.cpu().numpy(), sa.cpu().numpy(), cw.cpu().numpy(), sw.cpu().numpy()).y64
    assert np.all(np.abs(got - own) <= 2.0 ** -8 * np.abs(own) + 1e-6 * np.abs(own).max())
