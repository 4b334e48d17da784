"""GPU parity at group sizes 64 and 256 (ParoQuant page §4.1: g = 64 for layers with many
outliers; §6: g = 256 on mobile parts) against the oracle.

- pq_transform_quant / pq_pack_weights: block Hadamard at g = 64 and 256, Givens (with the
  channel scale) at g = 64: codes bit-exact outside the 1e-3 tie band, within 1 inside it; scales
  within the float32 error of each transform.  Ragged row counts, several row tiles.
- pq_w4a4_gemm at g = 64 and 256: integer dots bit-exact at D = max(g, 128) (the largest
  |d| = 2^14 at g = 256); float32 Y within 1e-5 relative Frobenius, bf16 within one ulp, on both kernels
  (few-token and CTA-pair), split and unsplit; the whole chain against the oracle's.
"""
import numpy as np
import pytest

import oracle
from rotation_int4_w4a4_b200 import inputs
from tests.helpers import assert_codes_match, assert_scales_close, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

RTOL_H = 1e-5
RTOL_G = 2e-4


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def rel_fro(a, b):
    return float(np.linalg.norm(a.astype(np.float64) - b) / max(np.linalg.norm(b), 1e-300))


def givens_parts(seed, D, g, K):
    pairs = oracle.select_pairs(seed, D, g, K, g // 2)
    angles = ((inputs.uniform01(seed + 1, (D // g) * K * (g // 2)) * 2.0 - 1.0) * np.pi).astype(np.float32)
    beta = inputs.normal(seed + 2, D, 0.1).astype(np.float32)
    return pairs, angles.reshape(D // g, K, g // 2), beta


def plans(pq, kind, D, g, K=8, seed=501):
    if kind == "givens":
        pairs, angles, beta = givens_parts(seed, D, g, K)
        return (pq.Plan("givens", D, g=g, K=K, pairs=pairs, angles=angles, beta=beta),
                oracle.Plan("givens", D, g, K, pairs, angles, beta))
    return pq.Plan("hadamard", D, g=g), oracle.Plan("hadamard", D, g)


def run_tq(pq, plan, X_bits, D, g, weights=False):
    import torch
    T = X_bits.shape[0]
    codes = torch.empty((T, D // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((T, D // g), dtype=torch.float32, device="cuda")
    if weights:
        pq.pq_pack_weights(plan, to_dev_bf16(X_bits), codes, scales)
    else:
        pq.pq_transform_quant(plan, to_dev_bf16(X_bits), codes, scales)
    pq.pq_check_status(plan)
    return codes.cpu().numpy(), scales.cpu().numpy()


CASES = [("hadamard", 64), ("hadamard", 256), ("givens", 64)]


@pytest.mark.parametrize("kind,g", CASES)
@pytest.mark.parametrize("T", [1, 5, 129, 300])
def test_transform_quant(pq, kind, g, T):
    wl = inputs.workload("sweep", T=T)          # X [T, 4096], 8 outlier channels x30
    plan, oplan = plans(pq, kind, wl.D, g)
    codes, scales = run_tq(pq, plan, wl.X, wl.D, g)
    ref = oracle.transform_quant(wl.X, oplan)
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_G if kind == "givens" else RTOL_H)


@pytest.mark.parametrize("kind,g", CASES)
def test_transform_edge_rows(pq, kind, g):
    """Zero rows and groups, one non-zero channel, a huge outlier, tiny values."""
    D = 512
    x = np.random.default_rng(9).standard_normal((6, D))
    x[0] = 0.0
    x[1] = 0.0
    x[1, 70] = -3.0
    x[2, :g] = 0.0
    x[3, 7] = 1e30
    x[4] *= 1e-30
    xb = inputs.to_bf16_bits(x)
    plan, oplan = plans(pq, kind, D, g, K=4)
    codes, scales = run_tq(pq, plan, xb, D, g)
    ref = oracle.transform_quant(xb, oplan)
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_G if kind == "givens" else RTOL_H)


@pytest.mark.parametrize("kind,g", CASES)
@pytest.mark.parametrize("N", [100, 272])
def test_pack_weights(pq, kind, g, N):
    D = 1024
    W = inputs.to_bf16_bits(inputs.normal(600 + N, N * D, 0.02).reshape(N, D))
    plan, oplan = plans(pq, kind, D, g)
    codes, scales = run_tq(pq, plan, W, D, g, weights=True)
    ref = oracle.pack_weights(W, oplan)
    assert_codes_match(codes, ref)
    assert_scales_close(scales, ref.scales, RTOL_G if kind == "givens" else RTOL_H)


def run_gemm(pq, ca, sa, cw, sw, g, out="f32"):
    import torch
    T, N = ca.shape[0], cw.shape[0]
    Y = torch.empty((T, N), dtype=torch.float32 if out == "f32" else torch.bfloat16, device="cuda")
    pq.pq_w4a4_gemm(to_dev(ca), to_dev(sa), to_dev(cw), to_dev(sw), Y, g=g)
    pq.pq_check_status()
    return Y.float().cpu().numpy()


@pytest.mark.parametrize("g", [64, 256])
@pytest.mark.parametrize("T,N", [(1, 256), (100, 272), (130, 512), (257, 768)])
def test_dots_bit_exact(pq, g, T, N):
    """D = max(g, 128) (one group, or two at g = 64) and unit scales: Y is the sum of the integer
    dots itself; the first rows take the extremes (all -8 against all -8: d = 64 g per group)."""
    D = max(g, 128)
    ca, _ = inputs.random_codes(700 + T, T, D, g)
    cw, _ = inputs.random_codes(800 + N, N, D, g)
    ca[0] = 0x88
    cw[0] = 0x88
    cw[1] = 0x77
    ones_a = np.ones((T, D // g), np.float32)
    ones_w = np.ones((N, D // g), np.float32)
    Y = run_gemm(pq, ca, ones_a, cw, ones_w, g)
    d = oracle.group_dots(ca, cw, g).sum(axis=0)
    assert Y[0, 0] == 64 * D
    assert np.array_equal(Y.astype(np.int64), d)


@pytest.mark.parametrize("g", [64, 256])
@pytest.mark.parametrize("T,N,D,out", [(1, 4096, 4096, "f32"), (16, 512, 2048, "bf16"), (64, 1024, 1024, "f32"),
                                       (128, 272, 512, "f32"), (129, 256, 1024, "bf16"), (300, 512, 2048, "f32"),
                                       (256, 1024, 4096, "f32")])
def test_gemm_random_codes(pq, g, T, N, D, out):
    """Few-token kernel (T <= 128, group ranges split across SMs at N = 4096) and the CTA-pair
    kernel (split-K at 256 x 1024 x 4096)."""
    ca, sa = inputs.random_codes(900 + T, T, D, g)
    cw, sw = inputs.random_codes(950 + N, N, D, g)
    Y = run_gemm(pq, ca, sa, cw, sw, g, out)
    r = oracle.gemm(ca, sa, cw, sw, g)
    if out == "f32":
        assert rel_fro(Y, r.y64) < 1e-5
    else:
        ref = oracle.bf16_round(r.y32)
        ulp = np.maximum(np.abs(ref), 2.0 ** -126) * 2.0 ** -7
        d = oracle.group_dots(ca, cw, g).astype(np.float64)
        S = np.einsum("gtn,tg,ng->tn", np.abs(d), sa.astype(np.float64), sw.astype(np.float64))
        clear = np.abs(r.y64) > 2.0 ** -7 * S
        assert np.all((np.abs(Y - ref) <= ulp)[clear])
        assert np.all(np.abs(Y - r.y64) <= 2.0 ** -8 * np.abs(Y) + (D // g + 2) * 2.0 ** -24 * S)


@pytest.mark.parametrize("kind,g", CASES)
@pytest.mark.parametrize("T", [16, 300])
def test_chain_matches_oracle_chain(pq, kind, g, T):
    """Transform, pack and GEMM on the GPU against the oracle's chain on the same inputs."""
    import torch
    D, N = 1024, 256
    wl = inputs.workload("sweep", T=T)
    X = np.ascontiguousarray(wl.X[:, :D])
    W = inputs.to_bf16_bits(inputs.normal(1000 + T, N * D, 0.02).reshape(N, D))
    plan, oplan = plans(pq, kind, D, g)
    G = D // g
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device="cuda")
    sa = torch.empty((T, G), dtype=torch.float32, device="cuda")
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device="cuda")
    sw = torch.empty((N, G), dtype=torch.float32, device="cuda")
    Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    pq.pq_transform_quant(plan, to_dev_bf16(X), ca, sa)
    pq.pq_pack_weights(plan, to_dev_bf16(W), cw, sw)
    pq.pq_w4a4_gemm(ca, sa, cw, sw, Y, g=g)
    pq.pq_check_status(plan)
    a = oracle.transform_quant(X, oplan)
    w = oracle.pack_weights(W, oplan)
    ref = oracle.gemm(a.codes, a.scales, w.codes, w.scales, g).y64
    # a few near-tie codes may differ by one; the GEMM on the GPU's own codes is exact to 1e-5
    got = Y.cpu().numpy()
    own = oracle.gemm(ca.cpu().numpy(), sa.cpu().numpy(), cw.cpu().numpy(), sw.cpu().numpy(), g).y64
    assert rel_fro(got, own) < 1e-5
    assert rel_fro(got, ref) < 1e-2


@pytest.mark.parametrize("first", ["g64", "g256", "rrs"])
def test_first_pair_gemm_of_a_process(first):
    """The CTA-pair GEMM's occupancy query must hold whichever instantiation a process launches
    first (g = 64 or 256, or the row-scale variant): run each alone in a fresh process."""
    import subprocess
    import sys
    code = f"""
import numpy as np, torch
from rotation_int4_w4a4_b200 import pq, inputs
g = {{'g64': 64, 'g256': 256, 'rrs': 128}}['{first}']
T, N, D = 200, 256, 512
ca, sa = inputs.random_codes(1, T, D, g)
cw, sw = inputs.random_codes(2, N, D, g)
Y = torch.empty((T, N), dtype=torch.float32, device='cuda')
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
if '{first}' == 'rrs':
    pq.pq_rrs_gemm(dev(ca), dev(sa[:, 0].copy()), dev(cw), dev(sw), Y)
else:
    pq.pq_w4a4_gemm(dev(ca), dev(sa), dev(cw), dev(sw), Y, g=g)
pq.pq_check_status()
print('ok')
"""
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=root, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stderr[-2000:]
