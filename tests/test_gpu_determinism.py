"""Repeatability at full size: the same inputs must give bit-identical codes, scales and Y on
every run.  Each kernel computes every output element in a fixed order, so any difference
between runs is a race (for example a stage of shared memory refilled by the tensor-memory
accelerator while a thread is still reading it).  Every run starts from a flushed L2 and
compares against the first run on the device.  Workloads: the down_proj smoothing transform and
weight pack (X [8192, 14336], W [4096, 14336]), rotated runtime smoothing on the same shapes,
the q_proj Hadamard transform (tensor-core rotation) and the W4A4 GEMM of both shapes.
"""
import numpy as np
import pytest

from rotation_int4_w4a4_b200 import inputs

pytestmark = pytest.mark.gpu

REPEATS = 12


@pytest.fixture(scope="module")
def env():
    import torch
    from rotation_int4_w4a4_b200 import pq
    dev = torch.device("cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    return pq, dev, flush


def bf16(bits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def repeat_identical(flush, run, outputs):
    import torch
    flush.fill_(1)
    run()
    ref = [t.clone() for t in outputs]
    differing = 0
    for _ in range(REPEATS):
        flush.fill_(1)
        for t in outputs:
            t.zero_()
        run()
        differing += any(not torch.equal(a, b) for a, b in zip(ref, outputs))
    return differing


def test_smoothing_transform_and_pack(env):
    import torch
    pq, dev, flush = env
    wl = inputs.workload("down_proj")
    T, D, N, G = wl.T, wl.D, wl.N, wl.D // 128
    X, W = bf16(wl.X, dev), bf16(wl.W, dev)
    plan = pq.Plan("smooth_hadamard", D)
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device=dev)
    sa = torch.empty((T, G), dtype=torch.float32, device=dev)
    sm = torch.empty((T // 128, D), dtype=torch.float32, device=dev)
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device=dev)
    sw = torch.empty((N, G), dtype=torch.float32, device=dev)
    s_w = torch.ones(D, dtype=torch.float32, device=dev)

    def run():
        pq.pq_transform_quant(plan, X, ca, sa, sm)
        pq.pq_pack_weights(plan, W, cw, sw, s_w)

    assert repeat_identical(flush, run, (ca, sa, sm, cw, sw)) == 0
    pq.pq_check_status(plan)


def test_rotated_runtime_smoothing(env):
    import torch
    pq, dev, flush = env
    wl = inputs.workload("down_proj")
    T, D, N, G = wl.T, wl.D, wl.N, wl.D // 128
    X, W = bf16(wl.X, dev), bf16(wl.W, dev)
    plan = pq.Plan("hadamard", D)
    f32, i32, u8 = torch.float32, torch.int32, torch.uint8
    cm, gs = torch.empty(D, dtype=f32, device=dev), torch.empty(G, dtype=f32, device=dev)
    perm, inv = torch.empty(D, dtype=i32, device=dev), torch.empty(D, dtype=i32, device=dev)
    ca, ts = torch.empty((T, D // 2), dtype=u8, device=dev), torch.empty(T, dtype=f32, device=dev)
    cw, sw = torch.empty((N, D // 2), dtype=u8, device=dev), torch.empty((N, G), dtype=f32, device=dev)

    def run():
        pq.pq_rrs_prepare(plan, X, cm, perm, inv, gs)
        pq.pq_rrs_transform_quant(plan, X, perm, gs, ca, ts)
        pq.pq_rrs_pack_weights(plan, W, perm, gs, cw, sw)

    assert repeat_identical(flush, run, (cm, perm, inv, gs, ca, ts, cw, sw)) == 0
    pq.pq_check_status(plan)


@pytest.mark.parametrize("name", ["q_proj", "down_proj"])
def test_hadamard_transform_and_gemm(env, name):
    import torch
    pq, dev, flush = env
    wl = inputs.workload(name)
    T, D, N, G = wl.T, wl.D, wl.N, wl.D // 128
    X, W = bf16(wl.X, dev), bf16(wl.W, dev)
    plan = pq.Plan("hadamard", D)
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device=dev)
    sa = torch.empty((T, G), dtype=torch.float32, device=dev)
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device=dev)
    sw = torch.empty((N, G), dtype=torch.float32, device=dev)
    Y = torch.empty((T, N), dtype=torch.float32, device=dev)

    def run():
        pq.pq_transform_quant(plan, X, ca, sa)
        pq.pq_pack_weights(plan, W, cw, sw)
        pq.pq_w4a4_gemm(ca, sa, cw, sw, Y)

    assert repeat_identical(flush, run, (ca, sa, cw, sw, Y)) == 0
    pq.pq_check_status(plan)


def test_givens_transform_and_gemm(env):
    """up_proj: the Givens K = 16 rotation on the tensor cores (two bf16 terms), its weight pack
    and the 4096 x 14336 x 4096 GEMM."""
    import torch
    pq, dev, flush = env
    wl = inputs.workload("up_proj")
    T, D, N, G = wl.T, wl.D, wl.N, wl.D // 128
    X, W = bf16(wl.X, dev), bf16(wl.W, dev)
    pairs = pq.pq_select_pairs(wl.pair_seed, wl.D, wl.g, wl.K, wl.g // 2)
    plan = pq.Plan("givens", D, K=wl.K, pairs=pairs, angles=wl.angles, beta=wl.beta)
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device=dev)
    sa = torch.empty((T, G), dtype=torch.float32, device=dev)
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device=dev)
    sw = torch.empty((N, G), dtype=torch.float32, device=dev)
    Y = torch.empty((T, N), dtype=torch.float32, device=dev)

    def run():
        pq.pq_transform_quant(plan, X, ca, sa)
        pq.pq_pack_weights(plan, W, cw, sw)
        pq.pq_w4a4_gemm(ca, sa, cw, sw, Y)

    assert repeat_identical(flush, run, (ca, sa, cw, sw, Y)) == 0
    pq.pq_check_status(plan)


@pytest.mark.parametrize("T,N", [(1, 14336), (3, 4096), (16, 4096), (64, 14336)])
def test_decode_fused_call(env, T, N):
    """pq_w4a4_linear at decode sizes: the few-row transform, then the CUDA-core (T <= 4) or the
    few-token tensor-core GEMM (with its range reduction at N = 4096) as a programmatic
    dependent launch."""
    import torch
    pq, dev, flush = env
    wl = inputs.workload("sweep", T=T, N=N)
    D, G = wl.D, wl.D // 128
    X, W = bf16(wl.X, dev), bf16(wl.W, dev)
    plan = pq.Plan("hadamard", D)
    cw = torch.empty((N, D // 2), dtype=torch.uint8, device=dev)
    sw = torch.empty((N, G), dtype=torch.float32, device=dev)
    pq.pq_pack_weights(plan, W, cw, sw)
    ca = torch.empty((T, D // 2), dtype=torch.uint8, device=dev)
    sa = torch.empty((T, G), dtype=torch.float32, device=dev)
    Y = torch.empty((T, N), dtype=torch.float32, device=dev)

    def run():
        pq.pq_w4a4_linear(plan, X, ca, sa, cw, sw, Y)

    assert repeat_identical(flush, run, (ca, sa, Y)) == 0
    pq.pq_check_status(plan)
