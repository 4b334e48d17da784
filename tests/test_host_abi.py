"""Host-side checks of libpq that need no GPU: exports, argument validation, pair selection."""
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import build
    build.build()
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def header_functions():
    src = open(os.path.join(ROOT, "include", "pq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pq_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol(pq):
    declared = header_functions()
    assert declared, "no declarations parsed"
    for name in declared:
        assert hasattr(pq.lib, name), f"{name} not exported"
    assert sorted(pq.EXPORTS) == declared


@pytest.mark.parametrize("seed,K,N", [(0, 8, 64), (0x5EED0707, 16, 64), (42, 4, 17), (7, 64, 64)])
def test_select_pairs_matches_oracle(pq, seed, K, N):
    a = pq.pq_select_pairs(seed, 384, 128, K, N)
    b = oracle.select_pairs(seed, 384, 128, K, N)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("seed,K,N", [(3, 4, 32), (11, 8, 20)])
def test_select_pairs_g64_matches_oracle(pq, seed, K, N):
    a = pq.pq_select_pairs(seed, 384, 64, K, N)
    b = oracle.select_pairs(seed, 384, 64, K, N)
    assert np.array_equal(a, b)


def test_status_strings(pq):
    assert pq.lib.pq_status_string(0) == b"PQ_OK"
    assert pq.lib.pq_status_string(5) == b"PQ_ERR_TIMEOUT"
    assert pq.lib.pq_status_string(99) == b"PQ_ERR_UNKNOWN"


def test_select_pairs_rejects_bad_arguments(pq):
    out = np.empty(4096, dtype=np.uint8)
    assert pq.lib.pq_select_pairs(0, 256, 32, 4, 16, out.ctypes.data) == pq.PQ_ERR_UNSUPPORTED
    assert pq.lib.pq_select_pairs(0, 512, 256, 4, 16, out.ctypes.data) == pq.PQ_ERR_UNSUPPORTED
    assert pq.lib.pq_select_pairs(0, 200, 128, 4, 16, out.ctypes.data) == pq.PQ_ERR_INVALID_ARG
    assert pq.lib.pq_select_pairs(0, 256, 128, 0, 16, out.ctypes.data) == pq.PQ_ERR_INVALID_ARG
    assert pq.lib.pq_select_pairs(0, 256, 128, 4, 65, out.ctypes.data) == pq.PQ_ERR_INVALID_ARG
    assert pq.lib.pq_select_pairs(0, 256, 128, 4, 16, None) == pq.PQ_ERR_INVALID_ARG
    assert b"K=0" in pq.lib.pq_last_error() or True


def test_make_plan_validation_before_any_device_call(pq):
    with pytest.raises(pq.PQError) as e:
        pq.Plan("hadamard", 100)
    assert e.value.status == pq.PQ_ERR_INVALID_ARG
    # group sizes: 64/128/256 for Hadamard, 64/128 for Givens, 128 for smoothing
    for kind, D, g in (("hadamard", 256, 32), ("givens", 512, 256), ("smooth_hadamard", 256, 64),
                       ("smooth_hadamard", 512, 256)):
        with pytest.raises(pq.PQError) as e:
            pq.Plan(kind, D, g=g, K=2)
        assert e.value.status == pq.PQ_ERR_UNSUPPORTED, (kind, g)
    with pytest.raises(pq.PQError) as e:
        pq.Plan("hadamard", 384, g=256)                   # D not a multiple of g
    assert e.value.status == pq.PQ_ERR_INVALID_ARG
    # 8-bit outlier groups: rotation plans at g = 128, distinct groups below D/g
    for kind, g, groups, status in (("smooth_hadamard", 128, [0], pq.PQ_ERR_UNSUPPORTED),
                                    ("hadamard", 64, [0], pq.PQ_ERR_UNSUPPORTED),
                                    ("hadamard", 128, [1, 1], pq.PQ_ERR_INVALID_ARG),
                                    ("hadamard", 128, [2], pq.PQ_ERR_INVALID_ARG),
                                    ("hadamard", 128, [-1], pq.PQ_ERR_INVALID_ARG)):
        with pytest.raises(pq.PQError) as e:
            pq.Plan(kind, 256, g=g, groups8=groups)
        assert e.value.status == status, (kind, g, groups)
    with pytest.raises(pq.PQError) as e:
        pq.Plan("hadamard", 256, flags=pq.PQ_FLAG_SMOOTH_AFTER_ROTATE)
    assert e.value.status == pq.PQ_ERR_INVALID_ARG
    with pytest.raises(pq.PQError):
        pq.Plan("givens", 256, K=2)                      # no pairs / angles
    pairs = np.full((2, 1, 64, 2), 0xFF, dtype=np.uint8)
    pairs[0, 0, 0] = (3, 9)
    pairs[0, 0, 1] = (9, 20)                             # channel 9 twice in one layer
    with pytest.raises(pq.PQError) as e:
        pq.Plan("givens", 256, K=1, pairs=pairs, angles=np.zeros((2, 1, 64), np.float32))
    assert "disjoint" in str(e.value)
    pairs[0, 0, 1] = (30, 20)                            # i > j
    with pytest.raises(pq.PQError):
        pq.Plan("givens", 256, K=1, pairs=pairs, angles=np.zeros((2, 1, 64), np.float32))
    pairs[0, 0, 1] = (20, 130)                           # outside the group
    with pytest.raises(pq.PQError):
        pq.Plan("givens", 256, K=1, pairs=pairs, angles=np.zeros((2, 1, 64), np.float32))


def test_gemm_and_transform_validation(pq):
    L = pq.lib
    p = 16  # any aligned non-null fake address: validation fails before use
    assert L.pq_w4a4_gemm(None, p, p, p, 4, 16, 128, 128, p, 0, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm(p, p, p, p, 4, 16, 128, 32, p, 0, None) == pq.PQ_ERR_UNSUPPORTED
    assert L.pq_w4a4_gemm(p, p, p, p, 4, 16, 384, 256, p, 0, None) == pq.PQ_ERR_INVALID_ARG   # D % g
    assert L.pq_rrs_gemm(p, p, p, p, 4, 16, 128, 32, p, 0, None) == pq.PQ_ERR_UNSUPPORTED
    assert L.pq_w4a4_gemm(p, p, p, p, 4, 24, 128, 128, p, 0, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm(p, p, p, p, 4, 16, 200, 128, p, 0, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm(p, p, p, p, 0, 16, 128, 128, p, 0, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm(p + 4, p, p, p, 4, 16, 128, 128, p, 0, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm(p, p, p, p, 4, 16, 128, 128, p, 7, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_transform_quant(None, p, 4, 128, p, p, None, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_linear(None, p, 4, 128, p, p, p, p, 16, p, 0, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm_launch_count_g(4, 16, 384, 256, None) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_pack_weights(None, p, 4, None, p, p, None) == pq.PQ_ERR_INVALID_ARG
    L.pq_destroy_plan(None)                              # no-op


def test_selftest_wait_timeout_validation(pq):
    """The limit is checked before anything is launched (runs without a GPU)."""
    for bad in (0, 999, 100_000_001):
        assert pq.lib.pq_selftest_wait_timeout(bad, None) == pq.PQ_ERR_INVALID_ARG
        assert b"limit_ns" in pq.lib.pq_last_error()



def test_gemm_launch_count_query(pq):
    """Host-only query (no GPU here, so 148 SMs are assumed): sizes are validated as for the
    GEMM.  More than 128 tokens: 2 or 3 launches (operand expansion, contraction, split-K
    reduction).  5 to 128 tokens: 1, or 2 with the group-range reduction.  At most 4 tokens:
    the CUDA-core kernel, 1."""
    import ctypes
    L = pq.lib
    n = ctypes.c_int(-1)
    assert L.pq_w4a4_gemm_launch_count(4, 24, 128, ctypes.byref(n)) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm_launch_count(4, 16, 200, ctypes.byref(n)) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm_launch_count(0, 16, 128, ctypes.byref(n)) == pq.PQ_ERR_INVALID_ARG
    assert L.pq_w4a4_gemm_launch_count(4, 16, 128, None) == pq.PQ_ERR_INVALID_ARG
    assert n.value == -1
    assert pq.pq_w4a4_gemm_launch_count(4096, 14336, 4096) == 2   # 896 pair tiles
    assert pq.pq_w4a4_gemm_launch_count(256, 4096, 4096) == 3     # 16 pair tiles, 32 groups
    assert pq.pq_w4a4_gemm_launch_count(129, 4096, 4096) == 3     # 129 tokens: CTA-pair kernel
    # at most 4 tokens: one CUDA-core launch whatever the shape
    for T in (1, 2, 3, 4):
        assert pq.pq_w4a4_gemm_launch_count(T, 4096, 4096) == 1
        assert pq.pq_w4a4_gemm_launch_count(T, 14336, 4096) == 1
        assert pq.pq_w4a4_gemm_launch_count(T, 16, 128) == 1
    # 5 to 128 tokens: 32 weight tiles of 128 rows -> group ranges in one wave over 148 SMs
    assert pq.pq_w4a4_gemm_launch_count(5, 4096, 4096) == 2
    assert pq.pq_w4a4_gemm_launch_count(17, 4096, 4096) == 2
    assert pq.pq_w4a4_gemm_launch_count(17, 4096, 512) == 1       # 4 groups: one range (one stage)
    assert pq.pq_w4a4_gemm_launch_count(17, 14336, 4096) == 1     # 112 tiles: one wave unsplit
    # 64 tokens: four ranges (the partial tiles stay below the weight bytes); 128 tokens at
    # N = 14336: 112 weight tiles fill one wave, one launch writes Y
    assert pq.pq_w4a4_gemm_launch_count(64, 4096, 4096) == 2
    assert pq.pq_w4a4_gemm_launch_count(128, 14336, 4096) == 1
    assert pq.pq_w4a4_gemm_launch_count(128, 4096, 4096) == 2
    # other group sizes: the same kernels, split by groups of g (ranges of 4 groups)
    for g in (64, 128, 256):
        assert pq.pq_w4a4_gemm_launch_count_g(4096, 14336, 4096, g) == 2
        assert pq.pq_w4a4_gemm_launch_count_g(17, 14336, 4096, g) == 1
        assert pq.pq_w4a4_gemm_launch_count_g(1, 4096, 4096, g) == 1
    assert pq.pq_w4a4_gemm_launch_count_g(17, 4096, 4096, 128) == pq.pq_w4a4_gemm_launch_count(17, 4096, 4096)
    assert pq.pq_w4a4_gemm_launch_count_g(17, 4096, 4096, 64) == 2    # 64 groups of 64: ranges
    assert pq.pq_w4a4_gemm_launch_count_g(17, 4096, 512, 64) == 1     # partial tiles would pass the weights
    assert pq.pq_w4a4_gemm_launch_count_g(17, 4096, 512, 256) == 1    # 2 groups: one range


def test_binding_rejects_host_and_strided_tensors(pq):
    """The binding checks device and layout before any call reaches the library."""
    import torch
    with pytest.raises(ValueError, match="CUDA"):
        pq._ptr(torch.zeros(4, 4))

    class FakeCuda:                       # stands in for a CUDA tensor on this GPU-less box
        is_cuda = True

        def __init__(self, contiguous, inner):
            self._c, self._s = contiguous, inner

        def is_contiguous(self):
            return self._c

        def stride(self, dim):
            return self._s

        def data_ptr(self):
            return 4096

    assert pq._ptr(FakeCuda(True, 1)) == 4096
    with pytest.raises(ValueError, match="contiguous"):
        pq._ptr(FakeCuda(False, 1))
    assert pq._ptr(FakeCuda(False, 1), rows_strided=True) == 4096   # padded rows (ldx > D)
    with pytest.raises(ValueError, match="last dimension"):
        pq._ptr(FakeCuda(False, 2), rows_strided=True)
    assert pq._ptr(None) is None and pq._ptr(16) == 16
