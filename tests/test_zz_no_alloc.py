"""pq_w4a4_gemm_noalloc: the W4A4 GEMM with the library's fixed device-array scratch.

Collected last on purpose, so that it also runs after every other test has used the allocating
entry point on the same device.  Two calls in a row on one stream (a larger call, then a smaller
one with ragged T and N) must each match pq_w4a4_gemm on the same inputs within the GEMM's
float32 tolerance; sizes beyond the fixed scratch are rejected before anything reaches the
device.
"""
import ctypes

import numpy as np
import pytest

from rotation_int4_w4a4_b200 import inputs
from tests.helpers import to_dev

F32_REL_FRO = 1e-5   # the float32 bound of the GEMM parity tests


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


def rel_fro(a, b):
    a, b = a.astype(np.float64), b.astype(np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def test_rejects_sizes_beyond_the_fixed_scratch(pq):
    """(T + N) * D above the limit fails with INVALID_ARG before any device call (runs on CPU)."""
    assert pq.lib.pq_w4a4_gemm_noalloc.argtypes == pq.lib.pq_w4a4_gemm.argtypes
    fake = 1 << 20   # 16-byte aligned, never dereferenced: the call must fail before launching
    limit = 32 * 1024 * 1024
    D = 4096
    T = limit // D - 16 + 1          # T + N = limit / D + 1 rows
    st = pq.lib.pq_w4a4_gemm_noalloc(fake, fake, fake, fake, T, 16, D, 128, fake, 0, None)
    assert st == pq.PQ_ERR_INVALID_ARG
    assert b"scratch" in pq.lib.pq_last_error()


@pytest.mark.gpu
def test_two_calls_match_the_allocating_entry(pq):
    import torch
    # The larger call runs first and leaves its operand bytes in the shared scratch; the second,
    # smaller call has T and N that are not multiples of the 256-wide tile, so its last tiles
    # reach past its own operands into bytes the first call wrote.  The tensor maps' bounds must
    # keep those bytes out of its result.
    cases = [(600, 1024, 1024, torch.float32, 11), (130, 272, 384, torch.bfloat16, 12)]
    assert (cases[0][0] + cases[0][1]) * cases[0][2] > (cases[1][0] + cases[1][1]) * cases[1][2]
    data = []
    for T, N, D, dt, seed in cases:
        ca, sa = inputs.random_codes(seed, T, D)
        cw, sw = inputs.random_codes(seed + 100, N, D)
        dev = [to_dev(a) for a in (ca, sa, cw, sw)]
        data.append((dev, torch.empty((T, N), dtype=dt, device="cuda"),
                     torch.empty((T, N), dtype=dt, device="cuda")))
    for dev, y_ref, _ in data:
        pq.pq_w4a4_gemm(*dev, y_ref)
    pq.pq_check_status()
    # the two calls back to back on the current stream, then one synchronisation
    for dev, _, y in data:
        pq.pq_w4a4_gemm_noalloc(*dev, y)
    pq.pq_check_status()
    for (dev, y_ref, y), (T, N, D, dt, _) in zip(data, cases):
        ref = y_ref.float().cpu().numpy()
        got = y.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert rel_fro(got, ref) < F32_REL_FRO, (T, N, D, dt)
