"""Failure detection without a GPU fault: a device-side bounded wait that runs out.

pq_selftest_wait_timeout launches one thread waiting on a barrier that nothing completes, with
the bounded wait all of the library's pipelines use.  The wait must give up after its limit,
report through the status word (pq_check_status -> PQ_ERR_TIMEOUT, which also clears it), and
leave the context usable for the next real call.
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


def test_bounded_wait_times_out_and_context_survives(pq):
    import torch
    assert pq.pq_check_status() == pq.PQ_OK           # nothing pending
    pq.pq_selftest_wait_timeout(2_000_000)            # 2 ms
    with pytest.raises(pq.PQError) as err:
        pq.pq_check_status()
    assert err.value.status == pq.PQ_ERR_TIMEOUT
    assert pq.pq_check_status() == pq.PQ_OK           # the status word was cleared
    # the context still runs real work correctly
    T, N, D = 130, 256, 512
    ca, sa = inputs.random_codes(71, T, D)
    cw, sw = inputs.random_codes(72, N, D)
    Y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    pq.pq_w4a4_gemm(to_dev(ca), to_dev(sa), to_dev(cw), to_dev(sw), Y)
    assert pq.pq_check_status() == pq.PQ_OK
    ref = oracle.gemm(ca, sa, cw, sw).y64
    assert np.linalg.norm(Y.cpu().numpy() - ref) / np.linalg.norm(ref) < 1e-5
