"""Shared test utilities: device tensors from the seeded generator, code comparisons."""
import numpy as np

import oracle


def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def empty_outputs(rows, D, g=128):
    import torch
    return (torch.empty((rows, D // 2), dtype=torch.uint8, device="cuda"),
            torch.empty((rows, D // g), dtype=torch.float32, device="cuda"))


def oracle_plan(kind, D, K=0, pairs=None, angles=None, beta=None, after=False):
    return oracle.Plan(kind, D, 128, K, pairs, angles, beta, smooth_after_rotate=after)


def assert_codes_match(gpu_packed, ref: "oracle.TQResult", rows=None):
    """Spec acceptance: bit-exact where the oracle's y/scale is more than 1e-3 from a
    half-integer, within 1 elsewhere."""
    g = oracle.unpack_nibbles(np.asarray(gpu_packed)).astype(np.int16)
    r = ref.q.codes.astype(np.int16)
    near = ref.q.near_tie
    if rows is not None:
        r, near = r[rows], near[rows]
    diff = np.abs(g - r)
    bad_far = (diff != 0) & ~near
    assert not bad_far.any(), (
        f"{bad_far.sum()} codes differ away from ties; first at {np.argwhere(bad_far)[:5].tolist()}")
    assert diff.max(initial=0) <= 1, f"code difference {diff.max()} > 1 near a tie"
    return int((diff != 0).sum()), int(near.sum())


def assert_scales_close(gpu, ref, rtol):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    zero = ref == 0
    assert np.all(gpu[zero] == 0), "zero groups must have scale 0"
    rel = np.abs(gpu[~zero] - ref[~zero]) / ref[~zero]
    assert rel.max(initial=0) <= rtol, f"scale rel err {rel.max()} > {rtol}"
    return float(rel.max(initial=0))
