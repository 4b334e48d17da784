"""The ctypes binding's own checks, on CPU: a tensor of the wrong dtype or with too few elements
is rejected with ValueError before anything reaches the C ABI (which sees only pointers, so a
float16 Y or a short scales buffer would otherwise be written or read past its end)."""
import pytest
import torch


@pytest.fixture(scope="module")
def pq():
    from rotation_int4_w4a4_b200 import build
    build.build()
    from rotation_int4_w4a4_b200 import pq as _pq
    return _pq


class FakeCuda:
    """Stands in for a contiguous CUDA tensor of a given dtype and shape (never dereferenced:
    every case below must fail in the binding, before the library is called)."""

    def __init__(self, shape, dtype):
        self._t = torch.empty(shape, dtype=dtype)
        self.shape, self.dtype, self.is_cuda = self._t.shape, dtype, True

    def dim(self):
        return self._t.dim()

    def stride(self, i=None):
        return self._t.stride() if i is None else self._t.stride(i)

    def is_contiguous(self):
        return True

    def numel(self):
        return self._t.numel()

    def data_ptr(self):
        return 1 << 20


def gemm_args(T=4, N=32, D=256, y_dtype=torch.float32, short=None):
    sizes = {"ca": ((T, D // 2), torch.uint8), "sa": ((T, D // 128), torch.float32),
             "cw": ((N, D // 2), torch.uint8), "sw": ((N, D // 128), torch.float32),
             "y": ((T, N), y_dtype)}
    out = {}
    for k, (shape, dt) in sizes.items():
        if k == short:
            shape = (shape[0] - 1,) + shape[1:]
        out[k] = FakeCuda(shape, dt)
    return out


@pytest.mark.parametrize("fn", ["pq_w4a4_gemm", "pq_w4a4_gemm_noalloc"])
def test_gemm_rejects_y_dtype(pq, fn):
    a = gemm_args(y_dtype=torch.float16)
    with pytest.raises(ValueError, match="Y: dtype"):
        getattr(pq, fn)(a["ca"], a["sa"], a["cw"], a["sw"], a["y"], T=4, N=32, D=256)


@pytest.mark.parametrize("short", ["ca", "sa", "cw", "sw", "y"])
def test_gemm_rejects_short_buffers(pq, short):
    a = gemm_args(short=short)
    with pytest.raises(ValueError, match="holds"):
        pq.pq_w4a4_gemm(a["ca"], a["sa"], a["cw"], a["sw"], a["y"], T=4, N=32, D=256)


def test_gemm_rejects_scale_dtype(pq):
    a = gemm_args()
    a["sa"] = FakeCuda((4, 2), torch.bfloat16)
    with pytest.raises(ValueError, match="scales_A: dtype"):
        pq.pq_w4a4_gemm(a["ca"], a["sa"], a["cw"], a["sw"], a["y"], T=4, N=32, D=256)
    b = gemm_args()
    b["cw"] = FakeCuda((32, 128), torch.int8)
    with pytest.raises(ValueError, match="codes_W: dtype"):
        pq.pq_w4a4_gemm(b["ca"], b["sa"], b["cw"], b["sw"], b["y"], T=4, N=32, D=256)


def test_gemm_out_dtype_must_match_y(pq):
    a = gemm_args(y_dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="does not match"):
        pq.pq_w4a4_gemm(a["ca"], a["sa"], a["cw"], a["sw"], a["y"], T=4, N=32, D=256,
                        out_dtype=pq.PQ_OUT_F32)


class FakePlan:
    D, g, Gx, Dx = 256, 128, 2, 256
    handle = None


def test_transform_rejects_dtype_and_sizes(pq):
    T, D = 5, 256
    X = FakeCuda((T, D), torch.bfloat16)
    codes, scales = FakeCuda((T, D // 2), torch.uint8), FakeCuda((T, 2), torch.float32)
    with pytest.raises(ValueError, match="X: dtype"):
        pq.pq_transform_quant(FakePlan(), FakeCuda((T, D), torch.float16), codes, scales)
    with pytest.raises(ValueError, match="codes: holds"):
        pq.pq_transform_quant(FakePlan(), X, FakeCuda((T - 1, D // 2), torch.uint8), scales)
    with pytest.raises(ValueError, match="scales: holds"):
        pq.pq_transform_quant(FakePlan(), X, codes, FakeCuda((T, 1), torch.float32))
    with pytest.raises(ValueError, match="smooth_out: holds"):
        pq.pq_transform_quant(FakePlan(), X, codes, scales, smooth_out=FakeCuda((1, D - 1), torch.float32))
    with pytest.raises(ValueError, match="X: holds"):
        pq.pq_transform_quant(FakePlan(), X, codes, scales, T=T + 1, ldx=D)


def test_pack_rejects_dtype_and_sizes(pq):
    N, D = 16, 256
    W = FakeCuda((N, D), torch.bfloat16)
    codes, scales = FakeCuda((N, D // 2), torch.uint8), FakeCuda((N, 2), torch.float32)
    with pytest.raises(ValueError, match="W: dtype"):
        pq.pq_pack_weights(FakePlan(), FakeCuda((N, D), torch.float32), codes, scales)
    with pytest.raises(ValueError, match="smooth_w: holds"):
        pq.pq_pack_weights(FakePlan(), W, codes, scales, smooth_w=FakeCuda((D - 1,), torch.float32))
    with pytest.raises(ValueError, match="scales_W: dtype"):
        pq.pq_pack_weights(FakePlan(), W, codes, FakeCuda((N, 2), torch.float64))


def test_host_tensors_are_rejected(pq):
    ca = torch.zeros((4, 128), dtype=torch.uint8)
    a = gemm_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        pq.pq_w4a4_gemm(ca, a["sa"], a["cw"], a["sw"], a["y"], T=4, N=32, D=256)
