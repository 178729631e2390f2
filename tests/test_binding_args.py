"""The Python binding rejects malformed arguments before anything reaches the library.

The C entry points take bare pointers and sizes, so a tensor of the wrong dtype or shape would be
read or written past its end by the kernels.  These checks run on the CPU: the library loader is
replaced by one that fails the test if it is reached, so every case must raise first.
"""
import pytest
import torch

import two_sided_gptq_02_b200._lib as lib


@pytest.fixture
def no_library(monkeypatch):
    def _fail():
        raise AssertionError("the library was reached with malformed arguments")
    monkeypatch.setattr(lib, "load_library", _fail)


def _noalloc_args(m=6, n=5, dtype=torch.float64):
    return dict(W=torch.zeros(m, n, dtype=dtype), U_A=torch.eye(n, dtype=dtype), U_B=torch.eye(m, dtype=dtype),
                qmin=-4, qmax=3, row_scale=torch.ones(m, dtype=dtype), codes=torch.zeros(m, n, dtype=torch.int8),
                V=torch.zeros(m, n, dtype=dtype), E=torch.zeros(m, n, dtype=dtype),
                dev_status=torch.zeros(1, dtype=torch.int32))


@pytest.mark.parametrize("field,value,exc", [
    ("V", torch.zeros(6, 5, dtype=torch.float32), TypeError),        # V narrower than W
    ("V", torch.zeros(6, 4, dtype=torch.float64), ValueError),
    ("E", torch.zeros(6, 5, dtype=torch.float32), TypeError),
    ("E", torch.zeros(5, 6, dtype=torch.float64), ValueError),
    ("codes", torch.zeros(6, 5, dtype=torch.int32), TypeError),
    ("codes", torch.zeros(6, 6, dtype=torch.int8), ValueError),
    ("U_A", torch.eye(6, dtype=torch.float64), ValueError),
    ("U_A", torch.eye(5, dtype=torch.float32), TypeError),
    ("U_B", torch.eye(5, dtype=torch.float64), ValueError),
    ("U_B", torch.eye(6, dtype=torch.float32), TypeError),
    ("row_scale", torch.ones(5, dtype=torch.float64), ValueError),
    ("row_scale", torch.ones(6, dtype=torch.float32), TypeError),
    ("dev_status", torch.zeros(1, dtype=torch.int64), TypeError),
    ("dev_status", torch.zeros(0, dtype=torch.int32), TypeError),
    ("W", torch.zeros(6, 5, 1, dtype=torch.float64), ValueError),
])
def test_noalloc_rejects_bad_argument(no_library, field, value, exc):
    args = _noalloc_args()
    args[field] = value
    with pytest.raises(exc):
        lib.kron_gptq_quantize_noalloc(**args)


def test_noalloc_rejects_host_tensors(no_library):
    with pytest.raises(ValueError, match="CUDA device"):
        lib.kron_gptq_quantize_noalloc(**_noalloc_args())


def test_noalloc_rejects_f64_W_with_f32_factors(no_library):
    args = _noalloc_args()
    for k in ("U_A", "U_B", "row_scale", "V", "E"):
        args[k] = args[k].float()
    with pytest.raises(TypeError):
        lib.kron_gptq_quantize_noalloc(**args)


def test_loss_rejects_bad_shapes(no_library):
    W = torch.zeros(6, 5, dtype=torch.float64)
    with pytest.raises(ValueError):
        lib.kron_gptq_loss(W, torch.zeros(5, 6, dtype=torch.float64), torch.eye(5, dtype=torch.float64),
                           torch.eye(6, dtype=torch.float64), 0.01)
    with pytest.raises(ValueError):
        lib.kron_gptq_loss(W, W, torch.eye(6, dtype=torch.float64), torch.eye(6, dtype=torch.float64), 0.01)
    with pytest.raises(TypeError):
        lib.kron_gptq_loss(W, W.float(), torch.eye(5, dtype=torch.float64), torch.eye(6, dtype=torch.float64), 0.01)


def test_antidiagonal_and_prepare_reject_bad_shapes(no_library):
    W = torch.zeros(6, 5, dtype=torch.float64)
    with pytest.raises(ValueError):
        lib.kron_gptq_quantize_antidiagonal(W, torch.eye(5, dtype=torch.float64), torch.eye(5, dtype=torch.float64),
                                            -4, 3, torch.ones(6, dtype=torch.float64))
    with pytest.raises(TypeError):
        lib.kron_gptq_quantize_antidiagonal(W.float(), torch.eye(5), torch.eye(6), -4, 3, torch.ones(6))
    with pytest.raises(ValueError):
        lib.kron_gptq_prepare(torch.zeros(4, 5, dtype=torch.float64), None, 0.01)
    with pytest.raises(TypeError):
        lib.kron_gptq_prepare(torch.eye(4, dtype=torch.float64), torch.eye(4, dtype=torch.float32), 0.01)


def test_factors_and_scales_reject_bad_arguments(no_library):
    a = torch.zeros(10, 4, dtype=torch.float64)
    with pytest.raises(ValueError):
        lib.kron_gptq_factors(a, torch.zeros(9, 3, dtype=torch.float64))
    with pytest.raises(ValueError):
        lib.kron_gptq_factors(a, torch.zeros(10, 3, dtype=torch.float64), method="nope")
    with pytest.raises(ValueError):
        lib.kron_gptq_waterkron_scales(torch.zeros(4, 3, dtype=torch.float64), torch.eye(3, dtype=torch.float64), 0.1)
