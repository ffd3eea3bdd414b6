"""The Python binding's argument checks run on the host before any library
call: CPU tensors, wrong dtypes, shapes and layouts are rejected with a
ValueError naming the argument (no GPU needed)."""
import pytest
import torch

from fine_grained_fp8_sigmoid_b200 import binding as B


def test_cpu_tensors_are_rejected():
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    q = torch.zeros(4, 128, dtype=torch.uint8)
    s = torch.zeros(4, 1, dtype=torch.float32)
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        B.moe_quant_1x128(x, q, s)


def test_want_checks_dtype_shape_and_layout():
    # the checks themselves, on a tensor that merely reports being on CUDA
    class Fake:
        def __init__(self, t):
            self.t = t
            self.is_cuda = True
            self.dtype = t.dtype
            self.shape = t.shape

        def is_contiguous(self):
            return self.t.is_contiguous()

    good = torch.zeros(4, 8, dtype=torch.float32)
    assert B._want(Fake(good), torch.float32, (4, 8), "a") is not None
    with pytest.raises(ValueError, match="a: dtype"):
        B._want(Fake(good), torch.bfloat16, (4, 8), "a")
    with pytest.raises(ValueError, match="a: shape"):
        B._want(Fake(good), torch.float32, (8, 4), "a")
    with pytest.raises(ValueError, match="a must be contiguous"):
        B._want(Fake(good.t()), torch.float32, (8, 4), "a")
    with pytest.raises(ValueError, match="a is required"):
        B._want(None, torch.float32, (4, 8), "a")
    assert B._opt(None, torch.float32, (4, 8), "a") is None
