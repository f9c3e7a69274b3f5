"""The binding checks buffer shapes, dtypes, layout and device before it
hands plain pointers to the C ABI (which cannot see sizes): a wrong-shaped
output would otherwise be written past its end.  CPU tensors stand in for
device tensors; no call reaches the library."""
import pytest
import torch

import block_quantized_matmul_quant_b200 as kq


def test_check_tensor_accepts_the_exact_buffer():
    cpu = torch.device("cpu")
    kq._check_tensor("out", torch.empty((3, 5)), (3, 5), kq._ACT, cpu)
    kq._check_tensor("out", torch.empty((3, 5), dtype=torch.bfloat16), (3, 5), kq._ACT, cpu)


@pytest.mark.parametrize("t,msg", [
    (torch.empty((3, 4)), "shape"),                       # too small: would be written past its end
    (torch.empty((5, 3)), "shape"),                       # transposed
    (torch.empty((3, 5), dtype=torch.float64), "dtype"),
    (torch.empty((5, 3)).t(), "contiguous"),              # right shape, strided
])
def test_check_tensor_rejects(t, msg):
    with pytest.raises(ValueError, match=msg):
        kq._check_tensor("out", t, (3, 5), kq._ACT, torch.device("cpu"))


def test_check_tensor_rejects_another_device():
    with pytest.raises(ValueError, match="on"):
        kq._check_tensor("x", torch.empty((2, 2), device="meta"), (2, 2), kq._ACT, torch.device("cpu"))


def test_host_tensors_are_refused_before_the_library():
    w = torch.zeros((4, 144), dtype=torch.uint8)
    x = torch.zeros((1, 256))
    with pytest.raises(ValueError, match="CUDA"):
        kq.matmul(w, kq.Q4_K, x)
    with pytest.raises(ValueError, match="CUDA"):
        kq.dequantize(w, kq.Q4_K, 256)
    with pytest.raises(ValueError, match="CUDA"):
        kq.matmul_id(w.view(1, 4, 144), kq.Q4_K, x, torch.zeros((1, 1), dtype=torch.int32))
    with pytest.raises(ValueError):
        kq.moe_group(torch.zeros(4, dtype=torch.int64), 2)     # ids must be int32
