"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np

# Tolerances on the normwise relative error of one output row,
#   err = max_n |y_n - r_n| / max_n |r_n|,
# against the fp64 oracle.  The contract: 2e-3 for fp32 activations, 1e-2
# for bf16 activations.  Paths that decode weights exactly in fp32 and
# accumulate in fp32 (the CUDA-core kernels) must also meet FP32_PATH_TOL:
# their only error is fp32 summation, a few units of 2^-24 times sqrt(K)
# relative to the row norm -- well below 1e-4 for every K used here.
TOL = {"f32": 2e-3, "bf16": 1e-2}
FP32_PATH_TOL = 1e-4
# The bandwidth kernel rounds activations to 16-bit fixed point per 32-wide
# sub-block (error <= 2^-14 of the sub-block's max |x| per element, random
# in sign): the row error is ~3e-5 of the row norm for N(0,1) activations;
# 3e-4 leaves a 10x margin and still catches any decode slip.
GEMV_TOL = 3e-4
# A bf16 output adds its own rounding, at most 2^-8 of the value.
BF16_OUT = 2.0 ** -8


def row_rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    """Max over rows of max_n |y - ref| / max_n |ref| (rows = leading axes)."""
    y = np.asarray(y, dtype=np.float64).reshape(-1, ref.shape[-1])
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, ref.shape[-1])
    num = np.abs(y - ref).max(axis=1)
    den = np.abs(ref).max(axis=1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max())


def to_device_x(x_f32: np.ndarray, dtype: str):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)   # values are already bf16-exact
    return t.cuda()


def to_device_w(w: np.ndarray):
    import torch

    return torch.from_numpy(np.ascontiguousarray(w)).cuda()
