"""kq_matmul_id_noalloc: the expert-indexed product for callers that cannot
allocate device memory (they receive only their input and output buffers,
e.g. a plugin inside another framework's execution plan, or a host language
without a CUDA allocator), so they cannot hand kq_matmul_id its workspace.

The call is made through the C ABI and its result is compared with the
ordinary kq_matmul_id (caller-owned workspace) on two calls in a row with
different inputs, so stale contents of the library's built-in scratch array
from the first call cannot pass for the second.  Both entry points run the
same kernels on the same grouping, so the outputs must be identical bit for
bit.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest

import synth
from kqtest import to_device_w, to_device_x

pytestmark = pytest.mark.gpu

KQ_ERR_WORKSPACE = -7


def _noalloc(kq, codec, w, x, ids, y):
    import torch

    fn = kq.lib().kq_matmul_id_noalloc
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    fn.argtypes = [ctypes.c_int, vp, i64, i64, i64, i64, vp, ctypes.c_int, i64, vp, i64, vp,
                   ctypes.c_int, vp]
    fn.restype = ctypes.c_int
    e, n, _ = w.shape
    t, k = x.shape
    xdt = kq.BF16 if x.dtype == torch.bfloat16 else kq.F32
    ydt = kq.F32 if y.dtype == torch.float32 else kq.BF16
    return fn(codec, vp(w.data_ptr()), e, n, k, w.stride(0), vp(x.data_ptr()), xdt, t,
              vp(ids.data_ptr()), ids.shape[1], vp(y.data_ptr()), ydt,
              vp(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_on_two_calls(kq):
    import torch

    wl = synth.WORKLOADS["moe_q4_k_e64_1408x2048_t32_top6"]
    for seed in (0, 1):
        w, x, ids = synth.make_inputs(wl, seed=seed)
        wd = to_device_w(w)
        xd = to_device_x(x, wl.x_dtype)
        idd = torch.from_numpy(ids).cuda()
        ref = kq.matmul_id(wd, wl.codec, xd, idd).cpu().numpy()
        y = torch.full((wl.m, wl.top_k, wl.n), float("nan"), device="cuda")
        assert _noalloc(kq, wl.codec, wd, xd, idd, y) == 0
        got = y.cpu().numpy()
        assert np.isfinite(got).all()
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
        assert kq.device_status() == 0


def test_noalloc_rejects_requests_beyond_its_scratch(kq):
    import torch

    # 40000 tokens x 8 slots needs far more grouping scratch than the 256 KiB built in.
    e, n, k, t, top_k = 16, 8, 256, 40000, 8
    assert kq.matmul_id_workspace_bytes(t, top_k, e) > 256 * 1024
    w = torch.zeros((e, n, kq.row_bytes(synth.Q4_K, k)), dtype=torch.uint8, device="cuda")
    x = torch.zeros((t, k), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((t, top_k), dtype=torch.int32, device="cuda")
    y = torch.zeros((t, top_k, n), device="cuda")
    assert _noalloc(kq, synth.Q4_K, w, x, ids, y) == KQ_ERR_WORKSPACE
