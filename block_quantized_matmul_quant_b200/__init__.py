"""Python binding of libkq (block-quantized matrix products on B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libkq.so`` (built in-tree from ``csrc/`` by ``_build.py``).  torch
supplies device memory and the current stream; each buffer's shape, dtype,
layout and device are checked here, since the C ABI receives bare pointers.
There is no CPU fallback: when the library is missing or the device is not
an sm_100 GPU the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import _build

Q8_0, Q2_K, Q4_K, Q5_K, Q6_K, TQ1_G128 = 8, 10, 12, 13, 14, 1001
CODECS = {"q8_0": Q8_0, "q2_k": Q2_K, "q4_k": Q4_K, "q5_k": Q5_K, "q6_k": Q6_K, "tq1_g128": TQ1_G128}
F32, BF16, F16 = 0, 1, 2
PATH_AUTO, PATH_SIMPLE, PATH_GEMV, PATH_GEMM, PATH_GEMV_TC = 0, 1, 2, 3, 4
FLAG_CONST_WEIGHTS = 0x100
FLAG_INDEPENDENT = 0x200

_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}

# KQ_DEBUG_LIBRARY=1 in the environment loads the KQ_DEBUG build instead
# (device bounds checks, short bounded waits; include/kq_debug.h).
DEBUG_LIBRARY = os.environ.get("KQ_DEBUG_LIBRARY", "") == "1"
LIB_PATH = _build.LIB_DEBUG if DEBUG_LIBRARY else _build.LIB


class KQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def ensure_built() -> str:
    """Build libkq.so if it is missing or older than its sources."""
    return _build.build()


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                "or python -m block_quantized_matmul_quant_b200._build")
        L = ctypes.CDLL(LIB_PATH)
        i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        sz = ctypes.c_size_t
        L.kq_block_weights.argtypes = [i32]
        L.kq_block_bytes.argtypes = [i32]
        L.kq_row_bytes.argtypes = [i32, i64]
        L.kq_row_bytes.restype = i64
        L.kq_dequantize.argtypes = [i32, vp, i64, i64, vp, i32, vp]
        L.kq_matmul.argtypes = [i32, vp, i64, i64, vp, i32, i64, vp, i32, vp]
        L.kq_matmul_ex.argtypes = [i32, vp, i64, i64, vp, i32, i64, vp, i32, i32, vp]
        L.kq_matmul_id_workspace_bytes.argtypes = [i64, i64, i64]
        L.kq_matmul_id_workspace_bytes.restype = sz
        L.kq_matmul_id.argtypes = [i32, vp, i64, i64, i64, i64, vp, i32, i64, vp, i64, vp, i32,
                                   vp, sz, vp]
        L.kq_matmul_id_ex.argtypes = [i32, vp, i64, i64, i64, i64, vp, i32, i64, vp, i64, vp, i32,
                                      vp, sz, i32, vp]
        L.kq_moe_group.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.kq_validate.argtypes = [i32, vp, i64, i64, ctypes.POINTER(i64), vp]
        L.kq_get_rows.argtypes = [i32, vp, i64, i64, vp, i64, vp, i32, vp]
        L.kq_matmul_id_glu.argtypes = [i32, vp, vp, i64, i64, i64, i64, vp, i32, i64, vp, i64, vp, i32,
                                       i32, vp, sz, vp]
        L.kq_matmul_id_mix_workspace_bytes.argtypes = [i64, i64, i64, i64]
        L.kq_matmul_id_mix_workspace_bytes.restype = sz
        L.kq_matmul_id_mix.argtypes = [i32, vp, i64, i64, i64, i64, vp, i32, i64, vp, vp, i64, vp, i32,
                                       vp, sz, i32, vp]
        if DEBUG_LIBRARY:
            L.kq_debug_wait_timeout.argtypes = [i32, vp]
            L.kq_debug_wait_timeout.restype = i32
            L.kq_debug_spin_limit.argtypes = []
            L.kq_debug_spin_limit.restype = i32
        L.kq_device_status.argtypes = [vp]
        L.kq_status_string.argtypes = [i32]
        L.kq_status_string.restype = ctypes.c_char_p
        for f in ("kq_block_weights", "kq_block_bytes", "kq_dequantize", "kq_matmul",
                  "kq_matmul_ex", "kq_matmul_id", "kq_matmul_id_ex", "kq_moe_group", "kq_validate",
                  "kq_device_status", "kq_get_rows", "kq_matmul_id_glu", "kq_matmul_id_mix"):
            getattr(L, f).restype = i32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kq_status_string(int(status)).decode()


def _check(st: int, what: str):
    if st != 0:
        raise KQError(st, what)


def _codec(c) -> int:
    return CODECS[c] if isinstance(c, str) else int(c)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr())


def block_weights(codec) -> int:
    return lib().kq_block_weights(_codec(codec))


def block_bytes(codec) -> int:
    return lib().kq_block_bytes(_codec(codec))


def row_bytes(codec, k: int) -> int:
    return int(lib().kq_row_bytes(_codec(codec), int(k)))


def _on_current_device(name: str, t: torch.Tensor):
    # the library works on the current CUDA device; its pointers must live there
    if not t.is_cuda or t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} must be a CUDA tensor on the current device, not {t.device}")


def _check_tensor(name: str, t: torch.Tensor, shape, dtypes, device):
    """The C ABI takes plain pointers, so sizes are checked here: a buffer of
    the wrong shape would be read or written past its end."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}; expected one of {sorted(map(str, dtypes))}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the weights on {device}")


_ACT = (torch.float32, torch.bfloat16)


def _weights(w: torch.Tensor, codec: int, k: int):
    if w.dtype != torch.uint8 or not w.is_contiguous() or not w.is_cuda:
        raise ValueError("w must be a contiguous uint8 CUDA tensor of wire blocks")
    _on_current_device("w", w)
    rb = row_bytes(codec, k)
    if rb <= 0 or w.numel() % rb:
        raise ValueError(f"w holds {w.numel()} bytes, not a whole number of {rb}-byte rows")
    return w.numel() // rb


def dequantize(w: torch.Tensor, codec, k: int, dtype=torch.float32, out=None) -> torch.Tensor:
    """Decode wire blocks [rows, row_bytes] into a [rows, k] float tensor."""
    c = _codec(codec)
    rows = _weights(w, c, k)
    if out is None:
        out = torch.empty((rows, k), dtype=dtype, device=w.device)
    _check_tensor("out", out, (rows, k), tuple(_DT), w.device)
    _check(lib().kq_dequantize(c, _ptr(w), rows, k, _ptr(out), _DT[out.dtype], _stream()),
           "kq_dequantize")
    return out


def get_rows(w: torch.Tensor, codec, k: int, ids: torch.Tensor, dtype=torch.float32,
             out=None) -> torch.Tensor:
    """out[t] = decode of row ids[t] of w ([rows, row_bytes] wire blocks); an id
    outside the table gives a zero row and sets the device error word."""
    c = _codec(codec)
    rows = _weights(w, c, k)
    if ids.dim() != 1:
        raise ValueError("ids must be a 1-D int32 tensor")
    _check_tensor("ids", ids, (ids.shape[0],), (torch.int32,), w.device)
    if out is None:
        out = torch.empty((ids.shape[0], k), dtype=dtype, device=w.device)
    _check_tensor("out", out, (ids.shape[0], k), tuple(_DT), w.device)
    _check(lib().kq_get_rows(c, _ptr(w), rows, k, _ptr(ids), ids.shape[0], _ptr(out), _DT[out.dtype],
                             _stream()), "kq_get_rows")
    return out


def matmul(w: torch.Tensor, codec, x: torch.Tensor, out=None, out_dtype=torch.float32,
           path: int = PATH_AUTO, const_weights: bool = False,
           independent: bool = False) -> torch.Tensor:
    """y[m, n] = sum_k dequant(w)[n, k] * x[m, k]; x [m, k] fp32/bf16.

    const_weights: no earlier work on the stream writes w.
    independent: no earlier work on the stream writes w or x, or touches
    out; consecutive independent calls may then run side by side."""
    c = _codec(codec)
    if x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous [m, k] tensor")
    m, k = x.shape
    n = _weights(w, c, k)
    _check_tensor("x", x, (m, k), _ACT, w.device)
    if out is None:
        out = torch.empty((m, n), dtype=out_dtype, device=x.device)
    _check_tensor("out", out, (m, n), _ACT, w.device)
    flags = path | (FLAG_CONST_WEIGHTS if const_weights else 0) | (FLAG_INDEPENDENT if independent else 0)
    _check(lib().kq_matmul_ex(c, _ptr(w), n, k, _ptr(x), _DT[x.dtype], m, _ptr(out),
                              _DT[out.dtype], flags, _stream()), "kq_matmul")
    return out


def matmul_id_workspace_bytes(n_tokens: int, top_k: int, n_experts: int) -> int:
    return int(lib().kq_matmul_id_workspace_bytes(n_tokens, top_k, n_experts))


def matmul_id(w: torch.Tensor, codec, x: torch.Tensor, ids: torch.Tensor, out=None,
              out_dtype=torch.float32, workspace=None, path: int = PATH_AUTO) -> torch.Tensor:
    """y[t, s, n] = sum_k dequant(w[ids[t, s]])[n, k] * x[t, k].
    w: [E, n, row_bytes] uint8; x: [T, k]; ids: [T, top_k] int32."""
    c = _codec(codec)
    if w.dim() != 3 or w.dtype != torch.uint8:
        raise ValueError("w must be uint8 [n_experts, n, row_bytes]")
    e, n, rb = w.shape
    if x.dim() != 2:
        raise ValueError("x must be [n_tokens, k]")
    t, k = x.shape
    if rb != row_bytes(c, k):
        raise ValueError("w's last dimension does not match k")
    # rows of one expert packed back to back; experts w.stride(0) bytes apart
    if w.stride(2) != 1 or w.stride(1) != rb:
        raise ValueError("each expert's rows must be packed back to back")
    _on_current_device("w", w)
    _check_tensor("x", x, (t, k), _ACT, w.device)
    if ids.dim() != 2:
        raise ValueError("ids must be int32 [n_tokens, top_k]")
    top_k = ids.shape[1]
    _check_tensor("ids", ids, (t, top_k), (torch.int32,), w.device)
    if out is None:
        out = torch.empty((t, top_k, n), dtype=out_dtype, device=x.device)
    _check_tensor("out", out, (t, top_k, n), _ACT, w.device)
    need = matmul_id_workspace_bytes(t, top_k, e)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.device != w.device:
        raise ValueError("workspace must be a contiguous uint8 tensor on the weights' device")
    _check(lib().kq_matmul_id_ex(c, _ptr(w), e, n, k, w.stride(0), _ptr(x), _DT[x.dtype], t,
                                 _ptr(ids), top_k, _ptr(out), _DT[out.dtype], _ptr(workspace),
                                 workspace.numel(), path, _stream()), "kq_matmul_id")
    return out


ACTS = {"silu": 0, "gelu": 1}


def matmul_id_glu(w_gate: torch.Tensor, w_up: torch.Tensor, codec, x: torch.Tensor, ids: torch.Tensor,
                  act: str = "silu", out=None, out_dtype=torch.float32, workspace=None) -> torch.Tensor:
    """y[t, s, n] = act(x[t] @ dequant(w_gate[e])^T)[n] * (x[t] @ dequant(w_up[e])^T)[n],
    e = ids[t, s]; act 'silu' or 'gelu' (tanh approximation).  Stacks as matmul_id."""
    c = _codec(codec)
    for nm, w in (("w_gate", w_gate), ("w_up", w_up)):
        if w.dim() != 3 or w.dtype != torch.uint8:
            raise ValueError(f"{nm} must be uint8 [n_experts, n, row_bytes]")
        _on_current_device(nm, w)
    if w_up.shape != w_gate.shape or w_up.stride() != w_gate.stride():
        raise ValueError("w_gate and w_up must have the same shape and layout")
    e, n, rb = w_gate.shape
    if x.dim() != 2:
        raise ValueError("x must be [n_tokens, k]")
    t, k = x.shape
    if rb != row_bytes(c, k):
        raise ValueError("the stacks' last dimension does not match k")
    if w_gate.stride(2) != 1 or w_gate.stride(1) != rb:
        raise ValueError("each expert's rows must be packed back to back")
    _check_tensor("x", x, (t, k), _ACT, w_gate.device)
    if ids.dim() != 2:
        raise ValueError("ids must be int32 [n_tokens, top_k]")
    top_k = ids.shape[1]
    _check_tensor("ids", ids, (t, top_k), (torch.int32,), w_gate.device)
    if act not in ACTS:
        raise ValueError(f"act must be one of {sorted(ACTS)}")
    if out is None:
        out = torch.empty((t, top_k, n), dtype=out_dtype, device=x.device)
    _check_tensor("out", out, (t, top_k, n), _ACT, w_gate.device)
    need = matmul_id_workspace_bytes(t, top_k, e)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.device != w_gate.device:
        raise ValueError("workspace must be a contiguous uint8 tensor on the weights' device")
    _check(lib().kq_matmul_id_glu(c, _ptr(w_gate), _ptr(w_up), e, n, k, w_gate.stride(0), _ptr(x),
                                  _DT[x.dtype], t, _ptr(ids), top_k, _ptr(out), _DT[out.dtype], ACTS[act],
                                  _ptr(workspace), workspace.numel(), _stream()), "kq_matmul_id_glu")
    return out


FLAG_REUSE_GROUPING = 0x400


def matmul_id_mix_workspace_bytes(n_tokens: int, top_k: int, n_experts: int, n: int) -> int:
    return int(lib().kq_matmul_id_mix_workspace_bytes(n_tokens, top_k, n_experts, n))


def matmul_id_mix(w: torch.Tensor, codec, x: torch.Tensor, ids: torch.Tensor, scores: torch.Tensor,
                  out=None, out_dtype=torch.float32, workspace=None, path: int = PATH_AUTO,
                  reuse_grouping: bool = False) -> torch.Tensor:
    """y[t, n] = sum_s scores[t, s] * (x[t, s] @ dequant(w[ids[t, s]])^T)[n].
    w: [E, n, row_bytes] uint8; x: [T, top_k, k] (one row per routed slot);
    ids: [T, top_k] int32; scores: [T, top_k] float32.  reuse_grouping: the
    workspace already holds the grouping of these ids from an earlier
    expert-indexed call on this stream (see kq.h)."""
    c = _codec(codec)
    if w.dim() != 3 or w.dtype != torch.uint8:
        raise ValueError("w must be uint8 [n_experts, n, row_bytes]")
    e, n, rb = w.shape
    if x.dim() != 3:
        raise ValueError("x must be [n_tokens, top_k, k]")
    t, top_k, k = x.shape
    if rb != row_bytes(c, k):
        raise ValueError("w's last dimension does not match k")
    if w.stride(2) != 1 or w.stride(1) != rb:
        raise ValueError("each expert's rows must be packed back to back")
    _on_current_device("w", w)
    _check_tensor("x", x, (t, top_k, k), _ACT, w.device)
    _check_tensor("ids", ids, (t, top_k), (torch.int32,), w.device)
    _check_tensor("scores", scores, (t, top_k), (torch.float32,), w.device)
    if out is None:
        out = torch.empty((t, n), dtype=out_dtype, device=x.device)
    _check_tensor("out", out, (t, n), _ACT, w.device)
    need = matmul_id_mix_workspace_bytes(t, top_k, e, n)
    if workspace is None:
        if reuse_grouping:
            raise ValueError("reuse_grouping needs the workspace that holds the grouping")
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.device != w.device:
        raise ValueError("workspace must be a contiguous uint8 tensor on the weights' device")
    flags = path | (FLAG_REUSE_GROUPING if reuse_grouping else 0)
    _check(lib().kq_matmul_id_mix(c, _ptr(w), e, n, k, w.stride(0), _ptr(x), _DT[x.dtype], t,
                                  _ptr(ids), _ptr(scores), top_k, _ptr(out), _DT[out.dtype],
                                  _ptr(workspace), workspace.numel(), flags, _stream()),
           "kq_matmul_id_mix")
    return out


def moe_group(ids: torch.Tensor, n_experts: int):
    """(counts [E], offsets [E+1], perm [P]) of the device-side expert grouping."""
    if ids.dtype != torch.int32:
        raise ValueError("ids must be int32")
    _on_current_device("ids", ids)
    ids = ids.contiguous().view(-1)
    p = ids.numel()
    counts = torch.empty(n_experts, dtype=torch.int32, device=ids.device)
    offsets = torch.empty(n_experts + 1, dtype=torch.int32, device=ids.device)
    perm = torch.empty(p, dtype=torch.int32, device=ids.device)
    _check(lib().kq_moe_group(_ptr(ids), p, n_experts, _ptr(counts), _ptr(offsets), _ptr(perm),
                              _stream()), "kq_moe_group")
    return counts, offsets, perm


def validate(w: torch.Tensor, codec, k: int) -> int:
    """Index of the first block with an illegal TQ1 byte, or -1 (synchronizes)."""
    c = _codec(codec)
    rows = _weights(w, c, k)
    out = ctypes.c_int64(-1)
    _check(lib().kq_validate(c, _ptr(w), rows, k, ctypes.byref(out), _stream()), "kq_validate")
    return out.value


def device_status() -> int:
    """Synchronize and return (and clear) the device error word as a status code."""
    return int(lib().kq_device_status(_stream()))


def debug_wait_timeout(mode: int = 0) -> None:
    """KQ_DEBUG build only: launch one warp whose bounded wait runs out (mode 0
    the suspending wait loop, 1 the test-and-sleep loop); the next
    device_status() returns -10 (KQ_ERR_DEVICE_TIMEOUT)."""
    if not DEBUG_LIBRARY:
        raise RuntimeError("debug_wait_timeout needs the KQ_DEBUG build (KQ_DEBUG_LIBRARY=1)")
    _check(lib().kq_debug_wait_timeout(int(mode), _stream()), "kq_debug_wait_timeout")
