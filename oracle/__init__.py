"""CPU oracle for block-quantized matrix products (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``kq_oracle.c`` (plain C, fp64
accumulation; see that file's header for the codec definitions and the
passages they follow) through ctypes, and shares nothing with the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kq_oracle.c")
_LIB = os.path.join(_HERE, "libkq_oracle.so")

Q8_0, Q2_K, Q4_K, Q5_K, Q6_K, TQ1_G128 = 8, 10, 12, 13, 14, 1001


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64 = ctypes.c_int64
        lib.kqo_block_weights.argtypes = [ctypes.c_int]
        lib.kqo_block_bytes.argtypes = [ctypes.c_int]
        lib.kqo_decode.argtypes = [ctypes.c_int, u8p, i64, i64, i64, f32p, f64p]
        lib.kqo_decode.restype = ctypes.c_int
        lib.kqo_tq1_first_illegal.argtypes = [u8p, i64, i64, i64]
        lib.kqo_tq1_first_illegal.restype = i64
        lib.kqo_matmul.argtypes = [ctypes.c_int, u8p, i64, i64, i64, f64p, i64, f64p, ctypes.c_int]
        lib.kqo_matmul.restype = ctypes.c_int
        lib.kqo_matmul_id.argtypes = [ctypes.c_int, u8p, i64, i64, i64, i64, i64, f64p, i64,
                                      i32p, i64, f64p]
        lib.kqo_matmul_id.restype = ctypes.c_int
        lib.kqo_get_rows.argtypes = [ctypes.c_int, u8p, i64, i64, i64, i32p, i64, f32p]
        lib.kqo_get_rows.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def block_weights(codec: int) -> int:
    return _load().kqo_block_weights(codec)


def block_bytes(codec: int) -> int:
    return _load().kqo_block_bytes(codec)


def row_bytes(codec: int, k: int) -> int:
    return (k // block_weights(codec)) * block_bytes(codec)


def _as_rows(w: np.ndarray, codec: int, k: int) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.uint8)
    return w.reshape(-1, row_bytes(codec, k))


def decode_f32(codec: int, w: np.ndarray, k: int) -> np.ndarray:
    """fp32 decode (the IEEE operation sequence of the codec's definition)."""
    w = _as_rows(w, codec, k)
    out = np.empty((w.shape[0], k), dtype=np.float32)
    st = _load().kqo_decode(codec, _ptr(w, ctypes.c_uint8), w.shape[0], k, w.shape[1],
                            _ptr(out, ctypes.c_float), None)
    if st:
        raise ValueError("oracle decode rejected the arguments")
    return out


def decode_f64(codec: int, w: np.ndarray, k: int) -> np.ndarray:
    """Exact decoded weight values held in fp64."""
    w = _as_rows(w, codec, k)
    out = np.empty((w.shape[0], k), dtype=np.float64)
    st = _load().kqo_decode(codec, _ptr(w, ctypes.c_uint8), w.shape[0], k, w.shape[1],
                            None, _ptr(out, ctypes.c_double))
    if st:
        raise ValueError("oracle decode rejected the arguments")
    return out


def tq1_first_illegal(w: np.ndarray, k: int) -> int:
    w = _as_rows(w, TQ1_G128, k)
    return int(_load().kqo_tq1_first_illegal(_ptr(w, ctypes.c_uint8), w.shape[0], k, w.shape[1]))


def matmul(codec: int, w: np.ndarray, k: int, x: np.ndarray, threads: int = 1) -> np.ndarray:
    """Y[m, n] = sum_k W[n, k] X[m, k] in fp64.  w: [N, row_bytes] u8; x: [M, K]."""
    w = _as_rows(w, codec, k)
    x = np.ascontiguousarray(x, dtype=np.float64).reshape(-1, k)
    y = np.empty((x.shape[0], w.shape[0]), dtype=np.float64)
    st = _load().kqo_matmul(codec, _ptr(w, ctypes.c_uint8), w.shape[0], k, w.shape[1],
                            _ptr(x, ctypes.c_double), x.shape[0], _ptr(y, ctypes.c_double),
                            int(threads))
    if st:
        raise ValueError(f"oracle matmul failed ({st})")
    return y


def matmul_id(codec: int, w: np.ndarray, k: int, x: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Y[t, s, n] = sum_k W[ids[t, s], n, k] X[t, k] in fp64; NaN rows for bad ids.
    w: [E, N, row_bytes] u8; x: [T, K]; ids: [T, top_k] int32."""
    w = np.ascontiguousarray(w, dtype=np.uint8)
    e, n, rb = w.shape
    x = np.ascontiguousarray(x, dtype=np.float64).reshape(-1, k)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    t, top_k = ids.shape
    y = np.empty((t, top_k, n), dtype=np.float64)
    st = _load().kqo_matmul_id(codec, _ptr(w, ctypes.c_uint8), e, n, k, rb, n * rb,
                               _ptr(x, ctypes.c_double), t, _ptr(ids, ctypes.c_int32), top_k,
                               _ptr(y, ctypes.c_double))
    if st:
        raise ValueError(f"oracle matmul_id failed ({st})")
    return y


def get_rows(codec: int, w: np.ndarray, k: int, ids: np.ndarray) -> np.ndarray:
    """out[t] = fp32 decode of row ids[t] of w; ids outside the table give
    an all-zero row.  w: [rows, row_bytes] u8; ids: int32 [T]."""
    w = _as_rows(w, codec, k)
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    out = np.empty((ids.size, k), dtype=np.float32)
    st = _load().kqo_get_rows(codec, _ptr(w, ctypes.c_uint8), w.shape[0], k, w.shape[1],
                              _ptr(ids, ctypes.c_int32), ids.size, _ptr(out, ctypes.c_float))
    if st:
        raise ValueError(f"oracle get_rows failed ({st})")
    return out


def act_f64(g: np.ndarray, act: str) -> np.ndarray:
    """The GLU activations of mlx-kquant `moe_glu_gather_kq`, in fp64:
    'silu': g * sigmoid(g) = g / (1 + exp(-g));
    'gelu': the tanh approximation 0.5 * g * (1 + tanh(sqrt(2/pi) * (g + 0.044715 g^3)))."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        if act == "silu":
            return g / (1.0 + np.exp(-g))
        if act == "gelu":
            return 0.5 * g * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (g + 0.044715 * g ** 3)))
    raise ValueError(act)


def glu_id(codec: int, w_gate: np.ndarray, w_up: np.ndarray, k: int, x: np.ndarray, ids: np.ndarray,
           act: str = "silu") -> np.ndarray:
    """Fused MoE GLU (mlx-kquant bindings.cpp `moe_glu_gather_kq`): for every
    token t and slot s with e = ids[t][s],
        y[t][s] = act(x[t] @ dequant(w_gate[e])^T) * (x[t] @ dequant(w_up[e])^T),
    in fp64; an id outside [0, E) gives a NaN row.  w_*: [E, N, row_bytes]."""
    g = matmul_id(codec, w_gate, k, x, ids)
    u = matmul_id(codec, w_up, k, x, ids)
    return act_f64(g, act) * u


def mix_id(codec: int, w: np.ndarray, k: int, x_slotted: np.ndarray, ids: np.ndarray,
           scores: np.ndarray) -> np.ndarray:
    """MoE down projection with the routing mix folded in (mlx-kquant
    `gather_qmv_mix_kq`; slotted input of mlx-native's pooled slotted mm_id):
    every (token, slot) pair has its own activation row x[t][s] and
        y[t] = sum_s scores[t][s] * (x[t][s] @ dequant(w[ids[t][s]])^T),
    in fp64, slots summed in order; a token with an id outside [0, E) gets a
    NaN row.  w: [E, N, row_bytes]; x: [T, top_k, K]; ids, scores: [T, top_k]."""
    w = np.ascontiguousarray(w, dtype=np.uint8)
    e, n, rb = w.shape
    x = np.asarray(x_slotted, dtype=np.float64)
    t, top_k, kk = x.shape
    assert kk == k and ids.shape == (t, top_k) and scores.shape == (t, top_k)
    dec = decode_f64(codec, w.reshape(e * n, rb), k).reshape(e, n, k)
    y = np.zeros((t, n))
    for tt in range(t):
        for s in range(top_k):
            ee = int(ids[tt, s])
            if ee < 0 or ee >= e:
                y[tt, :] = np.nan
                break
            y[tt] += float(scores[tt, s]) * (dec[ee] @ x[tt, s])
    return y
