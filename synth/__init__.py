"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke run.

This module only draws random bytes and numbers and places them in the wire
fields of each block.  It holds none of the decode or product arithmetic: the
oracle (``oracle/``) and the CUDA library (``block_quantized_matmul_quant_b200``)
each decode these bytes with code of their own.

Draw order (numpy ``Generator(PCG64(seed))``), fixed so a seed names one input:

* weights, per codec, field by field in the order listed for ``gen_weights``,
  each field drawn for all blocks at once in row-major block order;
* activations ``x``: one ``standard_normal`` draw of ``M*K`` float32 values,
  rounded to bf16 (round to nearest even) when ``dtype == "bf16"``;
* MoE ids: per token, the first ``top_k`` entries of one permutation of
  ``0..E-1`` (experts drawn uniformly without replacement).

Value distributions (the workloads' own):

* Q8_0 (mlx-kquant / ds4 ``block_q8_0``): fp16 scale ``d`` uniform in
  [2^-8, 2^-4] rounded to fp16; int8 quants uniform in [-127, 127].
* Q4_K: fp16 ``d`` and ``dmin`` uniform in [2^-10, 2^-6]; the 12 packed
  scale/min bytes uniform in 0..255 (each of the 96 bits feeds exactly one
  6-bit field, so every scale and min is uniform in 0..63); the 128 quant
  bytes uniform (both nibbles uniform in 0..15).
* Q2_K: fp16 ``d`` and ``dmin`` as Q4_K; the 16 scale/min bytes and the 64
  quant bytes uniform in 0..255.
* Q5_K: as Q4_K, plus the 32 high-bit bytes uniform (every fifth bit uniform).
* Q6_K: fp16 ``d`` as Q4_K; the 128 low-bit bytes, the 64 high-bit bytes and
  the 16 int8 scales uniform over their byte values.
* TQ1_G128 (Ternary Bonsai ``ternel_packed_model.py``): 25 full code bytes
  uniform in 0..242 (five i.i.d. uniform trits), one tail byte uniform in
  0..26 (three trits), fp16 scale uniform in [2^-6, 2^-2].
"""
from __future__ import annotations

import dataclasses

import numpy as np

# Wire codec identifiers (GGML type numbers for the GGML codecs).
Q8_0 = 8
Q2_K = 10
Q4_K = 12
Q5_K = 13
Q6_K = 14
TQ1_G128 = 1001

CODEC_NAMES = {Q8_0: "q8_0", Q2_K: "q2_k", Q4_K: "q4_k", Q5_K: "q5_k", Q6_K: "q6_k", TQ1_G128: "tq1_g128"}
CODECS_BY_NAME = {v: k for k, v in CODEC_NAMES.items()}

# (weights per block, bytes per block) -- only used to size the byte arrays.
_GEOMETRY = {Q8_0: (32, 34), Q2_K: (256, 84), Q4_K: (256, 144), Q5_K: (256, 176), Q6_K: (256, 210),
             TQ1_G128: (128, 28)}


def geometry(codec: int) -> tuple[int, int]:
    return _GEOMETRY[codec]


def row_bytes(codec: int, k: int) -> int:
    qk, bb = _GEOMETRY[codec]
    if k % qk:
        raise ValueError(f"K={k} is not a multiple of {qk}")
    return (k // qk) * bb


def _fp16_bytes(values: np.ndarray) -> np.ndarray:
    """Round float64 values to fp16 (numpy's cast is round-to-nearest-even)
    and return their little-endian bytes, shape [..., 2]."""
    h = values.astype(np.float16).astype("<f2")
    return h.view(np.uint8).reshape(values.shape + (2,))


def gen_weights(codec: int, rows: int, k: int, rng: np.random.Generator) -> np.ndarray:
    """Wire bytes for a ``rows x k`` weight matrix, shape [rows, row_bytes].

    Field draw order per codec:
      Q8_0:  d, qs
      Q4_K:  d, dmin, scales[12], qs[128]
      Q2_K:  d, dmin, scales[16], qs[64]
      Q5_K:  d, dmin, scales[12], qh[32], qs[128]
      Q6_K:  d, ql[128], qh[64], scales[16]
      TQ1:   full codes[25], tail, scale
    """
    qk, bb = _GEOMETRY[codec]
    if k % qk:
        raise ValueError(f"K={k} is not a multiple of {qk}")
    nb = rows * (k // qk)
    out = np.empty((nb, bb), dtype=np.uint8)
    if codec == Q8_0:
        d = rng.uniform(2.0 ** -8, 2.0 ** -4, size=nb)
        qs = rng.integers(-127, 128, size=(nb, 32), dtype=np.int64).astype(np.int8)
        out[:, 0:2] = _fp16_bytes(d)
        out[:, 2:34] = qs.view(np.uint8)
    elif codec == Q4_K:
        d = rng.uniform(2.0 ** -10, 2.0 ** -6, size=nb)
        dmin = rng.uniform(2.0 ** -10, 2.0 ** -6, size=nb)
        sc = rng.integers(0, 256, size=(nb, 12), dtype=np.int64).astype(np.uint8)
        qs = rng.integers(0, 256, size=(nb, 128), dtype=np.int64).astype(np.uint8)
        out[:, 0:2] = _fp16_bytes(d)
        out[:, 2:4] = _fp16_bytes(dmin)
        out[:, 4:16] = sc
        out[:, 16:144] = qs
    elif codec == Q2_K:
        d = rng.uniform(2.0 ** -10, 2.0 ** -6, size=nb)
        dmin = rng.uniform(2.0 ** -10, 2.0 ** -6, size=nb)
        sc = rng.integers(0, 256, size=(nb, 16), dtype=np.int64).astype(np.uint8)
        qs = rng.integers(0, 256, size=(nb, 64), dtype=np.int64).astype(np.uint8)
        out[:, 0:16] = sc
        out[:, 16:80] = qs
        out[:, 80:82] = _fp16_bytes(d)
        out[:, 82:84] = _fp16_bytes(dmin)
    elif codec == Q5_K:
        d = rng.uniform(2.0 ** -10, 2.0 ** -6, size=nb)
        dmin = rng.uniform(2.0 ** -10, 2.0 ** -6, size=nb)
        sc = rng.integers(0, 256, size=(nb, 12), dtype=np.int64).astype(np.uint8)
        qh = rng.integers(0, 256, size=(nb, 32), dtype=np.int64).astype(np.uint8)
        qs = rng.integers(0, 256, size=(nb, 128), dtype=np.int64).astype(np.uint8)
        out[:, 0:2] = _fp16_bytes(d)
        out[:, 2:4] = _fp16_bytes(dmin)
        out[:, 4:16] = sc
        out[:, 16:48] = qh
        out[:, 48:176] = qs
    elif codec == Q6_K:
        d = rng.uniform(2.0 ** -10, 2.0 ** -6, size=nb)
        ql = rng.integers(0, 256, size=(nb, 128), dtype=np.int64).astype(np.uint8)
        qh = rng.integers(0, 256, size=(nb, 64), dtype=np.int64).astype(np.uint8)
        sc = rng.integers(0, 256, size=(nb, 16), dtype=np.int64).astype(np.uint8)
        out[:, 0:128] = ql
        out[:, 128:192] = qh
        out[:, 192:208] = sc
        out[:, 208:210] = _fp16_bytes(d)
    elif codec == TQ1_G128:
        full = rng.integers(0, 243, size=(nb, 25), dtype=np.int64).astype(np.uint8)
        tail = rng.integers(0, 27, size=nb, dtype=np.int64).astype(np.uint8)
        scale = rng.uniform(2.0 ** -6, 2.0 ** -2, size=nb)
        out[:, 0:25] = full
        out[:, 25] = tail
        out[:, 26:28] = _fp16_bytes(scale)
    else:
        raise ValueError(f"unknown codec {codec}")
    return out.reshape(rows, (k // qk) * bb)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bf16 value (ties to even), returned as float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x_bf16_valued: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are exactly bf16 values."""
    u = np.ascontiguousarray(x_bf16_valued, dtype=np.float32).view(np.uint32)
    return (u >> 16).astype(np.uint16)


def gen_x(m: int, k: int, dtype: str, rng: np.random.Generator) -> np.ndarray:
    """Activations ~N(0,1), shape [m, k], float32 holding the exact values of
    the requested dtype ("f32" or "bf16")."""
    x = rng.standard_normal(size=(m, k), dtype=np.float32)
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return x
    raise ValueError(dtype)


def gen_ids(n_tokens: int, top_k: int, n_experts: int, rng: np.random.Generator) -> np.ndarray:
    """Per-token top_k distinct expert ids, int32 [n_tokens, top_k]."""
    ids = np.empty((n_tokens, top_k), dtype=np.int32)
    for t in range(n_tokens):
        ids[t] = rng.permutation(n_experts)[:top_k]
    return ids


@dataclasses.dataclass(frozen=True)
class Workload:
    """One of the five measured configurations."""

    name: str
    kind: str          # "gemv", "gemm" or "moe"
    codec: int
    n: int             # weight rows (output features)
    k: int             # reduction length
    m: int             # activation rows (tokens)
    x_dtype: str
    y_dtype: str
    n_experts: int = 0
    top_k: int = 0
    seed: int = 0

    def weight_bytes(self) -> int:
        per = self.n * row_bytes(self.codec, self.k)
        return per * (self.n_experts if self.kind == "moe" else 1)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("q8_0_gemv_256x1024", "gemv", Q8_0, 256, 1024, 1, "f32", "f32"),
        Workload("q4_k_gemv_4096x4096", "gemv", Q4_K, 4096, 4096, 1, "bf16", "f32"),
        Workload("q4_k_gemm_512x11008x4096", "gemm", Q4_K, 11008, 4096, 512, "bf16", "bf16"),
        Workload("moe_q4_k_e64_1408x2048_t32_top6", "moe", Q4_K, 1408, 2048, 32, "bf16", "f32",
                 n_experts=64, top_k=6),
        Workload("tq1_g128_gemv_5120x17408", "gemv", TQ1_G128, 5120, 17408, 1, "bf16", "f32"),
        Workload("tq1_g128_gemm_512x5120x17408", "gemm", TQ1_G128, 5120, 17408, 512, "bf16", "bf16"),
    )
}


def make_inputs(w: Workload, seed: int | None = None):
    """(weights u8, x f32-valued, ids or None) for a workload, in draw order
    weights -> x -> ids from one generator."""
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    rows = w.n * (w.n_experts if w.kind == "moe" else 1)
    wq = gen_weights(w.codec, rows, w.k, rng)
    if w.kind == "moe":
        wq = wq.reshape(w.n_experts, w.n, -1)
    x = gen_x(w.m, w.k, w.x_dtype, rng)
    ids = gen_ids(w.m, w.top_k, w.n_experts, rng) if w.kind == "moe" else None
    return wq, x, ids
