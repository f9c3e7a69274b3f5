"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test pins one part of the oracle to something other than itself: the
constants printed on the pages (tests/golden/), hand-built blocks whose values
follow in closed form, exhaustive enumeration of the trit code, a library
routine (numpy fp64 matmul) on tiny inputs, and special cases of the product.
The block packers below are encoders written from the layout description;
they share no code with the oracle's decoders.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CODECS = {"q8_0": 8, "q2_k": 10, "q4_k": 12, "q5_k": 13, "q6_k": 14, "tq1_g128": 1001}


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def f16(v):
    """fp16 little-endian bytes of a value that must be exactly representable."""
    h = np.array([v], dtype=np.float16)
    assert float(h[0]) == v, v
    return h.view(np.uint8).tolist()


# ---------------------------------------------------------------- geometry

def test_block_geometry_matches_pages():
    for name, qk, bb, *_ in _golden_rows("block_geometry.txt"):
        c = CODECS[name]
        assert oracle.block_weights(c) == int(qk)
        assert oracle.block_bytes(c) == int(bb)
        assert synth.geometry(c) == (int(qk), int(bb))


def test_row_bytes_of_workloads():
    # Q8_0 row bytes per ds4's formula (K/32)*34; TQ1 per canonical_bytes.
    assert oracle.row_bytes(8, 1024) == (1024 // 32) * 34 == 1088
    assert oracle.row_bytes(12, 4096) == 2304
    assert oracle.row_bytes(1001, 17408) == 3808
    for label, rows, cols, _ in _golden_rows("tq1_shape_census.txt"):
        rows, cols = int(rows), int(cols)
        assert rows * oracle.row_bytes(1001, cols) == rows * (cols // 128) * 28
    # mlp.down_proj is the 5120 x 17408 TQ1 workload: 19 496 960 bytes.
    assert 5120 * oracle.row_bytes(1001, 17408) == 19_496_960


def test_shape_census_sums_to_page_total():
    rows = _golden_rows("tq1_shape_census.txt")
    assert sum(int(r[3]) for r in rows) == 497


# ---------------------------------------------------------------- Q8_0

def q8_0_block(d, qs):
    assert len(qs) == 32
    return bytes(f16(d) + [q & 0xFF for q in qs])


def test_q8_0_hand_block_identity():
    b = q8_0_block(1.0, [i - 16 for i in range(32)])
    w = oracle.decode_f32(8, np.frombuffer(b, np.uint8), 32)[0]
    assert w.tolist() == [float(i - 16) for i in range(32)]


def test_q8_0_scale_sign_and_subnormal():
    qs = [127, -127, 1, -1, 0] + [5] * 27
    for d in (-0.5, 2.0 ** -24, 65504.0):
        b = q8_0_block(d, qs)
        w = oracle.decode_f32(8, np.frombuffer(b, np.uint8), 32)[0]
        assert w.tolist() == [float(np.float32(d) * np.float32(q)) for q in qs]


# ---------------------------------------------------------------- Q4_K

def pack_q4_k(d, dmin, sc, mn, q):
    """Encoder for one GGUF Q4_K block: the inverse mapping of the layout,
    built field by field (scales of sub-blocks 0..3 in the low six bits of
    bytes 0..3, mins in bytes 4..7; sub-blocks 4..7 put their low four scale
    bits in the low nibble of bytes 8..11, low four min bits in the high
    nibble, and their top two bits in the high bits of bytes 0..3 (scale)
    and 4..7 (min)); quants: byte 32c+l holds weight 64c+l in its low nibble
    and weight 64c+32+l in its high nibble."""
    assert len(sc) == len(mn) == 8 and len(q) == 256
    s = [0] * 12
    for j in range(8):
        assert 0 <= sc[j] < 64 and 0 <= mn[j] < 64
        if j < 4:
            s[j] |= sc[j]
            s[j + 4] |= mn[j]
        else:
            s[j + 4] |= (sc[j] & 15) | ((mn[j] & 15) << 4)
            s[j - 4] |= (sc[j] >> 4) << 6
            s[j] |= (mn[j] >> 4) << 6
    qs = [0] * 128
    for c in range(4):
        for l in range(32):
            lo, hi = q[64 * c + l], q[64 * c + 32 + l]
            assert 0 <= lo < 16 and 0 <= hi < 16
            qs[32 * c + l] = lo | (hi << 4)
    return bytes(f16(d) + f16(dmin) + s + qs)


def q4_k_expected(d, dmin, sc, mn, q):
    return [Fraction(d) * sc[i // 32] * q[i] - Fraction(dmin) * mn[i // 32] for i in range(256)]


def _check_block(codec, blob, expected, k=256):
    w64 = oracle.decode_f64(codec, np.frombuffer(blob, np.uint8), k)[0]
    w32 = oracle.decode_f32(codec, np.frombuffer(blob, np.uint8), k)[0]
    for i, e in enumerate(expected):
        assert Fraction(float(w64[i])) == e, (i, w64[i], e)
        # one rounding of the exact value (products are exact)
        assert w32[i] == np.float32(float(e)), (i, w32[i], e)


def test_q4_k_unit_scales_give_quants():
    q = [(7 * i + 3) % 16 for i in range(256)]
    blob = pack_q4_k(1.0, 0.0, [1] * 8, [0] * 8, q)
    w = oracle.decode_f32(12, np.frombuffer(blob, np.uint8), 256)[0]
    assert w.tolist() == [float(v) for v in q]


@pytest.mark.parametrize("j", range(8))
@pytest.mark.parametrize("val", [0, 1, 32, 63])
def test_q4_k_each_scale_and_min_field(j, val):
    q = [(5 * i + 1) % 16 for i in range(256)]
    sc = [1] * 8
    sc[j] = val
    blob = pack_q4_k(0.5, 0.25, sc, [0] * 8, q)
    _check_block(12, blob, q4_k_expected(0.5, 0.25, sc, [0] * 8, q))
    mn = [0] * 8
    mn[j] = val
    blob = pack_q4_k(0.5, 0.25, [1] * 8, mn, q)
    _check_block(12, blob, q4_k_expected(0.5, 0.25, [1] * 8, mn, q))


def test_q4_k_random_blocks():
    rng = np.random.default_rng(1)
    for _ in range(20):
        sc = rng.integers(0, 64, 8).tolist()
        mn = rng.integers(0, 64, 8).tolist()
        q = rng.integers(0, 16, 256).tolist()
        d = float(np.float16(rng.uniform(-1, 1)))
        dmin = float(np.float16(rng.uniform(-1, 1)))
        _check_block(12, pack_q4_k(d, dmin, sc, mn, q), q4_k_expected(d, dmin, sc, mn, q))


# ---------------------------------------------------------------- Q5_K

def pack_q5_k(d, dmin, sc, mn, q):
    """Encoder for one GGUF Q5_K block: Q4_K's header and scale packing
    (pack_q4_k), then 32 high-bit bytes and 128 nibble bytes; weight 64c+l
    keeps its low four bits in the low nibble of quant byte 32c+l and its
    fifth bit in bit 2c of high-bit byte l; weight 64c+32+l the high nibble
    and bit 2c+1."""
    assert len(q) == 256 and all(0 <= v < 32 for v in q)
    q4 = [v & 15 for v in q]
    head = pack_q4_k(d, dmin, sc, mn, q4)   # 16-byte header + 128 nibble bytes
    qh = [0] * 32
    for c in range(4):
        for l in range(32):
            qh[l] |= (q[64 * c + l] >> 4) << (2 * c)
            qh[l] |= (q[64 * c + 32 + l] >> 4) << (2 * c + 1)
    return bytes(head[:16]) + bytes(qh) + bytes(head[16:])


def test_q5_k_unit_scales_give_quants():
    q = [(11 * i + 5) % 32 for i in range(256)]
    blob = pack_q5_k(1.0, 0.0, [1] * 8, [0] * 8, q)
    assert oracle.block_bytes(13) == len(blob) == 176
    w = oracle.decode_f32(13, np.frombuffer(blob, np.uint8), 256)[0]
    assert w.tolist() == [float(v) for v in q]


def test_q5_k_random_blocks_and_fields():
    rng = np.random.default_rng(5)
    for it in range(24):
        sc = rng.integers(0, 64, 8).tolist()
        mn = rng.integers(0, 64, 8).tolist()
        if it < 8:                       # each field at its extremes once
            sc[it], mn[it] = 63, 63
        q = rng.integers(0, 32, 256).tolist()
        d = float(np.float16(rng.uniform(-1, 1)))
        dmin = float(np.float16(rng.uniform(-1, 1)))
        exp = [Fraction(d) * sc[i // 32] * q[i] - Fraction(dmin) * mn[i // 32] for i in range(256)]
        _check_block(13, pack_q5_k(d, dmin, sc, mn, q), exp)


# ---------------------------------------------------------------- Q6_K

def pack_q6_k(d, sc, q):
    """Encoder for one GGUF Q6_K block: 128 low-bit bytes, 64 high-bit bytes,
    16 int8 scales, fp16 d.  Half h, position l: weights 128h+l and
    128h+64+l share low-bit byte 64h+l (low and high nibble), weights
    128h+32+l and 128h+96+l share byte 64h+32+l; the four weights' top two
    bits fill high-bit byte 32h+l from bit 0 up.  Stored quants are q + 32."""
    assert len(sc) == 16 and len(q) == 256 and all(-32 <= v < 32 for v in q)
    u = [v + 32 for v in q]
    ql, qh = [0] * 128, [0] * 64
    for h in range(2):
        for l in range(32):
            a, b, c, e = (u[128 * h + l], u[128 * h + 32 + l], u[128 * h + 64 + l], u[128 * h + 96 + l])
            ql[64 * h + l] = (a & 15) | ((c & 15) << 4)
            ql[64 * h + 32 + l] = (b & 15) | ((e & 15) << 4)
            qh[32 * h + l] = (a >> 4) | ((b >> 4) << 2) | ((c >> 4) << 4) | ((e >> 4) << 6)
    return bytes(ql + qh + [s & 0xFF for s in sc] + f16(d))


def test_q6_k_unit_scales_give_quants():
    q = [(13 * i + 7) % 64 - 32 for i in range(256)]
    blob = pack_q6_k(1.0, [1] * 16, q)
    assert oracle.block_bytes(14) == len(blob) == 210
    w = oracle.decode_f32(14, np.frombuffer(blob, np.uint8), 256)[0]
    assert w.tolist() == [float(v) for v in q]


def test_q6_k_random_blocks_and_signed_scales():
    rng = np.random.default_rng(6)
    for it in range(24):
        sc = rng.integers(-128, 128, 16).tolist()
        if it < 16:
            sc[it] = -128 if it % 2 else 127
        q = rng.integers(-32, 32, 256).tolist()
        d = float(np.float16(rng.uniform(-1, 1)))
        blob = pack_q6_k(d, sc, q)
        w64 = oracle.decode_f64(14, np.frombuffer(blob, np.uint8), 256)[0]
        w32 = oracle.decode_f32(14, np.frombuffer(blob, np.uint8), 256)[0]
        for i in range(256):
            e = Fraction(d) * sc[i // 16] * q[i]
            assert Fraction(float(w64[i])) == e
            # fp32: (d * sc) is exact, the product with q rounds once
            assert w32[i] == np.float32(float(e))


# ---------------------------------------------------------------- row gather

@pytest.mark.parametrize("name", list(CODECS))
def test_get_rows_is_decode_of_the_rows(name):
    c = CODECS[name]
    qk = oracle.block_weights(c)
    k = qk * (3 if qk == 256 else 5)
    rng = np.random.Generator(np.random.PCG64(9))
    w = synth.gen_weights(c, 40, k, rng)
    ids = np.array([0, 39, 7, 7, 40, -1, 2 ** 31 - 1, 13], dtype=np.int32)
    got = oracle.get_rows(c, w, k, ids)
    dec = oracle.decode_f32(c, w, k)
    for t, i in enumerate(ids):
        if 0 <= i < 40:
            assert np.array_equal(got[t].view(np.uint32), dec[i].view(np.uint32))
        else:
            assert np.all(got[t] == 0.0)      # outside the table: an all-zero row


# ---------------------------------------------------------------- Q2_K

def pack_q2_k(d, dmin, sc, mn, q):
    """Encoder for one GGUF Q2_K block: 16 sub-blocks of 16 weights; byte j of
    the scale field holds sub-block j's scale (low nibble) and min (high
    nibble); quant byte 32h+l holds weights 128h+l, +32, +64, +96 in bit pairs
    0, 1, 2, 3; fp16 d and dmin follow the 80 bytes."""
    assert len(sc) == len(mn) == 16 and len(q) == 256
    s = [(sc[j] & 15) | ((mn[j] & 15) << 4) for j in range(16)]
    qs = [0] * 64
    for h in range(2):
        for l in range(32):
            b = 0
            for j in range(4):
                v = q[128 * h + 32 * j + l]
                assert 0 <= v < 4
                b |= v << (2 * j)
            qs[32 * h + l] = b
    return bytes(s + qs + f16(d) + f16(dmin))


def q2_k_expected(d, dmin, sc, mn, q):
    return [Fraction(d) * sc[i // 16] * q[i] - Fraction(dmin) * mn[i // 16] for i in range(256)]


def test_q2_k_unit_scale_and_min():
    q = [(3 * i + 1) % 4 for i in range(256)]
    blob = pack_q2_k(1.0, 0.0, [1] * 16, [0] * 16, q)
    assert oracle.decode_f32(10, np.frombuffer(blob, np.uint8), 256)[0].tolist() == [float(v) for v in q]
    # scale 0, min 1, dmin 1: every weight is -1 (the s = 0x10 case)
    blob = pack_q2_k(1.0, 1.0, [0] * 16, [1] * 16, q)
    assert oracle.decode_f32(10, np.frombuffer(blob, np.uint8), 256)[0].tolist() == [-1.0] * 256


def test_q2_k_random_blocks():
    rng = np.random.default_rng(2)
    for _ in range(20):
        sc = rng.integers(0, 16, 16).tolist()
        mn = rng.integers(0, 16, 16).tolist()
        q = rng.integers(0, 4, 256).tolist()
        d = float(np.float16(rng.uniform(-2, 2)))
        dmin = float(np.float16(rng.uniform(-2, 2)))
        _check_block(10, pack_q2_k(d, dmin, sc, mn, q), q2_k_expected(d, dmin, sc, mn, q))


# ---------------------------------------------------------------- TQ1_G128

def tq1_block(full, tail, scale):
    assert len(full) == 25
    return bytes(list(full) + [tail] + f16(scale))


def test_tq1_special_codes():
    fmt = {r[0]: r[1] for r in _golden_rows("tq1_format.txt")}
    mf, mt = int(fmt["max_full_code_byte"]), int(fmt["max_tail_code_byte"])
    assert (mf, mt) == (3 ** 5 - 1, 3 ** 3 - 1)
    for code, val in ((0, -1.0), (121, 0.0), (mf, 1.0)):
        for tail, tv in ((0, -1.0), (13, 0.0), (mt, 1.0)):
            w = oracle.decode_f32(1001, np.frombuffer(tq1_block([code] * 25, tail, 1.0), np.uint8), 128)[0]
            assert w[:125].tolist() == [val] * 125
            assert w[125:].tolist() == [tv] * 3


def test_tq1_digit_positions():
    # All-zero weights (121 = digits 1,1,1,1,1) except one +1 at (slot, digit).
    for slot in range(25):
        for i in range(5):
            full = [121] * 25
            full[slot] = 121 + 3 ** i
            w = oracle.decode_f32(1001, np.frombuffer(tq1_block(full, 13, 2.0), np.uint8), 128)[0]
            nz = np.flatnonzero(w)
            assert nz.tolist() == [5 * slot + i] and w[5 * slot + i] == 2.0
    for i in range(3):
        w = oracle.decode_f32(1001, np.frombuffer(tq1_block([121] * 25, 13 + 3 ** i, 2.0), np.uint8), 128)[0]
        assert np.flatnonzero(w).tolist() == [125 + i]


def test_tq1_exhaustive_codes_reconstruct_byte():
    for p in range(256):
        full = [121] * 25
        full[7] = p
        tail = p if p < 256 else 0
        w = oracle.decode_f64(1001, np.frombuffer(tq1_block(full, tail, 1.0), np.uint8), 128)[0]
        digits = [int(v) + 1 for v in w[35:40]]
        tdigits = [int(v) + 1 for v in w[125:128]]
        if p <= 242:
            assert all(t in (0, 1, 2) for t in digits)
            assert sum(t * 3 ** i for i, t in enumerate(digits)) == p
        else:  # illegal full byte: every weight decodes to zero
            assert digits == [1] * 5
        if p <= 26:
            assert sum(t * 3 ** i for i, t in enumerate(tdigits)) == p
        else:
            assert tdigits == [1] * 3


def test_tq1_scale_sign_gives_signed_zero():
    w = oracle.decode_f32(1001, np.frombuffer(tq1_block([121] * 25, 13, -0.5), np.uint8), 128)[0]
    assert np.all(w == 0) and np.all(np.signbit(w))
    w = oracle.decode_f32(1001, np.frombuffer(tq1_block([0] * 25, 0, -0.5), np.uint8), 128)[0]
    assert np.all(w == 0.5)


def test_lut23_div9_identity():
    fmt = {r[0]: r[1] for r in _golden_rows("tq1_format.txt")}
    for p in range(int(fmt["hi_div9_exact_up_to"]) + 1):
        assert (p * 57) >> 9 == p // 9


def test_tq1_illegal_scan():
    rng = np.random.default_rng(3)
    w = synth.gen_weights(1001, 4, 512, rng)
    assert oracle.tq1_first_illegal(w, 512) == -1
    w[2, 28 + 25] = 27          # tail byte of block 1 in row 2
    assert oracle.tq1_first_illegal(w, 512) == 2 * 4 + 1
    w[1, 3] = 243
    assert oracle.tq1_first_illegal(w, 512) == 4


# ---------------------------------------------------------------- fp32 decode = one rounding

@pytest.mark.parametrize("codec", [8, 10, 12, 13, 14, 1001])
def test_f32_decode_is_rounded_exact_value(codec):
    rng = np.random.default_rng(4)
    k = 512
    w = synth.gen_weights(codec, 16, k, rng)
    w64 = oracle.decode_f64(codec, w, k)
    w32 = oracle.decode_f32(codec, w, k)
    assert np.array_equal(w32.view(np.uint32), w64.astype(np.float32).view(np.uint32))


# ---------------------------------------------------------------- products

def _brute(codec, w, k, x):
    wd = oracle.decode_f64(codec, w, k)
    y = np.zeros((x.shape[0], wd.shape[0]))
    for m in range(x.shape[0]):
        for n in range(wd.shape[0]):
            s = 0.0
            for kk in range(k):
                s += float(wd[n, kk]) * float(x[m, kk])
            y[m, n] = s
    return y


@pytest.mark.parametrize("codec", [8, 10, 12, 13, 14, 1001])
@pytest.mark.parametrize("blocks", [1, 2])
def test_matmul_tiny_brute_force(codec, blocks):
    rng = np.random.default_rng(5)
    qk = synth.geometry(codec)[0]
    k = qk * blocks
    w = synth.gen_weights(codec, 5, k, rng)
    x = synth.gen_x(3, k, "f32", rng).astype(np.float64)
    y = oracle.matmul(codec, w, k, x)
    yb = _brute(codec, w, k, x)
    assert np.allclose(y, yb, rtol=1e-12, atol=1e-12)
    # library routine: numpy fp64 matmul of the decoded weights
    wd = oracle.decode_f64(codec, w, k)
    assert np.allclose(y, x @ wd.T, rtol=1e-12, atol=1e-12)


def test_matmul_unit_vectors_and_ones():
    rng = np.random.default_rng(6)
    k = 512
    w = synth.gen_weights(12, 7, k, rng)
    wd = oracle.decode_f64(12, w, k)
    eye = np.eye(k)
    y = oracle.matmul(12, w, k, eye[[0, 37, 300, 511]])
    assert np.array_equal(y, wd[:, [0, 37, 300, 511]].T)
    y1 = oracle.matmul(12, w, k, np.ones((1, k)))
    assert np.allclose(y1[0], wd.sum(axis=1), rtol=1e-13)


def test_matmul_threads_agree():
    rng = np.random.default_rng(7)
    w = synth.gen_weights(12, 37, 1024, rng)
    x = synth.gen_x(4, 1024, "bf16", rng)
    assert np.array_equal(oracle.matmul(12, w, 1024, x, threads=1),
                          oracle.matmul(12, w, 1024, x, threads=5))


def test_matmul_id_identity_routing_equals_dense():
    rng = np.random.default_rng(8)
    e, n, k, t = 3, 6, 256, 4
    w = synth.gen_weights(12, e * n, k, rng).reshape(e, n, -1)
    x = synth.gen_x(t, k, "f32", rng)
    ids = np.tile(np.arange(e, dtype=np.int32), (t, 1))
    y = oracle.matmul_id(12, w, k, x, ids)
    for s in range(e):
        assert np.array_equal(y[:, s, :], oracle.matmul(12, w[s], k, x))


def test_matmul_id_duplicates_and_bad_ids():
    rng = np.random.default_rng(9)
    e, n, k, t = 3, 5, 128, 3
    w = synth.gen_weights(1001, e * n, k, rng).reshape(e, n, -1)
    x = synth.gen_x(t, k, "f32", rng)
    ids = np.array([[1, 1], [2, -1], [3, 0]], dtype=np.int32)
    y = oracle.matmul_id(1001, w, k, x, ids)
    assert np.array_equal(y[0, 0], y[0, 1])
    assert np.array_equal(y[0, 0], oracle.matmul(1001, w[1], k, x[:1])[0])
    assert np.all(np.isnan(y[1, 1])) and np.all(np.isnan(y[2, 0]))
    assert np.array_equal(y[2, 1], oracle.matmul(1001, w[0], k, x[2:3])[0])


# ---------------------------------------------------------------- generator

def test_generator_field_ranges():
    rng = np.random.default_rng(10)
    w = synth.gen_weights(8, 64, 1024, rng).reshape(-1, 34)
    d = w[:, 0:2].copy().view("<f2").astype(np.float64)
    assert d.min() >= 2.0 ** -8 and d.max() <= 2.0 ** -4
    q = w[:, 2:].view(np.int8)
    assert q.min() >= -127 and q.max() <= 127
    w = synth.gen_weights(12, 64, 1024, rng).reshape(-1, 144)
    for off in (0, 2):
        v = w[:, off:off + 2].copy().view("<f2").astype(np.float64)
        assert v.min() >= 2.0 ** -10 and v.max() <= 2.0 ** -6
    w = synth.gen_weights(1001, 64, 1024, rng).reshape(-1, 28)
    assert w[:, :25].max() <= 242 and w[:, 25].max() <= 26
    s = w[:, 26:28].copy().view("<f2").astype(np.float64)
    assert s.min() >= 2.0 ** -6 and s.max() <= 2.0 ** -2


def test_bf16_rounding_matches_torch():
    import torch

    x = np.random.default_rng(11).standard_normal(4096).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(synth.round_to_bf16(x), ref)


def test_ids_are_distinct_and_in_range():
    ids = synth.gen_ids(32, 6, 64, np.random.default_rng(0))
    assert ids.min() >= 0 and ids.max() < 64
    assert all(len(set(r)) == 6 for r in ids.tolist())


# ---------------------------------------------------------------- fused GLU

def test_glu_activations_match_torch_fp64():
    import torch
    import torch.nn.functional as F

    g = np.concatenate([np.linspace(-30, 30, 601), [0.0, -0.5, 1.0, 1e-8, -1e-8]])
    gt = torch.from_numpy(g)
    # equal up to fp64 rounding: relative 1e-13, plus an absolute 1e-13 where
    # 1 + tanh(.) or 1 + exp(.) cancels for negative g (a few ulp of |g|)
    assert np.allclose(oracle.act_f64(g, "silu"), F.silu(gt).numpy(), rtol=1e-13, atol=1e-13)
    assert np.allclose(oracle.act_f64(g, "gelu"), F.gelu(gt, approximate="tanh").numpy(), rtol=1e-13, atol=1e-13)
    assert oracle.act_f64(np.array([0.0]), "silu")[0] == 0.0
    # large positive g: silu(g) -> g; large negative: -> 0
    assert oracle.act_f64(np.array([50.0]), "silu")[0] == 50.0
    assert abs(oracle.act_f64(np.array([-50.0]), "silu")[0]) < 1e-19


def test_glu_id_brute_force_and_bad_ids():
    import math

    rng = np.random.default_rng(11)
    e, n, k, t, top_k = 3, 4, 256, 3, 2
    wg = synth.gen_weights(12, e * n, k, rng).reshape(e, n, -1)
    wu = synth.gen_weights(12, e * n, k, rng).reshape(e, n, -1)
    x = synth.gen_x(t, k, "f32", rng).astype(np.float64)
    ids = np.array([[0, 2], [1, 1], [2, 3]], dtype=np.int32)   # a duplicate, an id outside [0, E)
    dg = oracle.decode_f64(12, wg.reshape(e * n, -1), k).reshape(e, n, k)
    du = oracle.decode_f64(12, wu.reshape(e * n, -1), k).reshape(e, n, k)
    for act in ("silu", "gelu"):
        y = oracle.glu_id(12, wg, wu, k, x, ids, act)
        for tt in range(t):
            for s in range(top_k):
                ee = ids[tt, s]
                if ee >= e:
                    assert np.all(np.isnan(y[tt, s]))
                    continue
                for j in range(n):
                    gv = sum(dg[ee, j, kk] * x[tt, kk] for kk in range(k))
                    uv = sum(du[ee, j, kk] * x[tt, kk] for kk in range(k))
                    a = gv / (1 + math.exp(-gv)) if act == "silu" else \
                        0.5 * gv * (1 + math.tanh(math.sqrt(2 / math.pi) * (gv + 0.044715 * gv ** 3)))
                    assert abs(y[tt, s, j] - a * uv) <= 1e-9 * max(1.0, abs(a * uv))


# ---------------------------------------------------------------- down projection with the mix

def test_mix_id_reduces_to_matmul_id_and_brute_force():
    rng = np.random.default_rng(12)
    e, n, k, t, top_k = 4, 6, 256, 5, 3
    w = synth.gen_weights(12, e * n, k, rng).reshape(e, n, -1)
    ids = synth.gen_ids(t, top_k, e, rng)
    scores = rng.uniform(0, 1, (t, top_k)).astype(np.float32)
    # every slot carries its token's row: the mix of matmul_id's rows
    x = synth.gen_x(t, k, "f32", rng).astype(np.float64)
    xs = np.repeat(x[:, None, :], top_k, axis=1)
    y = oracle.mix_id(12, w, k, xs, ids, scores)
    yid = oracle.matmul_id(12, w, k, x, ids)
    assert np.allclose(y, (scores[..., None].astype(np.float64) * yid).sum(axis=1), rtol=1e-12, atol=1e-12)
    # distinct slot rows: brute force
    xs = synth.gen_x(t * top_k, k, "f32", rng).astype(np.float64).reshape(t, top_k, k)
    y = oracle.mix_id(12, w, k, xs, ids, scores)
    dec = oracle.decode_f64(12, w.reshape(e * n, -1), k).reshape(e, n, k)
    for tt in range(t):
        for j in range(n):
            v = sum(float(scores[tt, s]) * sum(dec[ids[tt, s], j, q] * xs[tt, s, q] for q in range(k))
                    for s in range(top_k))
            assert abs(y[tt, j] - v) <= 1e-9 * max(1.0, abs(v))
    # one-hot scores pick a slot's product; a bad id poisons its token
    sc = np.zeros((t, top_k), np.float32)
    sc[:, 1] = 1
    y = oracle.mix_id(12, w, k, xs, ids, sc)
    for tt in range(t):
        assert np.allclose(y[tt], dec[ids[tt, 1]] @ xs[tt, 1], rtol=1e-12, atol=1e-12)
    bad = ids.copy()
    bad[2, 0] = e
    y = oracle.mix_id(12, w, k, xs, bad, scores)
    assert np.all(np.isnan(y[2])) and np.isfinite(y[[0, 1, 3, 4]]).all()
