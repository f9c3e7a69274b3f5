"""Parity of the CUDA path with the CPU oracle (needs a B200).

Small cases span several CTAs / tiles and a ragged tail; the five measured
workloads run at full size in the launch configuration the benchmark times,
compared on all outputs (or on sampled weight rows where the oracle would
take long).  Decode is compared bit for bit; products by the normwise row
error of tests/kqtest.py.
"""
import numpy as np
import pytest

import oracle
import synth
from kqtest import BF16_OUT, FP32_PATH_TOL, GEMV_TOL, TOL, row_rel_err, to_device_w, to_device_x

pytestmark = pytest.mark.gpu

CODECS = [synth.Q8_0, synth.Q2_K, synth.Q4_K, synth.Q5_K, synth.Q6_K, synth.TQ1_G128]


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# ---------------------------------------------------------------- dequantize

@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("rows,nblocks", [(1, 1), (37, 3), (300, 8)])
def test_dequantize_bit_exact(kq, codec, rows, nblocks):
    import torch

    k = synth.geometry(codec)[0] * nblocks
    w = synth.gen_weights(codec, rows, k, rng(rows + codec))
    ref = oracle.decode_f32(codec, w, k)
    got = kq.dequantize(to_device_w(w), codec, k).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    for dt in (torch.bfloat16, torch.float16):
        g = kq.dequantize(to_device_w(w), codec, k, dtype=dt).cpu()
        r = torch.from_numpy(ref).to(dt)   # round-to-nearest-even of the fp32 decode
        assert torch.equal(g.view(torch.int16), r.view(torch.int16))


def test_dequantize_illegal_tq1_bytes_and_validate(kq):
    w = synth.gen_weights(synth.TQ1_G128, 5, 384, rng(1))
    w[3, 28 + 7] = 250        # full byte of block 1, row 3
    w[4, 2 * 28 + 25] = 200   # tail byte of block 2, row 4
    ref = oracle.decode_f32(synth.TQ1_G128, w, 384)
    got = kq.dequantize(to_device_w(w), synth.TQ1_G128, 384).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert np.all(got[3, 128 + 35:128 + 40] == 0)
    assert kq.validate(to_device_w(w), synth.TQ1_G128, 384) == oracle.tq1_first_illegal(w, 384) == 3 * 3 + 1
    ok = synth.gen_weights(synth.TQ1_G128, 5, 384, rng(2))
    assert kq.validate(to_device_w(ok), synth.TQ1_G128, 384) == -1


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_dequantize_full_workload_weights(kq, name):
    wl = synth.WORKLOADS[name]
    w, _, _ = synth.make_inputs(wl)
    w = w.reshape(-1, synth.row_bytes(wl.codec, wl.k))
    ref = oracle.decode_f32(wl.codec, w, wl.k)
    got = kq.dequantize(to_device_w(w), wl.codec, wl.k).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


# ---------------------------------------------------------------- row gather

@pytest.mark.parametrize("codec", CODECS)
def test_get_rows_bit_exact(kq, codec):
    """Rows picked by id decode exactly as the oracle's fp32 decode (bf16 and
    f16 outputs: that value rounded to nearest even); ids outside the table
    give zero rows and the device error word."""
    import torch

    qk = synth.geometry(codec)[0]
    k = qk * (6 if qk == 256 else 20)
    rows = 257
    w = synth.gen_weights(codec, rows, k, rng(400 + codec))
    ids = np.array([0, 256, 13, 13, 100, 255, 1, 77, 200, 3, 5, 8], dtype=np.int32)
    wd = to_device_w(w)
    ref = oracle.get_rows(codec, w, k, ids)
    got = kq.get_rows(wd, codec, k, torch.from_numpy(ids).cuda()).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    for dt in (torch.bfloat16, torch.float16):
        g = kq.get_rows(wd, codec, k, torch.from_numpy(ids).cuda(), dtype=dt).cpu()
        assert torch.equal(g.view(torch.int16), torch.from_numpy(ref).to(dt).view(torch.int16))
    assert kq.device_status() == 0
    bad = np.array([4, -1, rows, 2 ** 31 - 1, 9, 0, 0, 0], dtype=np.int32)
    got = kq.get_rows(wd, codec, k, torch.from_numpy(bad).cuda()).cpu().numpy()
    ref = oracle.get_rows(codec, w, k, bad)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert np.all(got[1:4] == 0.0)
    assert kq.device_status() == -9    # KQ_ERR_DEVICE, then cleared
    assert kq.device_status() == 0


# ---------------------------------------------------------------- matmul

def _paths(kq):
    return {"simple": kq.PATH_SIMPLE, "gemv": kq.PATH_GEMV, "gemm": kq.PATH_GEMM}


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
@pytest.mark.parametrize("m", [1, 3, 8, 19])
def test_matmul_simple_path(kq, codec, xdt, m):
    import torch

    qk = synth.geometry(codec)[0]
    k = qk * (3 if qk == 256 else 9)
    n = 261
    r = rng(100 + m + codec)
    w = synth.gen_weights(codec, n, k, r)
    x = synth.gen_x(m, k, xdt, r)
    ref = oracle.matmul(codec, w, k, x)
    for ydt in (torch.float32, torch.bfloat16):
        y = kq.matmul(to_device_w(w), codec, to_device_x(x, xdt), out_dtype=ydt,
                      path=kq.PATH_SIMPLE).float().cpu().numpy()
        err = row_rel_err(y, ref)
        if ydt == torch.float32:
            assert err <= FP32_PATH_TOL
        else:
            assert err <= TOL[xdt] + BF16_OUT


GEMV_CASES = [
    # (n, k, m): several CTAs, ragged row counts, 1..32+ blocks per row
    (300, 256, 1), (1000, 1024, 1), (4099, 4096, 1), (777, 2048, 2), (513, 4096, 3),
    (1500, 9216, 1), (640, 8192, 4), (257, 4096, 8), (5, 512, 5), (2000, 11008 // 256 * 256, 1),
    (640, 1024, 19),   # more than eight activation rows: consecutive launches of eight
]


@pytest.mark.parametrize("n,k,m", GEMV_CASES)
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
def test_matmul_gemv_q4_k(kq, n, k, m, xdt):
    import torch

    r = rng(n + k + m)
    w = synth.gen_weights(synth.Q4_K, n, k, r)
    x = synth.gen_x(m, k, xdt, r)
    ref = oracle.matmul(synth.Q4_K, w, k, x, threads=8)
    wd, xd = to_device_w(w), to_device_x(x, xdt)
    ys = []
    for cw, ind in ((False, False), (True, False), (False, True)):
        y = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMV, const_weights=cw,
                      independent=ind).cpu().numpy()
        err = row_rel_err(y, ref)
        assert err <= GEMV_TOL, err
        ys.append(y)
    # every ordering mode computes each row the same way: identical bits
    assert all(np.array_equal(ys[0].view(np.uint32), yy.view(np.uint32)) for yy in ys[1:])
    yb = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMV, out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL[xdt] + BF16_OUT


TQ1_GEMV_CASES = [
    # table kernel (rows not a multiple of 16 bytes): one block, a ragged
    # last lane step, several steps per row, two rows per launch and a third
    (5, 128, 1), (300, 1280, 1), (777, 4096 + 128, 2),
    # split kernel (K a multiple of 512): 4 to 192 blocks a row (136 row
    # groups down to 2), rows not a multiple of the groups or the SM count,
    # ring slots reused within a CTA, one launch per activation row
    (1000, 17408, 1), (129, 8192, 3), (300, 512, 1), (2000, 5120, 2), (17, 24576, 1),
    (5120, 17408, 1), (4001, 4096, 1),
]


@pytest.mark.parametrize("n,k,m", TQ1_GEMV_CASES)
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
def test_matmul_gemv_tq1(kq, n, k, m, xdt):
    import torch

    r = rng(3 * n + k + m)
    w = synth.gen_weights(synth.TQ1_G128, n, k, r)
    # illegal code bytes decode to zero: a full byte and a tail byte
    w[0, 5] = 243
    w[n - 1, (k // 128 - 1) * 28 + 25] = 27
    x = synth.gen_x(m, k, xdt, r)
    ref = oracle.matmul(synth.TQ1_G128, w, k, x, threads=8)
    wd, xd = to_device_w(w), to_device_x(x, xdt)
    ys = []
    for cw, ind in ((False, False), (True, False), (False, True)):
        y = kq.matmul(wd, synth.TQ1_G128, xd, path=kq.PATH_GEMV, const_weights=cw,
                      independent=ind).cpu().numpy()
        assert row_rel_err(y, ref) <= GEMV_TOL
        ys.append(y)
    assert all(np.array_equal(ys[0].view(np.uint32), yy.view(np.uint32)) for yy in ys[1:])
    yb = kq.matmul(wd, synth.TQ1_G128, xd, path=kq.PATH_GEMV,
                   out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL[xdt] + BF16_OUT
    assert kq.device_status() == 0


@pytest.mark.parametrize("codec,n,k", [(synth.TQ1_G128, 300, 2048), (synth.TQ1_G128, 200, 1280),
                                       (synth.Q4_K, 300, 2048), (synth.Q4_K, 130, 4096)])
def test_matmul_gemv_nonfinite_activations(kq, codec, n, k):
    """An infinite and a NaN activation: the fixed-point kernels compute such
    a call exactly in fp32, so each output is NaN, +-inf or finite as in the
    IEEE product (the fp64 oracle), and the finite outputs stay in tolerance.
    One activation row (Q4_K: codes held in registers) and three rows; Q4_K
    also as an independent call (the shared-SM build)."""
    r = rng(41 + n)
    w = synth.gen_weights(codec, n, k, r)
    x = synth.gen_x(3, k, "f32", r)
    x[0, 7] = np.inf           # row 0: one +inf
    x[1, k - 3] = -np.inf      # row 1: one -inf and one NaN
    x[1, 11] = np.nan
    ref = oracle.matmul(codec, w, k, x, threads=8)
    assert np.isnan(ref[1]).all() and np.isinf(ref[0]).any()
    wd = to_device_w(w)

    def same_classes(y, ref):
        return (np.array_equal(np.isnan(y), np.isnan(ref)) and np.array_equal(np.isposinf(y), np.isposinf(ref))
                and np.array_equal(np.isneginf(y), np.isneginf(ref)))

    for indep in ((False, True) if codec == synth.Q4_K else (False,)):
        y = kq.matmul(wd, codec, to_device_x(x, "f32"), path=kq.PATH_GEMV, independent=indep).cpu().numpy()
        assert same_classes(y, ref)
        fin = np.isfinite(ref)
        assert row_rel_err(y[2:], ref[2:]) <= GEMV_TOL      # the finite row
        assert np.allclose(y[fin], ref[fin], rtol=1e-3, atol=1e-3 * np.abs(ref[2]).max())
        y1 = kq.matmul(wd, codec, to_device_x(x[:1], "f32"), path=kq.PATH_GEMV, independent=indep).cpu().numpy()
        assert same_classes(y1, ref[:1])
        assert np.allclose(y1[np.isfinite(ref[:1])], ref[:1][np.isfinite(ref[:1])], rtol=1e-3,
                           atol=1e-3 * np.abs(ref[2]).max())
    assert kq.device_status() == 0


@pytest.mark.parametrize("codec,n,path_name,tol", [(synth.Q4_K, 4096, "PATH_GEMV", GEMV_TOL),
                                                   (synth.Q8_0, 1024, "PATH_SIMPLE", FP32_PATH_TOL)])
def test_matmul_independent_calls_back_to_back(kq, codec, n, path_name, tol):
    """Many independent calls queued on one stream (they run side by side),
    then an ordinary call, queued right behind them, that reads the first
    call's output as its activations: every result must be the one computed
    alone, and the ordinary call must see the finished output (the bandwidth
    kernel, and the plain kernel that serves Q8_0)."""
    import torch

    path = getattr(kq, path_name)
    r = rng(23)
    k = n
    ws = [synth.gen_weights(codec, n, k, r) for _ in range(3)]
    x = synth.gen_x(1, k, "bf16", r)
    wds = [to_device_w(w) for w in ws]
    xd = to_device_x(x, "bf16")
    alone = [kq.matmul(wd, codec, xd, path=path).cpu().numpy() for wd in wds]
    outs = [torch.full((1, n), float("nan"), device="cuda") for _ in range(24)]
    y2 = torch.empty((1, n), device="cuda")
    torch.cuda.synchronize()
    for i, o in enumerate(outs):
        kq.matmul(wds[i % 3], codec, xd, out=o, path=path, independent=True)
    kq.matmul(wds[1], codec, outs[0], out=y2, path=path)   # fp32 x = outs[0]
    for i, o in enumerate(outs):
        assert np.array_equal(o.cpu().numpy().view(np.uint32), alone[i % 3].view(np.uint32))
    ref2 = oracle.matmul(codec, ws[1], k, alone[0].astype(np.float64), threads=8)
    assert row_rel_err(y2.cpu().numpy(), ref2) <= tol
    assert kq.device_status() == 0


def test_independent_flag_on_other_paths_keeps_stream_order(kq):
    """The flag lets the plain kernel overlap the preceding kernel and leaves
    the tensor-core kernels in stream order; both give their usual result."""
    import torch

    r = rng(31)
    n, k, m = 300, 1024, 20
    w = synth.gen_weights(synth.Q4_K, n, k, r)
    x = synth.gen_x(m, k, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    ref = oracle.matmul(synth.Q4_K, w, k, x, threads=8)
    for path in (kq.PATH_SIMPLE, kq.PATH_GEMM):
        a = kq.matmul(wd, synth.Q4_K, xd, path=path).cpu().numpy()
        b = kq.matmul(wd, synth.Q4_K, xd, path=path, independent=True).cpu().numpy()
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
        assert row_rel_err(b, ref) <= TOL["bf16"]
    assert kq.device_status() == 0


def test_tq1_auto_beyond_eight_rows_uses_the_plain_kernel(kq):
    r = rng(32)
    n, k, m = 100, 1280, 11
    w = synth.gen_weights(synth.TQ1_G128, n, k, r)
    x = synth.gen_x(m, k, "f32", r)
    ref = oracle.matmul(synth.TQ1_G128, w, k, x, threads=8)
    wd, xd = to_device_w(w), to_device_x(x, "f32")
    y = kq.matmul(wd, synth.TQ1_G128, xd).cpu().numpy()
    ys = kq.matmul(wd, synth.TQ1_G128, xd, path=kq.PATH_SIMPLE).cpu().numpy()
    assert np.array_equal(y.view(np.uint32), ys.view(np.uint32))   # the plain kernel served it
    assert row_rel_err(y, ref) <= FP32_PATH_TOL
    yg = kq.matmul(wd, synth.TQ1_G128, xd, path=kq.PATH_GEMV).cpu().numpy()   # six launches of two rows
    assert row_rel_err(yg, ref) <= GEMV_TOL
    assert kq.device_status() == 0


def test_matmul_gemv_deterministic(kq):
    r = rng(7)
    w = synth.gen_weights(synth.Q4_K, 4096, 4096, r)
    x = synth.gen_x(1, 4096, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    a = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMV).cpu().numpy()
    b = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMV).cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_matmul_unit_vector_selects_column(kq):
    # x = e_j  =>  y = column j of the decoded weights (exactly, in fp32).
    k, n = 1024, 333
    w = synth.gen_weights(synth.Q4_K, n, k, rng(8))
    dec = oracle.decode_f32(synth.Q4_K, w, k)
    x = np.zeros((2, k), np.float32)
    x[0, 5] = 1.0
    x[1, 1000] = 1.0
    for path in (kq.PATH_SIMPLE, kq.PATH_GEMV):
        y = kq.matmul(to_device_w(w), synth.Q4_K, to_device_x(x, "f32"), path=path).cpu().numpy()
        # one nonzero activation: both paths are exact up to fp32 rounding
        np.testing.assert_allclose(y[0], dec[:, 5], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(y[1], dec[:, 1000], rtol=1e-5, atol=1e-6)


GEMM_CASES = [
    # (n, k, m): one tile, ragged rows / tokens, several waves of tiles
    (128, 256, 16), (300, 512, 19), (261, 768, 33), (1000, 1024, 64), (777, 2048, 100),
    (4096, 4096, 128), (2000, 4096, 300), (2752, 4096, 512), (640, 8192, 1024),
]


def _bf16_weight_reference(w, k, x, codec=synth.Q4_K):
    """x @ bf16(decode_f32(w))^T in fp64: what the tensor-core path computes up
    to fp32 accumulation (weights rounded to nearest-even bf16)."""
    import torch

    dec = oracle.decode_f32(codec, w, k)
    wb = torch.from_numpy(dec).to(torch.bfloat16).to(torch.float64).numpy()
    return x.astype(np.float64) @ wb.T


@pytest.mark.parametrize("n,k,m", GEMM_CASES)
def test_matmul_gemm_q4_k(kq, n, k, m):
    import torch

    r = rng(1000 + n + k + m)
    w = synth.gen_weights(synth.Q4_K, n, k, r)
    x = synth.gen_x(m, k, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    y = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMM).cpu().numpy()
    ref = oracle.matmul(synth.Q4_K, w, k, x, threads=8)
    assert row_rel_err(y, ref) <= TOL["bf16"]
    # tight: equal to the bf16-rounded-weight product up to fp32 accumulation
    assert row_rel_err(y, _bf16_weight_reference(w, k, x)) <= FP32_PATH_TOL
    yb = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMM, out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL["bf16"] + BF16_OUT
    assert kq.device_status() == 0


TQ1_GEMM_CASES = [
    # one tile and one raw unit; ragged weight rows and tokens with narrow
    # token tiles (two 64-K atoms a stage); tokens past one tile; wide tiles
    # (one atom a stage) over several tiles each way; the long rows of the
    # measured TQ1 shape (34 raw units a tile, the raw ring lapped)
    (128, 512, 5), (300, 1024, 37), (129, 2048, 64), (1000, 4096, 300), (640, 17408, 24),
]


@pytest.mark.parametrize("n,k,m", TQ1_GEMM_CASES)
def test_matmul_gemm_tq1(kq, n, k, m):
    """TQ1_G128 on the tensor cores: the weights enter the MMA as
    bf16(scale) * (t - 1), the round-to-nearest-even bf16 of the decoded
    weight, so the product equals the bf16-weight product up to fp32
    accumulation; illegal code bytes (a full byte above 242, a tail byte
    above 26) decode to zeros as everywhere else."""
    import torch

    r = rng(2000 + n + k + m)
    w = synth.gen_weights(synth.TQ1_G128, n, k, r)
    w[0, 5] = 243
    w[n - 1, (k // 128 - 1) * 28 + 25] = 27
    w[n // 2, 28 + 12] = 255    # the byte shared by both 64-weight halves of a block
    x = synth.gen_x(m, k, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    y = kq.matmul(wd, synth.TQ1_G128, xd, path=kq.PATH_GEMM).cpu().numpy()
    ref = oracle.matmul(synth.TQ1_G128, w, k, x, threads=8)
    assert row_rel_err(y, ref) <= TOL["bf16"]
    assert row_rel_err(y, _bf16_weight_reference(w, k, x, synth.TQ1_G128)) <= FP32_PATH_TOL
    yb = kq.matmul(wd, synth.TQ1_G128, xd, path=kq.PATH_GEMM,
                   out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL["bf16"] + BF16_OUT
    assert kq.device_status() == 0


def test_matmul_gemm_tq1_decodes_every_byte_exactly(kq):
    """Every byte value at every code position (full bytes 0..24 and the tail
    byte 25 of each block, legal or not) under scales of both signs: with the
    identity as activations each output is one decoded weight, which must be
    the round-to-nearest-even bf16 of the oracle's decode."""
    import torch

    n, k = 128, 512
    r = rng(43)
    w = np.zeros((n, k // 128 * 28), dtype=np.uint8)
    for row in range(n):
        for b in range(k // 128):
            pos = np.arange(26)
            w[row, 28 * b + pos] = (pos * 37 + row * 2 + b * 128 + row // 64) % 256
            sc = np.float16(r.uniform(0.01, 2.0) * (-1.0 if (row + b) % 3 == 0 else 1.0))
            w[row, 28 * b + 26: 28 * b + 28] = np.frombuffer(sc.tobytes(), dtype=np.uint8)
    # every (value, position) pair occurs: 256 values, 26 positions, 512 blocks
    seen = {(int(w[i, 28 * b + j]), j) for i in range(n) for b in range(k // 128) for j in range(26)}
    assert len(seen) == 256 * 26
    x = np.eye(k, dtype=np.float32)
    y = kq.matmul(to_device_w(w), synth.TQ1_G128, to_device_x(x, "bf16"), path=kq.PATH_GEMM).cpu().numpy()
    dec = torch.from_numpy(oracle.decode_f32(synth.TQ1_G128, w, k)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(y, dec.T)   # -0 and +0 compare equal
    assert kq.device_status() == 0


Q8_0_GEMM_CASES = [
    # one tile and one raw unit (eight blocks); ragged rows and tokens with
    # narrow token tiles; wide tiles over several tiles each way; long rows
    (128, 256, 5), (300, 1024, 37), (1000, 4096, 300), (129, 8192, 64),
]


@pytest.mark.parametrize("n,k,m", Q8_0_GEMM_CASES)
def test_matmul_gemm_q8_0(kq, n, k, m):
    """Q8_0 on the tensor cores: each weight enters the MMA as the
    round-to-nearest-even bf16 of d * q, so the product equals the
    bf16-weight product up to fp32 accumulation."""
    import torch

    r = rng(3000 + n + k + m)
    w = synth.gen_weights(synth.Q8_0, n, k, r)
    x = synth.gen_x(m, k, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    y = kq.matmul(wd, synth.Q8_0, xd, path=kq.PATH_GEMM).cpu().numpy()
    ref = oracle.matmul(synth.Q8_0, w, k, x, threads=8)
    assert row_rel_err(y, ref) <= TOL["bf16"]
    assert row_rel_err(y, _bf16_weight_reference(w, k, x, synth.Q8_0)) <= FP32_PATH_TOL
    yb = kq.matmul(wd, synth.Q8_0, xd, path=kq.PATH_GEMM, out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL["bf16"] + BF16_OUT
    assert kq.device_status() == 0


def test_matmul_gemm_q8_0_decodes_every_code_exactly(kq):
    """Every int8 code at every position of the eight-block raw unit, under
    scales of both signs (normal and subnormal fp16): with the identity as
    activations each output is one decoded weight, which must be the
    round-to-nearest-even bf16 of the oracle's decode."""
    import torch

    n, k = 256, 256
    r = rng(47)
    w = np.zeros((n, k // 32 * 34), dtype=np.uint8)
    scales = [0.5, -0.25, 1.0e-3, -3.0e-2, 6.0e-8, -1.5, 7.0, 2.0 ** -14]
    for row in range(n):
        for b in range(k // 32):
            sc = np.float16(scales[(row + b) % len(scales)] * (1.0 + (row % 7) / 16.0))
            w[row, 34 * b: 34 * b + 2] = np.frombuffer(sc.tobytes(), dtype=np.uint8)
            w[row, 34 * b + 2: 34 * b + 34] = (np.arange(32) * 8 + row + 3 * b) % 256
    seen = {(int(w[i, 34 * b + 2 + j]), 32 * b + j) for i in range(n) for b in range(k // 32) for j in range(32)}
    assert len(seen) == 256 * k
    x = np.eye(k, dtype=np.float32)
    y = kq.matmul(to_device_w(w), synth.Q8_0, to_device_x(x, "bf16"), path=kq.PATH_GEMM).cpu().numpy()
    dec = torch.from_numpy(oracle.decode_f32(synth.Q8_0, w, k)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(y, dec.T)
    assert kq.device_status() == 0


Q2_K_GEMM_CASES = [
    # one tile and one raw unit (four super-blocks); ragged rows and tokens;
    # wide tiles over several tiles each way; long rows
    (128, 1024, 5), (300, 2048, 37), (1000, 4096, 300), (129, 8192, 64),
]


@pytest.mark.parametrize("n,k,m", Q2_K_GEMM_CASES)
def test_matmul_gemm_q2_k(kq, n, k, m):
    """Q2_K on the tensor cores: the bf16 rounding of d*sc*q - dmin*m per
    weight, so the product equals the bf16-weight product up to fp32
    accumulation."""
    import torch

    r = rng(4000 + n + k + m)
    w = synth.gen_weights(synth.Q2_K, n, k, r)
    x = synth.gen_x(m, k, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    y = kq.matmul(wd, synth.Q2_K, xd, path=kq.PATH_GEMM).cpu().numpy()
    ref = oracle.matmul(synth.Q2_K, w, k, x, threads=8)
    assert row_rel_err(y, ref) <= TOL["bf16"]
    assert row_rel_err(y, _bf16_weight_reference(w, k, x, synth.Q2_K)) <= FP32_PATH_TOL
    yb = kq.matmul(wd, synth.Q2_K, xd, path=kq.PATH_GEMM, out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL["bf16"] + BF16_OUT
    assert kq.device_status() == 0


def test_matmul_gemm_q2_k_decodes_every_weight_exactly(kq):
    """Every scale/min byte at every sub-block position and every 2-bit code
    at every position of the four-super-block raw unit, under d and dmin of
    both signs: with the identity as activations each output is one decoded
    weight, which must be the round-to-nearest-even bf16 of the oracle's
    decode."""
    import torch

    n, k = 256, 1024
    r = rng(53)
    w = r.integers(0, 256, size=(n, k // 256 * 84), dtype=np.uint8)
    ds = [0.25, -0.5, 1.0e-3, -2.0e-2, 6.0e-8, 3.0]
    for row in range(n):
        for b in range(k // 256):
            o = 84 * b
            w[row, o: o + 16] = (np.arange(16) * 16 + row + 5 * b) % 256   # every scale/min byte per position
            dd = np.array([ds[(row + b) % len(ds)], -ds[(row + 2 * b + 1) % len(ds)]], dtype=np.float16)
            w[row, o + 80: o + 84] = np.frombuffer(dd.tobytes(), dtype=np.uint8)
    seen = {(int(w[i, 84 * b + j]), j) for i in range(n) for b in range(k // 256) for j in range(16)}
    assert len(seen) == 256 * 16
    x = np.eye(k, dtype=np.float32)
    y = kq.matmul(to_device_w(w), synth.Q2_K, to_device_x(x, "bf16"), path=kq.PATH_GEMM).cpu().numpy()
    dec = torch.from_numpy(oracle.decode_f32(synth.Q2_K, w, k)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(y, dec.T)
    assert kq.device_status() == 0


@pytest.mark.parametrize("n,k,m", [(128, 256, 5), (300, 1024, 37), (1000, 4096, 300), (129, 8192, 64)])
def test_matmul_gemm_q5_k(kq, n, k, m):
    """Q5_K on the tensor cores: the bf16 rounding of d*sc*q - dmin*m per
    weight (q the five-bit code), so the product equals the bf16-weight
    product up to fp32 accumulation."""
    import torch

    r = rng(5000 + n + k + m)
    w = synth.gen_weights(synth.Q5_K, n, k, r)
    x = synth.gen_x(m, k, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    y = kq.matmul(wd, synth.Q5_K, xd, path=kq.PATH_GEMM).cpu().numpy()
    ref = oracle.matmul(synth.Q5_K, w, k, x, threads=8)
    assert row_rel_err(y, ref) <= TOL["bf16"]
    assert row_rel_err(y, _bf16_weight_reference(w, k, x, synth.Q5_K)) <= FP32_PATH_TOL
    yb = kq.matmul(wd, synth.Q5_K, xd, path=kq.PATH_GEMM, out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL["bf16"] + BF16_OUT
    assert kq.device_status() == 0


def test_matmul_gemm_q5_k_decodes_every_code_exactly(kq):
    """Every five-bit code (four low bits from qs, the fifth from qh) at every
    position of a super-block, random packed scales and mins, d and dmin of
    both signs: with the identity as activations each output is one decoded
    weight, which must be the round-to-nearest-even bf16 of the oracle's
    decode."""
    import torch

    n, k = 256, 256
    r = rng(59)
    w = r.integers(0, 256, size=(n, 176), dtype=np.uint8)
    ds = [0.25, -0.5, 1.0e-3, -2.0e-2, 6.0e-8, 3.0]
    codes = np.zeros((n, 256), dtype=np.int64)
    for row in range(n):
        dd = np.array([ds[row % len(ds)], -ds[(row // 3) % len(ds)]], dtype=np.float16)
        w[row, 0:4] = np.frombuffer(dd.tobytes(), dtype=np.uint8)
        for c in range(4):
            for l in range(32):
                w[row, 48 + 32 * c + l] = (row + 7 * l + 3 * c) % 256
        # fifth bits: low-nibble codes (even bits) follow row // 16, the
        # high-nibble ones (odd bits) row % 2, so every (q4, bit) pair occurs
        w[row, 16:48] = ((row >> 4) & 1) * 0x55 | (row & 1) * 0xAA
        for c in range(4):
            for h in range(2):
                for l in range(32):
                    q4 = (int(w[row, 48 + 32 * c + l]) >> (4 * h)) & 15
                    hb = (int(w[row, 16 + l]) >> (2 * c + h)) & 1
                    codes[row, 64 * c + 32 * h + l] = q4 + 16 * hb
    seen = {(int(codes[i, j]), j) for i in range(n) for j in range(256)}
    assert len(seen) == 32 * 256
    x = np.eye(k, dtype=np.float32)
    y = kq.matmul(to_device_w(w), synth.Q5_K, to_device_x(x, "bf16"), path=kq.PATH_GEMM).cpu().numpy()
    dec = torch.from_numpy(oracle.decode_f32(synth.Q5_K, w, k)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(y, dec.T)
    assert kq.device_status() == 0


@pytest.mark.parametrize("codec,k", [(synth.Q8_0, 1408), (synth.Q2_K, 512), (synth.Q5_K, 256 * 3)])
def test_matmul_gemm_shapes_it_cannot_take(kq, codec, k):
    """K that the tensor-core kernel's raw units do not tile (Q8_0: 44
    blocks, Q2_K: two super-blocks) is refused on the explicit path and
    served by the plain kernel on the automatic one; Q5_K at K = 768 is
    taken (one super-block a unit)."""
    import torch

    r = rng(61 + k + codec)
    n, m = 200, 24
    w = synth.gen_weights(codec, n, k, r)
    x = synth.gen_x(m, k, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    ref = oracle.matmul(codec, w, k, x, threads=8)
    y = kq.matmul(wd, codec, xd).cpu().numpy()
    if codec == synth.Q5_K:
        g = kq.matmul(wd, codec, xd, path=kq.PATH_GEMM).cpu().numpy()
        assert np.array_equal(y.view(np.uint32), g.view(np.uint32))
        assert row_rel_err(y, ref) <= TOL["bf16"]
    else:
        with pytest.raises(kq.KQError):
            kq.matmul(wd, codec, xd, path=kq.PATH_GEMM)
        ys = kq.matmul(wd, codec, xd, path=kq.PATH_SIMPLE).cpu().numpy()
        assert np.array_equal(y.view(np.uint32), ys.view(np.uint32))
        assert row_rel_err(y, ref) <= FP32_PATH_TOL
    assert kq.device_status() == 0


def test_matmul_tq1_auto_prefill_uses_the_tensor_cores(kq):
    r = rng(41)
    n, k, m = 384, 2048, 40
    w = synth.gen_weights(synth.TQ1_G128, n, k, r)
    x = synth.gen_x(m, k, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    a = kq.matmul(wd, synth.TQ1_G128, xd).cpu().numpy()
    g = kq.matmul(wd, synth.TQ1_G128, xd, path=kq.PATH_GEMM).cpu().numpy()
    assert np.array_equal(a.view(np.uint32), g.view(np.uint32))
    assert row_rel_err(a, oracle.matmul(synth.TQ1_G128, w, k, x, threads=8)) <= TOL["bf16"]
    # K not a multiple of 512: the plain kernel
    w2 = synth.gen_weights(synth.TQ1_G128, n, 1280, r)
    x2 = synth.gen_x(m, 1280, "bf16", r)
    with pytest.raises(kq.KQError):
        kq.matmul(to_device_w(w2), synth.TQ1_G128, to_device_x(x2, "bf16"), path=kq.PATH_GEMM)
    y2 = kq.matmul(to_device_w(w2), synth.TQ1_G128, to_device_x(x2, "bf16")).cpu().numpy()
    assert row_rel_err(y2, oracle.matmul(synth.TQ1_G128, w2, 1280, x2, threads=8)) <= TOL["bf16"]
    assert kq.device_status() == 0


def test_matmul_gemm_deterministic(kq):
    r = rng(17)
    w = synth.gen_weights(synth.Q4_K, 1500, 4096, r)
    x = synth.gen_x(200, 4096, "bf16", r)
    wd, xd = to_device_w(w), to_device_x(x, "bf16")
    a = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMM).cpu().numpy()
    b = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMM).cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


# ---------------------------------------------------------------- workloads at full size

def _workload_check(kq, name, sample_rows=None):
    import torch

    wl = synth.WORKLOADS[name]
    w, x, ids = synth.make_inputs(wl)
    if wl.kind == "moe":
        ydt = torch.float32 if wl.y_dtype == "f32" else torch.bfloat16
        y = kq.matmul_id(to_device_w(w), wl.codec, to_device_x(x, wl.x_dtype),
                         torch.from_numpy(ids).cuda(), out_dtype=ydt).float().cpu().numpy()
        ref = oracle.matmul_id(wl.codec, w, wl.k, x, ids)
        return row_rel_err(y, ref)
    ydt = torch.float32 if wl.y_dtype == "f32" else torch.bfloat16
    y = kq.matmul(to_device_w(w), wl.codec, to_device_x(x, wl.x_dtype), out_dtype=ydt,
                  const_weights=True).float().cpu().numpy()
    if sample_rows is None:
        ref = oracle.matmul(wl.codec, w, wl.k, x, threads=8)
        return row_rel_err(y, ref)
    rows = np.unique(np.concatenate([sample_rows, [0, wl.n - 1]]))
    ref = oracle.matmul(wl.codec, w[rows], wl.k, x, threads=8)   # [m, len(rows)]
    return row_rel_err(y[:, rows], ref)


@pytest.mark.parametrize("name", ["q8_0_gemv_256x1024", "q4_k_gemv_4096x4096",
                                  "tq1_g128_gemv_5120x17408", "moe_q4_k_e64_1408x2048_t32_top6"])
def test_workload_full_size(kq, name):
    wl = synth.WORKLOADS[name]
    err = _workload_check(kq, name)
    assert err <= TOL[wl.x_dtype], err


@pytest.mark.parametrize("name", ["q4_k_gemm_512x11008x4096", "tq1_g128_gemm_512x5120x17408"])
def test_workload_prefill_gemm_sampled_rows(kq, name):
    wl = synth.WORKLOADS[name]
    # rows at tile boundaries plus a random sample
    rows = np.concatenate([np.arange(0, wl.n, 997), [127, 128, 255, 256, wl.n - 1 - 128],
                           rng(3).integers(0, wl.n, 40)])
    err = _workload_check(kq, wl.name, sample_rows=rows)
    assert err <= TOL[wl.x_dtype], err


# ---------------------------------------------------------------- expert-indexed

def _stable_group(ids, e):
    flat = ids.reshape(-1)
    valid = (flat >= 0) & (flat < e)
    counts = np.bincount(flat[valid], minlength=e)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    order = np.argsort(np.where(valid, flat, e), kind="stable")[: valid.sum()]
    return counts, offsets, order


@pytest.mark.parametrize("t,top_k,e", [(32, 6, 64), (7, 3, 5), (100, 8, 16), (1, 1, 1), (300, 2, 40)])
def test_moe_group_exact(kq, t, top_k, e):
    import torch

    ids = synth.gen_ids(t, top_k, e, rng(t))
    counts, offsets, perm = kq.moe_group(torch.from_numpy(ids).cuda(), e)
    c, o, p = _stable_group(ids, e)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offsets.cpu().numpy(), o)
    assert np.array_equal(perm.cpu().numpy(), p)
    assert kq.device_status() == 0


@pytest.mark.parametrize("codec", CODECS)
@pytest.mark.parametrize("path", ["simple", "auto"])
def test_matmul_id_small(kq, codec, path):
    import torch

    qk = synth.geometry(codec)[0]
    k = qk * (2 if qk == 256 else 8)
    e, n, t, top_k = 5, 70, 7, 3
    r = rng(codec)
    w = synth.gen_weights(codec, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, "bf16", r)
    ids = synth.gen_ids(t, top_k, e, r)
    ids[2, 1] = ids[2, 0]            # duplicate ids in a token are legal
    ref = oracle.matmul_id(codec, w, k, x, ids)
    p = {"simple": kq.PATH_SIMPLE, "auto": kq.PATH_AUTO}[path]
    y = kq.matmul_id(to_device_w(w), codec, to_device_x(x, "bf16"), torch.from_numpy(ids).cuda(),
                     path=p).cpu().numpy()
    if path == "auto" and codec == synth.Q4_K:
        # bf16 Q4_K: the dispatch picks one of the grouped kernels by pairs
        # per expert; the result is one of theirs, bit for bit, within the
        # bf16 contract
        assert row_rel_err(y, ref) <= TOL["bf16"]
        outs = [kq.matmul_id(to_device_w(w), codec, to_device_x(x, "bf16"), torch.from_numpy(ids).cuda(),
                             path=pp).cpu().numpy() for pp in (kq.PATH_GEMV, kq.PATH_GEMM, kq.PATH_GEMV_TC)]
        assert any(np.array_equal(y.view(np.uint32), o.view(np.uint32)) for o in outs)
    elif path == "auto" and _grouped_gemm_takes(codec, k):
        # bf16 activations: the grouped tensor-core GEMM, bit for bit
        assert row_rel_err(y, ref) <= TOL["bf16"]
        g = kq.matmul_id(to_device_w(w), codec, to_device_x(x, "bf16"), torch.from_numpy(ids).cuda(),
                         path=kq.PATH_GEMM).cpu().numpy()
        assert np.array_equal(y.view(np.uint32), g.view(np.uint32))
    else:
        assert row_rel_err(y, ref) <= FP32_PATH_TOL
    assert kq.device_status() == 0


def _grouped_gemm_takes(codec, k):
    """Whether the grouped tensor-core GEMM serves bf16 activations of this
    codec and K (the automatic path's choice for the codecs without a
    grouped bandwidth kernel)."""
    return (codec in (synth.Q8_0, synth.Q5_K) and k % 256 == 0) or (codec == synth.Q2_K and k % 1024 == 0)


@pytest.mark.parametrize("t,top_k,e,n,k", [
    (32, 6, 64, 1408, 2048),   # the MoE workload's shape
    (20, 4, 5, 300, 1024),     # ~16 pairs per expert: four rounds of four
    (24, 2, 3, 5000, 512),     # half the lanes of a group idle, many tiles, ring slots reused
    (3, 2, 40, 257, 4096),     # most experts hit by nobody; four warps a row group
    (7, 3, 4, 129, 512),
    (11, 3, 6, 333, 1280),     # 40 sub-blocks a row (a group of two warps, 24 lanes idle), ragged tiles
    (64, 8, 16, 96, 2048),     # 32 pairs per expert: eight rounds
])
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
def test_matmul_id_grouped_gemv(kq, t, top_k, e, n, k, xdt):
    import torch

    r = rng(t + e + n)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, xdt, r)
    ids = synth.gen_ids(t, top_k, e, r)
    ref = oracle.matmul_id(synth.Q4_K, w, k, x, ids)
    wd, xd, idd = to_device_w(w), to_device_x(x, xdt), torch.from_numpy(ids).cuda()
    y = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMV).cpu().numpy()
    assert row_rel_err(y, ref) <= GEMV_TOL
    y2 = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMV).cpu().numpy()
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))   # deterministic
    yb = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMV,
                      out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL[xdt] + BF16_OUT
    assert kq.device_status() == 0


def test_matmul_id_grouped_gemv_skewed_and_nonfinite(kq):
    """One expert takes most pairs (several rounds), experts with a single
    pair; then an infinite and a NaN activation: the rounds that stage them
    run exactly in fp32, so every output is NaN, +-inf or finite as in the
    IEEE product."""
    import torch

    t, top_k, e, n, k = 40, 2, 6, 200, 1024
    r = rng(77)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, "f32", r)
    ids = synth.gen_ids(t, top_k, e, r)
    ids[:, 0] = np.where(np.arange(t) % 13 == 0, 5, 1)
    wd, idd = to_device_w(w), torch.from_numpy(ids).cuda()
    ref = oracle.matmul_id(synth.Q4_K, w, k, x, ids)
    y = kq.matmul_id(wd, synth.Q4_K, to_device_x(x, "f32"), idd, path=kq.PATH_GEMV).cpu().numpy()
    assert row_rel_err(y, ref) <= GEMV_TOL
    x[3, 17] = np.inf
    x[9, 1000] = np.nan
    x[9, 5] = -np.inf
    ref = oracle.matmul_id(synth.Q4_K, w, k, x, ids)
    y = kq.matmul_id(wd, synth.Q4_K, to_device_x(x, "f32"), idd, path=kq.PATH_GEMV).cpu().numpy()
    assert np.array_equal(np.isnan(y), np.isnan(ref))
    assert np.array_equal(np.isposinf(y), np.isposinf(ref))
    assert np.array_equal(np.isneginf(y), np.isneginf(ref))
    fin = np.isfinite(ref).all(axis=2)
    assert row_rel_err(y[fin], ref[fin]) <= GEMV_TOL
    assert kq.device_status() == 0


@pytest.mark.parametrize("codec,t,top_k,e,n,k", [
    (synth.Q4_K, 32, 6, 64, 1408, 2048),   # the MoE workload's shape, gate and up stacks
    (synth.Q4_K, 20, 4, 5, 300, 1024),     # several rounds per expert
    (synth.Q4_K, 7, 3, 4, 129, 1280),      # ragged tiles, a group with idle lanes
    (synth.Q8_0, 9, 2, 3, 70, 256),        # Q8_0, Q2_K, Q5_K: two grouped GEMMs with bf16
    (synth.Q2_K, 40, 4, 6, 300, 2048),     # activations (up, then gate combined in the
    (synth.Q5_K, 9, 2, 3, 130, 512),       # epilogue), the plain fused kernel with fp32
    (synth.Q8_0, 9, 2, 3, 70, 1408),       # K the GEMM does not tile: the plain kernel
    (synth.Q6_K, 9, 2, 3, 70, 512),
    (synth.TQ1_G128, 9, 2, 3, 70, 384),
])
@pytest.mark.parametrize("act", ["silu", "gelu"])
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
def test_matmul_id_glu(kq, codec, t, top_k, e, n, k, act, xdt):
    """Fused MoE GLU: act(gate) * up per routed pair against the fp64
    oracle, with an out-of-range id giving a NaN row."""
    import torch

    r = rng(t + n + k + codec)
    wg = synth.gen_weights(codec, e * n, k, r).reshape(e, n, -1)
    wu = synth.gen_weights(codec, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, xdt, r)
    ids = synth.gen_ids(t, top_k, e, r)
    ids[t // 2, 0] = e                        # outside the stack: a NaN row
    ref = oracle.glu_id(codec, wg, wu, k, x, ids, act)
    y = kq.matmul_id_glu(to_device_w(wg), to_device_w(wu), codec, to_device_x(x, xdt),
                         torch.from_numpy(ids).cuda(), act=act).cpu().numpy()
    assert np.all(np.isnan(y[t // 2, 0]))
    good = ~np.isnan(ref[..., 0])
    # the product of two results each within its path's bound
    if xdt == "bf16" and _grouped_gemm_takes(codec, k):
        tol = 2 * TOL["bf16"]   # bf16 weights on the tensor cores
    else:
        tol = 2 * (GEMV_TOL if codec == synth.Q4_K else FP32_PATH_TOL)
    assert row_rel_err(y[good], ref[good]) <= tol
    assert kq.device_status() == -9
    assert kq.device_status() == 0
    if xdt == "bf16" and _grouped_gemm_takes(codec, k):
        # tight: act(gate) * up from the two grouped GEMM products themselves
        # (each checked against the oracle elsewhere), so a swapped or
        # misplaced operand of the combine cannot hide in the bf16 bound
        xd, idd = to_device_x(x, xdt), torch.from_numpy(ids).cuda()
        g = kq.matmul_id(to_device_w(wg), codec, xd, idd, path=kq.PATH_GEMM).cpu().numpy().astype(np.float64)
        u = kq.matmul_id(to_device_w(wu), codec, xd, idd, path=kq.PATH_GEMM).cpu().numpy().astype(np.float64)
        kq.device_status()   # the invalid id flagged again
        if act == "silu":
            a = g / (1.0 + np.exp(-g))
        else:
            a = 0.5 * g * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (g + 0.044715 * g ** 3)))
        assert row_rel_err(y[good], (a * u)[good]) <= 1e-5


def _pair_refs(codec, w, k, xs, ids):
    """Per-pair fp64 oracle products [T, top_k, n] of a slotted input."""
    t, top_k, _ = xs.shape
    flat = oracle.matmul_id(codec, w, k, xs.reshape(t * top_k, k), ids.reshape(-1, 1))
    return flat.reshape(t, top_k, -1)


def _mix_err_ok(y, ref, pair_ref, scores, tol):
    """|y - ref| per token within tol times the mix of its slots' row maxima:
    each slot's product is within tol of its row maximum and the mix weights
    it by |score|."""
    bound = tol * (np.abs(scores.astype(np.float64)) * np.abs(pair_ref).max(axis=2)).sum(axis=1)
    err = np.abs(np.asarray(y, np.float64) - ref).max(axis=1)
    return bool(np.all(err <= bound + 1e-30)), float((err / np.maximum(bound, 1e-30)).max())


@pytest.mark.parametrize("codec,path,xdt,t,top_k,e,n,k", [
    (synth.Q4_K, 2, "bf16", 32, 6, 64, 512, 1536),    # decode routing, a down projection's shape
    (synth.Q4_K, 2, "f32", 5, 3, 6, 130, 512),        # ragged rows
    (synth.Q4_K, 3, "bf16", 200, 4, 8, 300, 1024),    # tensor-core path, slotted rows by TMA
    (synth.Q4_K, 0, "bf16", 64, 6, 16, 256, 768),     # auto
    (synth.Q4_K, 1, "f32", 9, 2, 5, 129, 256),
    (synth.Q8_0, 0, "bf16", 11, 3, 6, 96, 1408),      # K = 1408: 44 blocks of 32
    (synth.Q2_K, 0, "f32", 6, 2, 4, 70, 512),
    (synth.Q5_K, 0, "bf16", 6, 2, 4, 70, 512),
    (synth.Q6_K, 0, "f32", 6, 2, 4, 70, 512),
    (synth.TQ1_G128, 0, "bf16", 7, 2, 4, 64, 1408),
])
def test_matmul_id_mix(kq, codec, path, xdt, t, top_k, e, n, k):
    """Down projection with the routing mix: per token, the score-weighted sum
    of its slots' products against the fp64 oracle; deterministic; bf16 out."""
    import torch

    r = rng(3 * t + n + k + codec + path)
    w = synth.gen_weights(codec, e * n, k, r).reshape(e, n, -1)
    xs = synth.gen_x(t * top_k, k, xdt, r).reshape(t, top_k, k)
    ids = synth.gen_ids(t, top_k, e, r)
    scores = r.uniform(0.0, 1.0, (t, top_k)).astype(np.float32)
    ref = oracle.mix_id(codec, w, k, xs, ids, scores)
    pref = _pair_refs(codec, w, k, xs, ids)
    wd, xd = to_device_w(w), to_device_x(xs, xdt)
    idd, sd = torch.from_numpy(ids).cuda(), torch.from_numpy(scores).cuda()
    y = kq.matmul_id_mix(wd, codec, xd, idd, sd, path=path).cpu().numpy()
    if path == 3 or (path == 0 and codec == synth.Q4_K and xdt == "bf16" and t * top_k > e) or \
            (path == 0 and xdt == "bf16" and _grouped_gemm_takes(codec, k)):
        tol = TOL["bf16"]
    elif codec == synth.Q4_K and path in (0, 2):
        tol = GEMV_TOL
    else:
        tol = FP32_PATH_TOL
    ok, worst = _mix_err_ok(y, ref, pref, scores, tol)
    assert ok, worst
    y2 = kq.matmul_id_mix(wd, codec, xd, idd, sd, path=path).cpu().numpy()
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))
    yb = kq.matmul_id_mix(wd, codec, xd, idd, sd, path=path, out_dtype=torch.bfloat16).float().cpu().numpy()
    assert np.all(np.abs(yb - y) <= BF16_OUT * np.abs(y) + 1e-30)


@pytest.mark.parametrize("path", [1, 2])
def test_matmul_id_mix_scores_and_bad_ids(kq, path):
    """One-hot scores give one slot's product; zero scores give zero rows;
    a token with an id outside the stack gets a NaN row and the error word."""
    import torch

    t, top_k, e, n, k = 10, 3, 5, 200, 512
    r = rng(91 + path)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    xs = synth.gen_x(t * top_k, k, "f32", r).reshape(t, top_k, k)
    ids = synth.gen_ids(t, top_k, e, r)
    wd, xd, idd = to_device_w(w), to_device_x(xs, "f32"), torch.from_numpy(ids).cuda()
    one = np.zeros((t, top_k), np.float32)
    one[:, 2] = 1.0
    y = kq.matmul_id_mix(wd, synth.Q4_K, xd, idd, torch.from_numpy(one).cuda(), path=path).cpu().numpy()
    y1 = kq.matmul_id(wd, synth.Q4_K, xd.reshape(t * top_k, k),
                      idd.reshape(-1, 1).contiguous(), path=path).cpu().numpy()[:, 0].reshape(t, top_k, n)
    assert np.array_equal(y.view(np.uint32), y1[:, 2].copy().view(np.uint32))
    z = kq.matmul_id_mix(wd, synth.Q4_K, xd, idd, torch.zeros(t, top_k).cuda(), path=path).cpu().numpy()
    assert np.all(z == 0)
    assert kq.device_status() == 0
    bad = ids.copy()
    bad[4, 1] = e
    bad[7, 0] = -3
    scores = r.uniform(0, 1, (t, top_k)).astype(np.float32)
    y = kq.matmul_id_mix(wd, synth.Q4_K, xd, torch.from_numpy(bad).cuda(), torch.from_numpy(scores).cuda(),
                         path=path).cpu().numpy()
    assert np.all(np.isnan(y[[4, 7]]))
    good = [i for i in range(t) if i not in (4, 7)]
    ref = oracle.mix_id(synth.Q4_K, w, k, xs, bad, scores)
    pref = _pair_refs(synth.Q4_K, w, k, xs[good], ids[good])
    ok, worst = _mix_err_ok(y[good], ref[good], pref, scores[good], GEMV_TOL if path == 2 else FP32_PATH_TOL)
    assert ok, worst
    assert kq.device_status() == -9
    assert kq.device_status() == 0


@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_moe_ffn_chain_reuses_the_grouping(kq, xdt):
    """GLU over the gate/up stacks, then the down projection with the mix on
    the GLU's slotted output, the second call reusing the first call's
    grouping from the shared workspace: the same bits as grouping again, and
    the oracle's mix of the GPU's GLU output within the path's bound."""
    import torch

    t, top_k, e, hdim, fdim = 12, 4, 16, 512, 768
    r = rng(1234 + len(xdt))
    wg = synth.gen_weights(synth.Q4_K, e * fdim, hdim, r).reshape(e, fdim, -1)
    wu = synth.gen_weights(synth.Q4_K, e * fdim, hdim, r).reshape(e, fdim, -1)
    wdn = synth.gen_weights(synth.Q4_K, e * hdim, fdim, r).reshape(e, hdim, -1)
    x = synth.gen_x(t, hdim, xdt, r)
    ids = synth.gen_ids(t, top_k, e, r)
    scores = r.uniform(0, 1, (t, top_k)).astype(np.float32)
    idd, sd = torch.from_numpy(ids).cuda(), torch.from_numpy(scores).cuda()
    ws = torch.empty(kq.matmul_id_mix_workspace_bytes(t, top_k, e, hdim), dtype=torch.uint8, device="cuda")
    h = kq.matmul_id_glu(to_device_w(wg), to_device_w(wu), synth.Q4_K, to_device_x(x, xdt), idd,
                         workspace=ws)
    y = kq.matmul_id_mix(to_device_w(wdn), synth.Q4_K, h, idd, sd, workspace=ws, reuse_grouping=True,
                         path=2).cpu().numpy()
    y_fresh = kq.matmul_id_mix(to_device_w(wdn), synth.Q4_K, h, idd, sd, path=2).cpu().numpy()
    assert np.array_equal(y.view(np.uint32), y_fresh.view(np.uint32))
    hn = h.cpu().numpy().astype(np.float64)
    ref = oracle.mix_id(synth.Q4_K, wdn, fdim, hn, ids, scores)
    ok, worst = _mix_err_ok(y, ref, _pair_refs(synth.Q4_K, wdn, fdim, hn, ids), scores, GEMV_TOL)
    assert ok, worst
    # and the whole block against the oracle's chain
    full = oracle.mix_id(synth.Q4_K, wdn, fdim, oracle.glu_id(synth.Q4_K, wg, wu, hdim, x, ids, "silu"),
                         ids, scores)
    assert row_rel_err(y, full) <= 4 * GEMV_TOL
    assert kq.device_status() == 0


@pytest.mark.parametrize("t,top_k,e,n,k,skew", [
    (32, 6, 64, 1408, 2048, False),    # the MoE workload: ~3 pairs per expert, one token tile each
    (5, 3, 6, 130, 512, False),        # ragged weight rows, one tile of rows and a partial one
    (100, 2, 3, 300, 1024, False),     # ~66 pairs per expert: five token tiles each
    (7, 3, 4, 129, 4096, False),       # the largest K the kernel takes
    (64, 4, 8, 256, 768, True),        # one expert takes most pairs: many tiles, other experts one
    (8, 2, 32, 1408, 2048, False),     # at most one pair per expert: the int8 form
])
@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_matmul_id_tensor_core_few_pairs(kq, t, top_k, e, n, k, skew, xdt):
    """The few-pairs tensor-core kernel: codes through the MMA, a sub-block
    accumulator each, scales applied after it -- against the fp64 oracle
    (bf16 activations exact in the MMA), f32 and bf16 outputs, bit-stable,
    and a NaN row for an id outside the stack."""
    import torch

    r = rng(11 * t + e + n + k)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, xdt, r)
    ids = synth.gen_ids(t, top_k, e, r)
    if skew:
        ids[:, 0] = np.where(np.arange(t) % 9 == 0, 1, 2)
    ids[t // 2, top_k - 1] = e                 # outside the stack: a NaN row
    ref = oracle.matmul_id(synth.Q4_K, w, k, x, ids)
    wd, xd, idd = to_device_w(w), to_device_x(x, xdt), torch.from_numpy(ids).cuda()
    y = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMV_TC).cpu().numpy()
    assert np.all(np.isnan(y[t // 2, top_k - 1]))
    good = ~np.isnan(ref[..., 0])
    err = row_rel_err(y[good], ref[good])
    assert err <= GEMV_TOL, err
    assert kq.device_status() == -9
    y2 = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMV_TC).cpu().numpy()
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))
    yb = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMV_TC,
                      out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb[good], ref[good]) <= GEMV_TOL + BF16_OUT
    assert kq.device_status() == -9
    assert kq.device_status() == 0


@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_matmul_id_tensor_core_nonfinite_and_slotted(kq, xdt):
    """Non-finite activations send their token tile through the exact fp32
    path (IEEE classes as the oracle's); the slotted input of the down
    projection (one activation row per pair) through the same kernel."""
    import torch

    t, top_k, e, n, k = 12, 2, 5, 160, 512
    r = rng(77)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, xdt, r)
    ids = synth.gen_ids(t, top_k, e, r)
    x[3, 10] = np.inf
    x[5, 100] = np.nan
    ref = oracle.matmul_id(synth.Q4_K, w, k, x, ids)
    y = kq.matmul_id(to_device_w(w), synth.Q4_K, to_device_x(x, xdt), torch.from_numpy(ids).cuda(),
                     path=kq.PATH_GEMV_TC).cpu().numpy()
    assert np.array_equal(np.isnan(y), np.isnan(ref))
    assert np.array_equal(np.isposinf(y), np.isposinf(ref)) and np.array_equal(np.isneginf(y), np.isneginf(ref))
    assert np.isinf(ref[3]).any() and np.isnan(ref[5]).all()
    fin = np.isfinite(ref)
    scale = np.abs(ref[fin]).max()
    assert np.all(np.abs(y[fin] - ref[fin]) <= GEMV_TOL * scale)
    assert kq.device_status() == 0
    xs = synth.gen_x(t * top_k, k, xdt, r).reshape(t, top_k, k)
    scores = r.uniform(0, 1, (t, top_k)).astype(np.float32)
    ym = kq.matmul_id_mix(to_device_w(w), synth.Q4_K, to_device_x(xs, xdt), torch.from_numpy(ids).cuda(),
                          torch.from_numpy(scores).cuda(), path=kq.PATH_GEMV_TC).cpu().numpy()
    refm = oracle.mix_id(synth.Q4_K, w, k, xs, ids, scores)
    ok, worst = _mix_err_ok(ym, refm, _pair_refs(synth.Q4_K, w, k, xs, ids), scores, GEMV_TOL)
    assert ok, worst
    assert kq.device_status() == 0


@pytest.mark.parametrize("n,k,m", [(4096, 4096, 1), (1000, 2048, 3), (300, 512, 16), (777, 4096, 21),
                                   (11008 // 8, 4096, 8)])
@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_matmul_dense_tensor_core_few_rows(kq, n, k, m, xdt):
    """The few-rows tensor-core kernel on one matrix (tiles of 16 bf16 or 8
    fp32 activation rows, ragged last tiles) against the fp64 oracle."""
    import torch

    r = rng(5 * n + k + m)
    w = synth.gen_weights(synth.Q4_K, n, k, r)
    x = synth.gen_x(m, k, xdt, r)
    ref = oracle.matmul(synth.Q4_K, w, k, x, threads=8)
    wd, xd = to_device_w(w), to_device_x(x, xdt)
    y = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMV_TC).cpu().numpy()
    assert row_rel_err(y, ref) <= GEMV_TOL
    yb = kq.matmul(wd, synth.Q4_K, xd, path=kq.PATH_GEMV_TC, out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= GEMV_TOL + BF16_OUT
    assert kq.device_status() == 0


def _bf16_weight_reference_id(w, k, x, ids, codec=synth.Q4_K):
    """y[t, s] = x[t] @ bf16(decode_f32(w[ids[t, s]]))^T in fp64 (NaN rows for
    ids outside [0, E)): the tensor-core expert product up to fp32 accumulation."""
    e_n = w.shape[0]
    ref = np.full(ids.shape + (w.shape[1],), np.nan)
    for e in range(e_n):
        hit = ids == e
        if hit.any():
            ye = _bf16_weight_reference(w[e], k, x, codec)   # [T, n]
            ref[hit] = ye[np.nonzero(hit)[0]]
    return ref


@pytest.mark.parametrize("t,top_k,e,n,k,skew", [
    (512, 6, 64, 384, 2048, False),    # the MoE routing at prefill length (3 weight tiles)
    (100, 2, 3, 300, 1024, False),     # ragged weight rows, ~66 pairs per expert
    (64, 4, 8, 129, 512, False),
    (7, 3, 4, 129, 512, False),        # a handful of pairs: token tiles of 16
    (300, 1, 4, 256, 512, True),       # one expert takes almost every token
])
def test_matmul_id_grouped_gemm(kq, t, top_k, e, n, k, skew):
    import torch

    r = rng(7 * t + e + n)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, "bf16", r)
    ids = synth.gen_ids(t, top_k, e, r)
    if skew:
        ids[:, 0] = np.where(np.arange(t) % 50 == 0, 1, 2)
    ref = oracle.matmul_id(synth.Q4_K, w, k, x, ids)
    wd, xd, idd = to_device_w(w), to_device_x(x, "bf16"), torch.from_numpy(ids).cuda()
    y = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMM).cpu().numpy()
    assert row_rel_err(y, ref) <= TOL["bf16"]
    assert row_rel_err(y, _bf16_weight_reference_id(w, k, x, ids)) <= FP32_PATH_TOL
    y2 = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMM).cpu().numpy()
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))   # deterministic
    yb = kq.matmul_id(wd, synth.Q4_K, xd, idd, path=kq.PATH_GEMM,
                      out_dtype=torch.bfloat16).float().cpu().numpy()
    assert row_rel_err(yb, ref) <= TOL["bf16"] + BF16_OUT
    assert kq.device_status() == 0


@pytest.mark.parametrize("codec,t,top_k,e,n,k", [
    (synth.Q8_0, 64, 4, 8, 300, 1024), (synth.Q8_0, 7, 3, 4, 129, 256),
    (synth.Q2_K, 64, 4, 8, 300, 2048), (synth.Q2_K, 200, 2, 5, 128, 1024),
    (synth.Q5_K, 64, 4, 8, 300, 1024), (synth.Q5_K, 9, 2, 3, 70, 512),
])
def test_matmul_id_grouped_gemm_other_codecs(kq, codec, t, top_k, e, n, k):
    """The grouped tensor-core GEMM for Q8_0, Q2_K and Q5_K experts (the
    automatic path for bf16 activations): the bf16-weight product per pair,
    deterministic, in stream order with the grouping."""
    import torch

    r = rng(11 * t + e + n + codec)
    w = synth.gen_weights(codec, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, "bf16", r)
    ids = synth.gen_ids(t, top_k, e, r)
    ref = oracle.matmul_id(codec, w, k, x, ids)
    wd, xd, idd = to_device_w(w), to_device_x(x, "bf16"), torch.from_numpy(ids).cuda()
    y = kq.matmul_id(wd, codec, xd, idd, path=kq.PATH_GEMM).cpu().numpy()
    assert row_rel_err(y, ref) <= TOL["bf16"]
    assert row_rel_err(y, _bf16_weight_reference_id(w, k, x, ids, codec)) <= FP32_PATH_TOL
    ya = kq.matmul_id(wd, codec, xd, idd).cpu().numpy()   # automatic: the same kernel
    assert np.array_equal(y.view(np.uint32), ya.view(np.uint32))
    assert kq.device_status() == 0


def test_matmul_id_auto_uses_tensor_cores_for_long_prefill(kq):
    import torch

    t, top_k, e, n, k = 512, 6, 64, 256, 1024   # 48 pairs per expert on average
    r = rng(99)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, "bf16", r)
    ids = synth.gen_ids(t, top_k, e, r)
    y = kq.matmul_id(to_device_w(w), synth.Q4_K, to_device_x(x, "bf16"),
                     torch.from_numpy(ids).cuda()).cpu().numpy()
    # equal to the bf16-weight product: the tensor-core path ran
    assert row_rel_err(y, _bf16_weight_reference_id(w, k, x, ids)) <= FP32_PATH_TOL
    assert kq.device_status() == 0


@pytest.mark.parametrize("path", ["auto", "gemm"])
def test_matmul_id_bad_ids_poison_rows_bf16(kq, path):
    import torch

    e, n, k, t = 4, 140, 512, 40
    r = rng(12)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, "bf16", r)
    ids = synth.gen_ids(t, 2, e, r)
    ids[1, 0] = 4
    ids[30, 1] = -7
    p = {"auto": kq.PATH_AUTO, "gemm": kq.PATH_GEMM}[path]
    y = kq.matmul_id(to_device_w(w), synth.Q4_K, to_device_x(x, "bf16"), torch.from_numpy(ids).cuda(),
                     path=p).cpu().numpy()
    ref = oracle.matmul_id(synth.Q4_K, w, k, x, ids)
    assert np.all(np.isnan(y[1, 0])) and np.all(np.isnan(y[30, 1]))
    good = ~np.isnan(ref[..., 0])
    assert row_rel_err(y[good], ref[good]) <= TOL["bf16"]
    assert kq.device_status() == -9    # KQ_ERR_DEVICE, then cleared
    assert kq.device_status() == 0


def test_matmul_id_bad_ids_poison_rows(kq):
    import torch

    e, n, k, t = 4, 33, 512, 5
    r = rng(11)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, "f32", r)
    ids = synth.gen_ids(t, 2, e, r)
    ids[1, 0] = 4
    ids[3, 1] = -7
    y = kq.matmul_id(to_device_w(w), synth.Q4_K, to_device_x(x, "f32"), torch.from_numpy(ids).cuda()
                     ).cpu().numpy()
    ref = oracle.matmul_id(synth.Q4_K, w, k, x, ids)
    assert np.all(np.isnan(y[1, 0])) and np.all(np.isnan(y[3, 1]))
    good = ~np.isnan(ref[..., 0])
    assert row_rel_err(y[good], ref[good]) <= GEMV_TOL
    assert kq.device_status() == -9    # KQ_ERR_DEVICE, then cleared
    assert kq.device_status() == 0


@pytest.mark.parametrize("xdt,path", [("f32", "auto"), ("bf16", "auto"), ("bf16", "gemm"), ("f32", "simple")])
def test_matmul_id_all_ids_invalid(kq, xdt, path):
    """No valid pair: the grouping leaves every expert empty (zero token
    tiles for the tensor-core path, zero passes for the grouped GEMV), every
    output row is the poison sentinel and the error word is set once."""
    import torch

    e, n, k, t, top_k = 3, 140, 512, 24, 2
    r = rng(13)
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    x = synth.gen_x(t, k, xdt, r)
    ids = np.where(np.arange(t * top_k).reshape(t, top_k) % 2 == 0, e, -1).astype(np.int32)
    p = {"auto": kq.PATH_AUTO, "gemm": kq.PATH_GEMM, "simple": kq.PATH_SIMPLE}[path]
    y = kq.matmul_id(to_device_w(w), synth.Q4_K, to_device_x(x, xdt), torch.from_numpy(ids).cuda(),
                     path=p).float().cpu().numpy()
    assert y.shape == (t, top_k, n)
    assert np.all(np.isnan(y))
    assert np.all(np.isnan(oracle.matmul_id(synth.Q4_K, w, k, x, ids)))
    assert kq.device_status() == -9
    assert kq.device_status() == 0


# ---------------------------------------------------------------- errors on device arguments

def test_error_codes(kq):
    import torch

    w = to_device_w(synth.gen_weights(synth.Q4_K, 8, 512, rng(1)))
    xf = torch.zeros((1, 512), dtype=torch.float32, device="cuda")
    with pytest.raises(kq.KQError) as ei:
        kq.matmul(w, synth.Q4_K, xf, path=kq.PATH_GEMM)       # tensor-core path needs bf16 x
    assert ei.value.status == -11
    bad_out = torch.empty((1, 9), device="cuda")[:, 1:]        # 4-byte offset
    with pytest.raises(kq.KQError) as ei:
        kq.matmul(w, synth.Q4_K, xf, out=bad_out, path=kq.PATH_SIMPLE)
    assert ei.value.status == -5
    assert kq.device_status() == 0


def test_binding_rejects_wrong_buffers_before_any_launch(kq):
    """Buffers whose size the C ABI cannot see are checked by the binding."""
    import torch

    w = to_device_w(synth.gen_weights(synth.Q4_K, 8, 512, rng(2)))
    x = torch.zeros((2, 512), dtype=torch.bfloat16, device="cuda")
    for bad in (torch.empty((2, 7), device="cuda"), torch.empty((8, 2), device="cuda").t(),
                torch.empty((2, 8), dtype=torch.float64, device="cuda")):
        with pytest.raises(ValueError):
            kq.matmul(w, synth.Q4_K, x, out=bad)
    with pytest.raises(ValueError):
        kq.dequantize(w, synth.Q4_K, 512, out=torch.empty((8, 256), device="cuda"))
    we = w.view(2, 4, -1)
    ids = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        kq.matmul_id(we, synth.Q4_K, x, ids, out=torch.empty((2, 1, 3), device="cuda"))
    with pytest.raises(ValueError):
        kq.matmul_id(we, synth.Q4_K, x, ids.to(torch.int64))
    assert kq.device_status() == 0
