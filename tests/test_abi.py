"""The C-ABI library loads and exports every symbol include/kq.h declares.
Runs without a GPU: only calls that do not touch a device are made."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    import block_quantized_matmul_quant_b200 as kq

    kq.ensure_built()
    return kq.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kq.h")).read()
    return re.findall(r"KQ_API\s+[\w\s\*]+?\b(kq_\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for required in ("kq_dequantize", "kq_matmul", "kq_matmul_id", "kq_device_status",
                     "kq_validate", "kq_row_bytes", "kq_matmul_id_workspace_bytes"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_block_geometry_and_row_bytes(L):
    assert (L.kq_block_weights(8), L.kq_block_bytes(8)) == (32, 34)
    assert (L.kq_block_weights(12), L.kq_block_bytes(12)) == (256, 144)
    assert (L.kq_block_weights(10), L.kq_block_bytes(10)) == (256, 84)
    assert (L.kq_block_weights(1001), L.kq_block_bytes(1001)) == (128, 28)
    assert (L.kq_block_weights(13), L.kq_block_bytes(13)) == (256, 176)
    assert (L.kq_block_weights(14), L.kq_block_bytes(14)) == (256, 210)
    assert L.kq_row_bytes(14, 1024) == 840
    assert L.kq_block_weights(3) == 0
    assert L.kq_row_bytes(12, 4096) == 2304
    assert L.kq_row_bytes(1001, 17408) == 3808
    assert L.kq_row_bytes(8, 1024) == 1088
    assert L.kq_row_bytes(12, 100) == -1


def test_status_strings(L):
    for st in range(0, -12, -1):
        assert L.kq_status_string(st)
    assert b"unknown" in L.kq_status_string(-99)


def test_workspace_size(L):
    b = L.kq_matmul_id_workspace_bytes(32, 6, 64)
    assert b >= 4 * (64 + 65 + 192) and b % 256 == 0
    assert L.kq_matmul_id_workspace_bytes(0, 6, 64) == 0


def test_argument_errors_before_any_launch(L):
    # All of these fail host validation, before the device is queried.
    vp = ctypes.c_void_p
    fake = vp(1 << 20)   # never dereferenced
    assert L.kq_matmul(12, None, 4, 256, fake, 1, 1, fake, 0, None) == -1          # null w
    assert L.kq_matmul(12, fake, 4, 100, fake, 1, 1, fake, 0, None) == -3          # K % 256
    assert L.kq_matmul(77, fake, 4, 256, fake, 1, 1, fake, 0, None) == -2          # codec
    assert L.kq_matmul(12, vp((1 << 20) + 8), 4, 256, fake, 1, 1, fake, 0, None) == -5  # align
    assert L.kq_matmul(12, fake, 4, 256, fake, 7, 1, fake, 0, None) == -4          # dtype
    assert L.kq_matmul(12, fake, 0, 256, fake, 1, 1, fake, 0, None) == -1          # n = 0
    assert L.kq_dequantize(1001, fake, 2, 130, fake, 0, None) == -3
    ws = L.kq_matmul_id_workspace_bytes(4, 2, 3)
    # top_k > n_experts
    assert L.kq_matmul_id(12, fake, 3, 8, 256, 8 * 144, fake, 1, 4, fake, 4, fake, 0, fake, ws,
                          None) == -1
    # expert stride smaller than one expert
    assert L.kq_matmul_id(12, fake, 3, 8, 256, 144, fake, 1, 4, fake, 2, fake, 0, fake, ws,
                          None) == -3
    # workspace too small
    assert L.kq_matmul_id(12, fake, 3, 8, 256, 8 * 144, fake, 1, 4, fake, 2, fake, 0, fake, 16,
                          None) == -7
    # overflow of n * row bytes
    assert L.kq_matmul(12, fake, 1 << 60, 256, fake, 1, 1, fake, 0, None) == -6


def test_more_argument_errors_before_any_launch(L):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    odd = vp((1 << 20) + 4)
    assert L.kq_matmul(12, fake, 4, 256, fake, 1, 0, fake, 0, None) == -1          # m = 0
    assert L.kq_matmul(12, fake, 4, 256, None, 1, 1, fake, 0, None) == -1          # null x
    assert L.kq_matmul(12, fake, 4, 256, fake, 1, 1, None, 0, None) == -1          # null y
    assert L.kq_matmul(12, fake, 4, 256, fake, 1, 1, odd, 0, None) == -5           # y alignment
    assert L.kq_matmul_ex(12, fake, 4, 256, fake, 1, 1, fake, 0, 7, None) == -1    # unknown path
    assert L.kq_dequantize(12, fake, 2, 256, fake, 9, None) == -4                  # out dtype
    ws = L.kq_matmul_id_workspace_bytes(4, 2, 3)

    def mid(n_experts=3, stride=8 * 144, ids=fake, top_k=2, work=fake, wsb=ws, path=0):
        return L.kq_matmul_id_ex(12, fake, n_experts, 8, 256, stride, fake, 1, 4, ids, top_k, fake, 0,
                                 work, wsb, path, None)

    assert mid(stride=8 * 144 + 8) == -3             # expert stride not a multiple of 16
    assert mid(ids=None) == -1
    assert mid(ids=odd) == -5
    assert mid(top_k=0) == -1
    assert mid(n_experts=70000, top_k=2) == -1       # beyond the grid's expert dimension
    assert mid(work=None) == -7
    assert mid(work=odd) == -5
    assert mid(path=9) == -1


def test_moe_group_argument_errors(L):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    assert L.kq_moe_group(None, 8, 4, fake, fake, fake, None) == -1
    assert L.kq_moe_group(fake, 0, 4, fake, fake, fake, None) == -1
    assert L.kq_moe_group(fake, 8, 70000, fake, fake, fake, None) == -1
    assert L.kq_moe_group(vp((1 << 20) + 4), 8, 4, fake, fake, fake, None) == -5   # ids alignment
    assert L.kq_moe_group(fake, 8, 4, vp((1 << 20) + 2), fake, fake, None) == -5   # counts alignment


def test_get_rows_argument_errors(L):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    assert L.kq_get_rows(12, fake, 8, 256, None, 4, fake, 0, None) == -1             # null ids
    assert L.kq_get_rows(12, fake, 8, 256, fake, 0, fake, 0, None) == -1             # no ids
    assert L.kq_get_rows(12, fake, 8, 100, fake, 4, fake, 0, None) == -3             # K % 256
    assert L.kq_get_rows(12, fake, 8, 256, vp((1 << 20) + 4), 4, fake, 0, None) == -5   # ids alignment
    assert L.kq_get_rows(12, fake, 8, 256, fake, 4, fake, 7, None) == -4             # out dtype
    assert L.kq_get_rows(99, fake, 8, 256, fake, 4, fake, 0, None) == -2             # codec


def test_mix_workspace_and_argument_errors(L):
    vp = ctypes.c_void_p
    idb = L.kq_matmul_id_workspace_bytes(4, 2, 3)
    mb = L.kq_matmul_id_mix_workspace_bytes(4, 2, 3, 100)
    # the grouping's sections, then the fp32 per-pair products (8 pairs x 100), 256-byte steps
    assert mb == idb + (8 * 100 * 4 + 255) // 256 * 256
    assert L.kq_matmul_id_mix_workspace_bytes(4, 2, 3, 0) == 0
    assert L.kq_matmul_id_mix_workspace_bytes(0, 2, 3, 100) == 0
    fake = vp(1 << 20)
    args = lambda **kw: dict(dict(t=12, w=fake, e=3, n=100, k=256, es=100 * 144, x=fake, xdt=0, nt=4,
                                  ids=fake, sc=fake, tk=2, y=fake, ydt=0, ws=fake, wsb=mb, path=0), **kw)

    def call(a):
        return L.kq_matmul_id_mix(a["t"], a["w"], a["e"], a["n"], a["k"], a["es"], a["x"], a["xdt"],
                                  a["nt"], a["ids"], a["sc"], a["tk"], a["y"], a["ydt"], a["ws"],
                                  a["wsb"], a["path"], None)

    assert call(args(sc=None)) == -1                         # null scores
    assert call(args(sc=vp((1 << 20) + 4))) == -5            # scores alignment
    assert call(args(wsb=idb)) == -7                         # no room for the per-pair products
    assert call(args(path=9)) == -1                          # unknown path
    assert call(args(ydt=2)) == -4                           # f16 output
    assert call(args(tk=4)) == -1                            # top_k > n_experts
    assert call(args(k=100)) == -3                           # K % 256


def test_debug_build_exports_its_entry_points(L):
    """libkq_debug.so exports kq.h's calls and kq_debug.h's; the release
    library has no debug entry points."""
    from block_quantized_matmul_quant_b200 import _build

    D = ctypes.CDLL(_build.LIB_DEBUG)
    src = open(os.path.join(ROOT, "include", "kq_debug.h")).read()
    debug_names = re.findall(r"KQ_API\s+[\w\s\*]+?\b(kq_\w+)\s*\(", src)
    assert set(debug_names) == {"kq_debug_wait_timeout", "kq_debug_spin_limit"}
    for name in declared_functions() + debug_names:
        assert hasattr(D, name), name
    for name in debug_names:
        assert not hasattr(L, name), name
    D.kq_debug_spin_limit.restype = ctypes.c_int
    assert D.kq_debug_spin_limit() == _build.DEBUG_SPIN_LIMIT
    D.kq_debug_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_void_p]
    assert D.kq_debug_wait_timeout(5, None) == -1     # unknown mode, before any device call
