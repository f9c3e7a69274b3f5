"""The KQ_DEBUG build of the library (libkq_debug.so, include/kq_debug.h).

* A bounded wait that runs out reports KQ_ERR_DEVICE_TIMEOUT through
  kq_device_status, the next status is clean, and the context stays usable.
* Grouping entries out of range (a workspace grouping reused when it does
  not fit, the misuse KQ_FLAG_REUSE_GROUPING warns about) are caught by the
  device bounds checks: KQ_ERR_DEVICE_BOUNDS instead of reads or writes
  outside the buffers, and every other token's result unchanged.  The
  buffers are padded past their ends, so even a check that did not fire
  would stay inside memory the test owns.
* The small parity cases pass under the KQ_DEBUG build.

The library a process loads is fixed at import, so the parent test runs
this file and the parity file's small cases in a child process with
KQ_DEBUG_LIBRARY=1; the debug-only tests skip in the parent.
"""
import os
import subprocess
import sys
import time

import numpy as np
import pytest

import oracle
import synth
from kqtest import FP32_PATH_TOL, row_rel_err, to_device_w, to_device_x

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
IN_CHILD = os.environ.get("KQ_DEBUG_LIBRARY", "") == "1"
debug_only = pytest.mark.skipif(not IN_CHILD, reason="runs in the KQ_DEBUG child process")


@pytest.mark.skipif(IN_CHILD, reason="the child itself")
def test_debug_build_runs_the_checks_and_the_small_parity_cases(kq):
    env = dict(os.environ, KQ_DEBUG_LIBRARY="1")
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-rs", "-m", "gpu", "-p", "no:cacheprovider",
         os.path.join(HERE, "test_gpu_debug_build.py"), os.path.join(HERE, "test_gpu_parity.py"),
         "-k", "not full_size and not sampled_rows"],
        env=env, cwd=ROOT, capture_output=True, text=True, timeout=1500)
    tail = r.stdout[-4000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail
    # the debug-only tests ran there (none skipped), and the parity file with them
    assert "runs in the KQ_DEBUG child process" not in r.stdout, tail
    print(r.stdout[-1500:])


@debug_only
@pytest.mark.parametrize("mode", [0, 1])
def test_bounded_wait_runs_out_and_the_context_stays_usable(kq, mode):
    import torch

    assert kq.DEBUG_LIBRARY and kq.lib().kq_debug_spin_limit() > 0
    assert kq.device_status() == 0
    t0 = time.perf_counter()
    kq.debug_wait_timeout(mode)
    assert kq.device_status() == -10          # KQ_ERR_DEVICE_TIMEOUT (synchronizes)
    assert time.perf_counter() - t0 < 10.0    # the debug limit is milliseconds
    assert kq.device_status() == 0            # read and cleared
    r = np.random.Generator(np.random.PCG64(5 + mode))
    w = synth.gen_weights(synth.Q4_K, 96, 512, r)
    x = synth.gen_x(3, 512, "f32", r)
    y = kq.matmul(to_device_w(w), synth.Q4_K, to_device_x(x, "f32"), path=kq.PATH_SIMPLE)
    assert row_rel_err(y.cpu().numpy(), oracle.matmul(synth.Q4_K, w, 512, x)) <= FP32_PATH_TOL
    assert kq.device_status() == 0
    torch.cuda.synchronize()


def _up256(v):
    return (v + 255) // 256 * 256


@debug_only
@pytest.mark.parametrize("path", [1, 2, 3, 4])
def test_bounds_checks_catch_a_grouping_out_of_range(kq, path):
    import torch

    t, top_k, e, n, k = 24, 4, 8, 160, 512
    pairs = t * top_k
    r = np.random.Generator(np.random.PCG64(40 + path))
    w = synth.gen_weights(synth.Q4_K, e * n, k, r).reshape(e, n, -1)
    xdt = "bf16" if path in (3, 4) else "f32"
    xs = synth.gen_x(pairs, k, xdt, r)
    ids = synth.gen_ids(t, top_k, e, r)
    scores = r.uniform(0, 1, (t, top_k)).astype(np.float32)
    wd, idd, sd = to_device_w(w), torch.from_numpy(ids).cuda(), torch.from_numpy(scores).cuda()
    # x padded by 64 rows and the workspace by 64 output rows past their ends
    xpad = torch.zeros((pairs + 64, k), dtype=torch.bfloat16 if xdt == "bf16" else torch.float32, device="cuda")
    xpad[:pairs] = to_device_x(xs, xdt)
    xd = xpad[:pairs].view(t, top_k, k)
    need = kq.matmul_id_mix_workspace_bytes(t, top_k, e, n)
    ws = torch.zeros(need + 64 * n * 4 + 4096, dtype=torch.uint8, device="cuda")
    clean = kq.matmul_id_mix(wd, synth.Q4_K, xd, idd, sd, workspace=ws, path=path).cpu().numpy()
    assert kq.device_status() == 0
    # the grouping the clean call left: counts [E], offsets [E+1], perm [pairs]
    off_offsets = _up256(4 * e)
    off_perm = off_offsets + _up256(4 * (e + 1))
    counts = ws[:4 * e].view(torch.int32)
    offsets = ws[off_offsets:off_offsets + 4 * (e + 1)].view(torch.int32)
    perm = ws[off_perm:off_perm + 4 * pairs].view(torch.int32)
    assert int(offsets[e]) == pairs and int(counts.sum()) == pairs
    lost_pair = int(perm[0])
    perm[0] = pairs + 1                  # a pair id past the end
    counts[e - 1] += 3                   # the last expert's segment runs past perm's end
    offsets[e] += 3
    y = kq.matmul_id_mix(wd, synth.Q4_K, xd, idd, sd, workspace=ws, reuse_grouping=True,
                         path=path).cpu().numpy()
    assert kq.device_status() == -12     # KQ_ERR_DEVICE_BOUNDS
    assert kq.device_status() == 0
    # tokens with no pair on the last expert and not the displaced pair are unchanged
    keep = [i for i in range(t) if (ids[i] != e - 1).all() and i != lost_pair // top_k]
    assert len(keep) >= 4
    assert np.array_equal(y[keep].view(np.uint32), clean[keep].view(np.uint32))
    # and the context is fine: a fresh grouping gives the clean result again
    again = kq.matmul_id_mix(wd, synth.Q4_K, xd, idd, sd, path=path).cpu().numpy()
    assert np.array_equal(again.view(np.uint32), clean.view(np.uint32))
    assert kq.device_status() == 0
