"""Benchmark of the block-quantized product path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step runs the hot path once over one batch of synthetic input: for the
headline workload (Q4_K decode GEMV, W 4096x4096, x bf16 batch 1) the batch is
a pool of independent weight matrices whose total size is at least four times
the L2 cache, each multiplied by its own activation vector -- so every call
streams its weights from HBM (no L2 flush needed).  Steps are replayed from a
CUDA graph; the timed region is bracketed by a barrier and a synchronize and
timed with CUDA events on the launching stream (max over ranks).

Under torchrun (N > 1) every rank runs an independent replica (no collective:
the path has no exchange step) and the value is the sum over ranks of the
bytes moved divided by the slowest rank's time.

`--impl reference` times the CPU oracle (fp64, plain C) on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
HEADLINE = "q4_k_gemv_4096x4096"


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def strip_comments(src: str) -> str:
    """C/C++ source without comments and whitespace (the code a capture ran)."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            i = src.find("\n", i)
            i = n if i < 0 else i
        elif src.startswith("/*", i):
            i = src.find("*/", i + 2)
            i = n if i < 0 else i + 2
        elif src[i] in "\"'":
            q, j = src[i], i + 1
            while j < n and src[j] != q:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return "".join("".join(out).split())


def kernel_source_hash(names, read=None):
    """Hash of the kernel sources' code (comments and whitespace ignored)."""
    h = hashlib.sha256()
    for n in names:
        if read is None:
            with open(os.path.join(ROOT, "block_quantized_matmul_quant_b200", "csrc", n)) as f:
                text = f.read()
        else:
            text = read(n)
        h.update(strip_comments(text).encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel_key, sources):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        e = t[kernel_key]
        if e["source_hash"] == kernel_source_hash(sources):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            try:
                idle = bool(int(parts[4], 16) & 1)   # the GPU-idle reason bit
            except ValueError:
                idle = False
            rows.append((sm, mx, idle, parts[5:9]))
        busy = [r for r in rows if not r[2]]
        use = busy or rows   # samples under load; all of them if none was
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        reasons = {n for r in use for n, v in zip(names, r[3]) if v.lower() == "active"}
        out = {"sm_mhz": statistics.median(r[0] for r in use), "sm_max_mhz": max(r[1] for r in use),
               "reasons": sorted(reasons), "samples": len(use)}
        if not busy:
            out["idle_samples_only"] = True
        return out


def clocks_rejected(summary):
    """A timed region sampled under a hardware or thermal slowdown, or with
    the SM clock stuck well below its maximum under load and no reason given
    (a clock lock left by someone else), is measured again once."""
    if {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"} & set(summary.get("reasons", [])):
        return True
    if summary.get("idle_samples_only"):
        return False
    sm, mx = summary.get("sm_mhz"), summary.get("sm_max_mhz")
    return bool(sm and mx and sm < 0.8 * mx and not summary.get("reasons"))


# ---------------------------------------------------------------- workloads on the GPU

def _torch_setup():
    import torch

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    return torch, rank, world, local, pg


def _x_tensor(torch, x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


class GemvStep:
    """One step = every weight matrix of the pool multiplied by its activations."""

    def __init__(self, torch, kq, wl, l2_bytes):
        w, x, _ = synth.make_inputs(wl)
        self.wl = wl
        self.wbytes = w.nbytes
        self.pool = pool_size(w.nbytes, l2_bytes)
        base = torch.from_numpy(w).cuda()
        # replicas of the seeded matrix: distinct HBM addresses, same values
        self.ws = [base.clone() for _ in range(self.pool)]
        xt = _x_tensor(torch, x, wl.x_dtype).cuda()
        self.xs = [xt.clone() for _ in range(self.pool)]
        ydt = torch.float32 if wl.y_dtype == "f32" else torch.bfloat16
        self.ys = [torch.empty((wl.m, wl.n), dtype=ydt, device="cuda") for _ in range(self.pool)]
        self.kq = kq
        self.launches = self.pool
        self.x_bytes = x.size * (2 if wl.x_dtype == "bf16" else 4)
        self.y_bytes = wl.m * wl.n * (4 if wl.y_dtype == "f32" else 2)
        self.algo_bytes_per_launch = self.wbytes + self.x_bytes + self.y_bytes
        self.host_w = torch.from_numpy(w).pin_memory()
        self.host_x = _x_tensor(torch, x, wl.x_dtype).pin_memory()
        self.host_y = torch.empty((wl.m, wl.n), dtype=ydt).pin_memory()

    def run(self):
        """The pool's GEMVs have no data dependency on one another, and the
        calls say so (independent=True): consecutive calls stream side by
        side.  Each call still stages its activations, decodes every weight
        and writes its output."""
        for i in range(self.pool):
            self.kq.matmul(self.ws[i], self.wl.codec, self.xs[i], out=self.ys[i],
                           independent=True)

    def run_serial(self):
        """The same calls, each ordered after the one before it (a chain of
        dependent layers): weights stream early, activations are read only
        after the preceding kernel completes."""
        for i in range(self.pool):
            self.kq.matmul(self.ws[i], self.wl.codec, self.xs[i], out=self.ys[i],
                           const_weights=True)

    def run_e2e(self):
        """Through the public API from pinned host buffers: copy the step's
        weights and activations in, multiply, copy the result out."""
        for i in range(self.pool):
            self.ws[i].copy_(self.host_w, non_blocking=True)
            self.xs[i].copy_(self.host_x, non_blocking=True)
            self.kq.matmul(self.ws[i], self.wl.codec, self.xs[i], out=self.ys[i])
            self.host_y.copy_(self.ys[i], non_blocking=True)

    def step_units(self):
        return self.wbytes * self.pool  # weight bytes per step


class PoolStep:
    """A workload's calls over a pool of weight copies larger than 4x L2."""

    def __init__(self, torch, kq, wl, l2_bytes, glu=False):
        w, x, ids = synth.make_inputs(wl)
        self.wl, self.kq, self.glu = wl, kq, glu
        self.wbytes = w.nbytes
        self.pool = max(4, -(-4 * l2_bytes // w.nbytes))
        base = torch.from_numpy(w).cuda()
        self.ws = [base.clone() for _ in range(self.pool)]
        self.x = _x_tensor(torch, x, wl.x_dtype).cuda()
        self.ids = torch.from_numpy(ids).cuda() if ids is not None else None
        ydt = torch.float32 if wl.y_dtype == "f32" else torch.bfloat16
        shape = (wl.m, wl.top_k, wl.n) if wl.kind == "moe" else (wl.m, wl.n)
        self.y = torch.empty(shape, dtype=ydt, device="cuda")
        # independent calls must not share an output buffer
        self.ys = [torch.empty(shape, dtype=ydt, device="cuda") for _ in range(self.pool)] \
            if wl.kind == "gemv" else None
        if wl.kind == "moe":
            self.ws_bytes = kq.matmul_id_workspace_bytes(wl.m, wl.top_k, wl.n_experts)
            self.scratch = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
            self.hit_experts = len(np.unique(ids))

    def run(self):
        for i in range(self.pool):
            if self.wl.kind == "moe" and self.glu:
                # fused gate and up projections: two stacks of the pool per call
                self.kq.matmul_id_glu(self.ws[i], self.ws[(i + 1) % self.pool], self.wl.codec, self.x,
                                      self.ids, out=self.y, workspace=self.scratch)
            elif self.wl.kind == "moe":
                self.kq.matmul_id(self.ws[i], self.wl.codec, self.x, self.ids, out=self.y,
                                  workspace=self.scratch)
            elif self.wl.kind == "gemv":
                # the pool's calls are unrelated, as in the headline step
                self.kq.matmul(self.ws[i], self.wl.codec, self.x, out=self.ys[i], independent=True)
            else:
                self.kq.matmul(self.ws[i], self.wl.codec, self.x, out=self.y, const_weights=True)


def secondary_metrics(torch, kq, l2, peaks):
    """The other measured workloads, one short timed graph each."""
    out = {}
    for name in ("q4_k_gemm_512x11008x4096", "moe_q4_k_e64_1408x2048_t32_top6",
                 "tq1_g128_gemv_5120x17408", "tq1_g128_gemm_512x5120x17408", "q8_0_gemv_256x1024"):
        wl = synth.WORKLOADS[name]
        st = PoolStep(torch, kq, wl, l2)
        ms = time_graph(torch, st.run, 5, 3, None)
        us = ms * 1e3 / (5 * st.pool)
        out[name] = secondary_entry(wl, us, st.wbytes, getattr(st, "hit_experts", 0), peaks)
        del st
        torch.cuda.empty_cache()
    # the fused GLU (gate and up in one call) on the MoE workload's routing
    name = "moe_q4_k_e64_1408x2048_t32_top6"
    wl = synth.WORKLOADS[name]
    st = PoolStep(torch, kq, wl, l2, glu=True)
    ms = time_graph(torch, st.run, 5, 3, None)
    us = ms * 1e3 / (5 * st.pool)
    out[name + "_glu"] = glu_entry(wl, us, st.wbytes, st.hit_experts, out[name]["gate_up_pair_us"], peaks)
    del st
    torch.cuda.empty_cache()
    return out


def glu_entry(wl, us, wbytes, hit_experts, gate_up_pair_us, peaks):
    """The fused GLU's figures: both stacks' hit experts stream once per call."""
    per_expert = wbytes // wl.n_experts
    moved = 2 * hit_experts * per_expert + wl.m * wl.k * 2 + wl.m * wl.top_k * wl.n * 4
    return {"us_per_call": round(us, 2), "vs_gate_up_pair_us": gate_up_pair_us,
            "GB/s": round(moved / (us * 1e-6) / 1e9, 1),
            "frac_hbm": round(moved / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
            "kernel": "moe_group + fused GLU (kq_matmul_id_glu)"}


def secondary_entry(wl, us, wbytes, hit_experts, peaks):
    """One secondary workload's figures from its time per call."""
    if wl.kind == "gemm":
        tf = 2.0 * wl.m * wl.n * wl.k / (us * 1e-6) / 1e12
        return {"us_per_call": round(us, 2), "TFLOP/s": round(tf, 1),
                "frac_burst": round(tf / peaks["bf16_tflops"], 4),
                "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                "kernel": ("gemm_tq1_kernel" if wl.codec == synth.TQ1_G128 else "gemm_q4k_kernel") + " (tcgen05)"}
    if wl.kind == "moe":
        per_expert = wbytes // wl.n_experts
        moved = hit_experts * per_expert + wl.m * wl.k * 2 + wl.m * wl.top_k * wl.n * 4
        # consecutive calls share the ids and use different expert stacks:
        # a gate projection followed by an up projection
        return {"us_per_call": round(us, 2), "gate_up_pair_us": round(2 * us, 2),
                "tokens/s": round(wl.m / (us * 1e-6), 1),
                "GB/s": round(moved / (us * 1e-6) / 1e9, 1),
                "frac_hbm": round(moved / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                "hit_experts": hit_experts, "kernel": "moe_group + grouped product"}
    gbs = wbytes / (us * 1e-6) / 1e9
    return {"us_per_call": round(us, 3), "weight GB/s": round(gbs, 1),
            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}


def time_graph(torch, fn, steps, warmup, pg):
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fn()
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(steps):
            g.replay()
        b.record(s)
        b.synchronize()
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
    ms = a.elapsed_time(b)
    del g
    return ms


def time_eager(torch, fn, steps, warmup, pg):
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(steps):
            fn()
        b.record(s)
        b.synchronize()
        if pg is not None:
            pg.barrier()
    return a.elapsed_time(b)


def max_over_ranks(torch, pg, v):
    """The slowest rank's time: every rank's replica must finish."""
    if pg is None:
        return v
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, steps, world, ms):
    """Whole-job rate: the units every replica processed over the slowest
    rank's time (weak scaling: each rank streams its own pool)."""
    return units_per_rank_step * steps * world / (ms / 1e3)


def _time_oracle_gemvs(wl, w, x, threads, budget_s):
    import oracle

    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.matmul(wl.codec, w, wl.k, x, threads=threads)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 10000:
            return n, el


def cpu_baseline_gemv(wl, budget_s=10.0):
    """The oracle as it stands, on the host's cores, over whole GEMVs of the
    workload repeated until ~budget_s of CPU work; GB/s of weight bytes.  It
    runs on every core of the process's affinity set, and once more on a
    single thread for a third of the budget."""
    w, x, _ = synth.make_inputs(wl)
    cores = len(os.sched_getaffinity(0))
    n, el = _time_oracle_gemvs(wl, w, x, cores, budget_s)
    n1, el1 = _time_oracle_gemvs(wl, w, x, 1, budget_s / 3)
    name = f"{wl.n}x{wl.k} {synth.CODEC_NAMES[wl.codec]}"
    return {"value": w.nbytes * n / el / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} whole {name} GEMVs (fp64 accumulate) in {el:.1f} s on {cores} threads",
            "single_thread": {"value": w.nbytes * n1 / el1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"{n1} whole {name} GEMVs in {el1:.1f} s on one thread"}}


def headline_config(wl, wbytes, pool, l2, world):
    """The `config` object of the bench line; both arms print the same one."""
    return {
        "workload": wl.name,
        "weights": f"{wl.n}x{wl.k} {synth.CODEC_NAMES[wl.codec].upper()} ({wbytes} B)",
        "x": f"{wl.x_dtype} [{wl.m},{wl.k}]",
        "y": f"{wl.y_dtype} [{wl.m},{wl.n}]",
        "pool_matrices_per_step": pool,
        "l2_policy": f"inputs larger than L2: each step streams {pool} distinct weight "
                     f"matrices ({pool * wbytes / 1e6:.0f} MB > 4x L2 {l2 / 1e6:.0f} MB)",
        "parallelism": f"replicas x{world}",
        "calls": "independent (kq flag: no call reads or writes another's buffers; "
                 "each still stages x, decodes every weight, writes y)",
    }


def pool_size(wbytes, l2):
    """Distinct weight matrices per step: at least four times the L2 cache."""
    return max(8, -(-4 * l2 // wbytes))


# B200 L2 as the CUDA runtime reports it; used only when no device is visible.
B200_L2_BYTES = 132644864


def l2_bytes(local=0):
    try:
        import torch

        if torch.cuda.is_available():
            return int(torch.cuda.get_device_properties(local).L2_cache_size)
    except Exception:
        pass
    return B200_L2_BYTES


def run_gpu(args):
    torch, rank, world, local, pg = _torch_setup()
    import block_quantized_matmul_quant_b200 as kq

    kq.lib()
    wl = synth.WORKLOADS[args.workload]
    if wl.kind != "gemv":
        raise SystemExit("the bench's headline step is the decode GEMV workload")
    l2 = l2_bytes(local)
    step = GemvStep(torch, kq, wl, l2)
    peaks = load_peaks()
    for attempt in range(2):
        with ClockSampler(local) as clk:
            ms = time_graph(torch, step.run, args.steps, args.warmup, pg)
        clocks = clk.summary()
        # every rank takes the same number of attempts
        if attempt == 1 or max_over_ranks(torch, pg, float(clocks_rejected(clocks))) == 0.0:
            break
    clocks["remeasured"] = attempt == 1
    ms = max_over_ranks(torch, pg, ms)
    serial_steps = max(3, args.steps // 4)
    serial_ms = max_over_ranks(torch, pg, time_graph(torch, step.run_serial, serial_steps, 3, pg))
    serial_us = serial_ms * 1e3 / (serial_steps * step.launches)
    e2e_ms = time_eager(torch, step.run_e2e, max(1, args.steps // 4), 1, pg)
    e2e_ms = max_over_ranks(torch, pg, e2e_ms) / max(1, args.steps // 4)
    status = kq.device_status()
    if status != 0:  # a kernel reported a bad input or a wait that gave up: no number
        raise SystemExit(f"device status {status} during the timed steps")
    per_step_ms = ms / args.steps
    value = job_throughput(step.step_units(), args.steps, world, ms) / 1e9
    launch_us = ms * 1e3 / (args.steps * step.launches)
    achieved = step.algo_bytes_per_launch / (launch_us * 1e-6) / 1e9
    traffic = measured_traffic("gemv_q4k_4096x4096", ["kq_gemv.cu", "kq_ptx.cuh", "kq_common.cuh", "kq_decode.cuh"])
    out = {
        "metric": "Q4_K GEMV weight GB/s",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(per_step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int16 activation codes x u4 quants (dp2a, int32), f32 scale-and-sum",
        "data": "synthetic (seeded Q4_K wire bytes and N(0,1) bf16 activations)",
        "config": headline_config(wl, step.wbytes, step.pool, l2, world),
        "serial_chain": {
            "us_per_call": round(serial_us, 4),
            "GB/s": round(step.wbytes / (serial_us * 1e-6) / 1e9, 1),
            "note": "same calls, each ordered after the previous kernel (dependent layers)",
        },
        "gpu_launches": args.steps * step.launches,
        "e2e": {
            "value": round(step.step_units() / (e2e_ms / 1e3) / 1e9 * world, 3),
            "unit": "GB/s",
            "h2d_bytes_per_step": (step.wbytes + step.x_bytes) * step.pool,
            "d2h_bytes_per_step": step.y_bytes * step.pool,
        },
        "roofline": {
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"],
            "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic,
            "peak_source": peaks["source"],
            "kernel": "gemv_q4k_kernel",
            "launch_us": round(launch_us, 4),
        },
        "clocks": clocks,
    }
    if world == 1 and not args.no_secondary:
        out["secondary"] = secondary_metrics(torch, kq, l2, peaks)
        status = kq.device_status()
        if status != 0:
            raise SystemExit(f"device status {status} during the secondary workloads")
    if rank == 0 and world == 1:
        out["cpu_baseline"] = cpu_baseline_gemv(wl, budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def run_reference(args):
    """The oracle (CPU) as the reference arm: each step is one whole GEMV of
    the workload on all host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    wl = synth.WORKLOADS[args.workload]
    w, x, _ = synth.make_inputs(wl)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    l2 = l2_bytes()
    cores = len(os.sched_getaffinity(0))
    for _ in range(args.warmup):
        oracle.matmul(wl.codec, w, wl.k, x, threads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.matmul(wl.codec, w, wl.k, x, threads=cores)
    el = time.perf_counter() - t0
    value = w.nbytes * args.steps / el / 1e9
    print(json.dumps({
        "impl": "reference",
        "metric": "Q4_K GEMV weight GB/s",
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8 Q4_K weights, fp64 accumulate",
        "data": "synthetic",
        "config": headline_config(wl, w.nbytes, pool_size(w.nbytes, l2), l2, world),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"one whole {wl.n}x{wl.k} GEMV per step on {cores} threads"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_profile(args):
    """A few eager calls of one workload, for ncu captures (no timing)."""
    import torch

    import block_quantized_matmul_quant_b200 as kq

    kq.lib()
    wl = synth.WORKLOADS[args.profile]
    w, x, ids = synth.make_inputs(wl)
    wd = torch.from_numpy(w).cuda()
    xd = _x_tensor(torch, x, wl.x_dtype).cuda()
    ydt = torch.float32 if wl.y_dtype == "f32" else torch.bfloat16
    if wl.kind == "moe":
        idd = torch.from_numpy(ids).cuda()
        y = torch.empty((wl.m, wl.top_k, wl.n), dtype=ydt, device="cuda")
        for _ in range(args.profile_calls):
            kq.matmul_id(wd, wl.codec, xd, idd, out=y)
    else:
        y = torch.empty((wl.m, wl.n), dtype=ydt, device="cuda")
        indep = args.profile_mode == "independent"
        for _ in range(args.profile_calls):
            kq.matmul(wd, wl.codec, xd, out=y, const_weights=not indep, independent=indep)
    torch.cuda.synchronize()
    status = kq.device_status()
    if status != 0:  # a kernel reported a bad input or a wait that gave up
        raise SystemExit(f"device status {status} after {wl.name}")
    print(json.dumps({"profiled": wl.name, "calls": args.profile_calls}))


def run_tq1_sweep(torch, kq, l2):
    """TQ1_G128 5120 x 17408 (bf16 activations): the bandwidth kernel (one
    launch per two rows, up to 16 rows here) against the tensor-core kernel
    over the activation-row count."""
    dense = synth.Workload("sweep_tq1", "gemm", synth.TQ1_G128, 5120, 17408, 1, "bf16", "f32")
    w, _, _ = synth.make_inputs(dense)
    wd = torch.from_numpy(w).cuda()
    pool = [wd.clone() for _ in range(pool_size(w.nbytes, l2))]
    r = np.random.Generator(np.random.PCG64(2))
    for m in (1, 2, 4, 5, 6, 8, 12, 16, 32, 64, 128, 256, 512):
        x = torch.from_numpy(synth.gen_x(m, dense.k, "bf16", r)).to(torch.bfloat16).cuda()
        y = torch.empty((m, dense.n), device="cuda")
        line = {"sweep": "dense_tq1_g128_5120x17408", "m": m, "pool": len(pool)}
        for name, path in (("gemv", kq.PATH_GEMV), ("gemm", kq.PATH_GEMM)):
            if name == "gemv" and m > 16:
                continue
            def fn():
                for wi in pool:
                    kq.matmul(wi, synth.TQ1_G128, x, out=y, path=path, const_weights=True)
            line[name + "_us"] = round(time_graph(torch, fn, 5, 3, None) * 1e3 / (5 * len(pool)), 2)
        print(json.dumps(line), flush=True)
    del pool, wd
    torch.cuda.empty_cache()


def run_q8_0_sweep(torch, kq, l2):
    """Q8_0 and Q2_K, 4096 x 4096 (bf16 activations): the plain kernel
    against the tensor-core kernel over the activation-row count."""
    for codec, cname in ((synth.Q8_0, "q8_0"), (synth.Q2_K, "q2_k")):
        dense = synth.Workload("sweep_" + cname, "gemm", codec, 4096, 4096, 1, "bf16", "f32")
        w, _, _ = synth.make_inputs(dense)
        wd = torch.from_numpy(w).cuda()
        pool = [wd.clone() for _ in range(pool_size(w.nbytes, l2))]
        r = np.random.Generator(np.random.PCG64(3))
        for m in (1, 2, 3, 4, 8, 16, 32, 64, 128, 512):
            x = torch.from_numpy(synth.gen_x(m, dense.k, "bf16", r)).to(torch.bfloat16).cuda()
            y = torch.empty((m, dense.n), device="cuda")
            line = {"sweep": f"dense_{cname}_4096x4096", "m": m, "pool": len(pool)}
            for name, path in (("plain", kq.PATH_SIMPLE), ("gemm", kq.PATH_GEMM)):
                def fn():
                    for wi in pool:
                        kq.matmul(wi, codec, x, out=y, path=path, const_weights=True)
                line[name + "_us"] = round(time_graph(torch, fn, 5, 3, None) * 1e3 / (5 * len(pool)), 2)
            print(json.dumps(line), flush=True)
        del pool, wd
        torch.cuda.empty_cache()


def run_id_codecs_sweep(torch, kq, l2):
    """Expert-indexed Q2_K, Q8_0 and Q5_K (64 experts of 1408 x 2048, top-6,
    bf16 activations): the plain grouped kernel against the grouped
    tensor-core GEMM over the token count."""
    for codec, cname in ((synth.Q2_K, "q2_k"), (synth.Q8_0, "q8_0"), (synth.Q5_K, "q5_k")):
        for t in (1, 4, 8, 32, 128):
            wl = synth.Workload("sweep_id", "moe", codec, 1408, 2048, t, "bf16", "f32", n_experts=64, top_k=6)
            w, x, ids = synth.make_inputs(wl)
            wd = torch.from_numpy(w).cuda()
            pool = [wd.clone() for _ in range(max(4, -(-4 * l2 // w.nbytes)))]
            xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
            idd = torch.from_numpy(ids).cuda()
            y = torch.empty((t, 6, 1408), device="cuda")
            ws = torch.empty(kq.matmul_id_workspace_bytes(t, 6, 64), dtype=torch.uint8, device="cuda")
            line = {"sweep": f"moe_{cname}_e64_1408x2048_top6", "tokens": t, "pool": len(pool)}
            for name, path in (("plain", kq.PATH_SIMPLE), ("gemm", kq.PATH_GEMM)):
                def fn():
                    for wi in pool:
                        kq.matmul_id(wi, codec, xd, idd, out=y, workspace=ws, path=path)
                line[name + "_us"] = round(time_graph(torch, fn, 5, 3, None) * 1e3 / (5 * len(pool)), 2)
            print(json.dumps(line), flush=True)
            del pool, wd
            torch.cuda.empty_cache()
        # the fused GLU at 32 tokens (two grouped GEMMs over one grouping)
        # beside one expert product on the same routing
        wl = synth.Workload("sweep_id", "moe", codec, 1408, 2048, 32, "bf16", "f32", n_experts=64, top_k=6)
        line = {"sweep": f"moe_{cname}_e64_1408x2048_top6_glu", "tokens": 32}
        for glu in (False, True):
            st = PoolStep(torch, kq, wl, l2, glu=glu)
            line["glu_us" if glu else "product_us"] = round(time_graph(torch, st.run, 5, 3, None) * 1e3 / (5 * st.pool), 2)
            del st
            torch.cuda.empty_cache()
        print(json.dumps(line), flush=True)


def run_sweep(args):
    """Dispatch evidence: per-call time of the bandwidth kernel against the
    tensor-core kernel over the activation-row count (dense Q4_K product,
    11008 x 4096; dense TQ1_G128, 5120 x 17408) and the token count (MoE, 64
    experts of 1408 x 2048, top-6), bf16 activations, each call on its own
    weight copy of a pool larger than 4x L2.  One JSON line per point
    (`--sweep tq1`: the TQ1 points only)."""
    import torch

    import block_quantized_matmul_quant_b200 as kq

    kq.lib()
    l2 = l2_bytes(0)
    if args.sweep in ("q8_0", "id_codecs"):
        (run_q8_0_sweep if args.sweep == "q8_0" else run_id_codecs_sweep)(torch, kq, l2)
        status = kq.device_status()
        if status != 0:
            raise SystemExit(f"device status {status} after the sweep")
        return
    run_tq1_sweep(torch, kq, l2)
    if args.sweep == "tq1":
        status = kq.device_status()
        if status != 0:
            raise SystemExit(f"device status {status} after the sweep")
        return
    dense = synth.Workload("sweep_dense", "gemm", synth.Q4_K, 11008, 4096, 1, "bf16", "f32")
    w, _, _ = synth.make_inputs(dense)
    wd = torch.from_numpy(w).cuda()
    pool = [wd.clone() for _ in range(pool_size(w.nbytes, l2))]
    r = np.random.Generator(np.random.PCG64(1))
    for m in (1, 2, 4, 8, 9, 12, 16, 24, 32, 48, 64):
        x = torch.from_numpy(synth.gen_x(m, dense.k, "bf16", r)).to(torch.bfloat16).cuda()
        y = torch.empty((m, dense.n), device="cuda")
        line = {"sweep": "dense_q4_k_11008x4096", "m": m, "pool": len(pool)}
        for name, path in (("gemv", kq.PATH_GEMV), ("gemm", kq.PATH_GEMM), ("gemv_tc", kq.PATH_GEMV_TC)):
            def fn():
                for wi in pool:
                    kq.matmul(wi, synth.Q4_K, x, out=y, path=path, const_weights=True)
            line[name + "_us"] = round(time_graph(torch, fn, 5, 3, None) * 1e3 / (5 * len(pool)), 2)
        print(json.dumps(line), flush=True)
    del pool, wd
    torch.cuda.empty_cache()
    for t in (8, 16, 32, 64, 128, 256, 512):
        wl = synth.Workload("sweep_moe", "moe", synth.Q4_K, 1408, 2048, t, "bf16", "f32", n_experts=64, top_k=6)
        w, x, ids = synth.make_inputs(wl)
        wd = torch.from_numpy(w).cuda()
        pool = [wd.clone() for _ in range(pool_size(w.nbytes, l2))]
        xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
        idd = torch.from_numpy(ids).cuda()
        y = torch.empty((t, 6, 1408), device="cuda")
        ws = torch.empty(kq.matmul_id_workspace_bytes(t, 6, 64), dtype=torch.uint8, device="cuda")
        line = {"sweep": "moe_q4_k_e64_1408x2048_top6", "tokens": t, "pairs_per_expert": round(6 * t / 64, 2),
                "pool": len(pool)}
        for name, path in (("gemv", kq.PATH_GEMV), ("gemm", kq.PATH_GEMM), ("gemv_tc", kq.PATH_GEMV_TC)):
            def fn():
                for wi in pool:
                    kq.matmul_id(wi, synth.Q4_K, xd, idd, out=y, workspace=ws, path=path)
            line[name + "_us"] = round(time_graph(torch, fn, 5, 3, None) * 1e3 / (5 * len(pool)), 2)
        print(json.dumps(line), flush=True)
        del pool, wd
        torch.cuda.empty_cache()
    status = kq.device_status()
    if status != 0:
        raise SystemExit(f"device status {status} after the sweep")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="kq", choices=["kq", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile", default=None, choices=sorted(synth.WORKLOADS),
                    help="run a few eager calls of one workload (for ncu) and exit")
    ap.add_argument("--profile-calls", type=int, default=3)
    ap.add_argument("--profile-mode", default="independent", choices=["independent", "const"],
                    help="GEMV call ordering in --profile (the headline step uses independent calls)")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads' numbers (prefill GEMM, MoE, TQ1, Q8_0)")
    ap.add_argument("--sweep", default=None, choices=["dispatch", "tq1", "q8_0", "id_codecs"],
                    help="print the dispatch sweep (bandwidth vs tensor-core kernel) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.sweep:
        run_sweep(args)
    elif args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
