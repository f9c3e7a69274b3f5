"""Host logic of bench.py: the measured DRAM traffic it reports counts only
while the kernel sources' code is the code that was captured, and a comment
or whitespace edit does not change that."""
import json

import bench

SRC = {
    "a.cu": 'int f(int x) {  // doubles x\n    return 2 * x; /* fast */\n}\nconst char *u = "http://x";\n',
}


def _reader(files):
    return lambda name: files[name]


def test_strip_comments_keeps_code_and_string_literals():
    out = bench.strip_comments(SRC["a.cu"])
    assert "doubles" not in out and "fast" not in out
    assert "return2*x;" in out
    assert '"http://x"' in out  # a // inside a string is code


def test_hash_ignores_comments_and_whitespace_but_not_code():
    h0 = bench.kernel_source_hash(["a.cu"], _reader(SRC))
    commented = {"a.cu": "// header\n" + SRC["a.cu"].replace("// doubles x", "/* twice */")}
    spaced = {"a.cu": SRC["a.cu"].replace("return 2 * x;", "return   2*x ;")}
    changed = {"a.cu": SRC["a.cu"].replace("2 * x", "3 * x")}
    assert bench.kernel_source_hash(["a.cu"], _reader(commented)) == h0
    assert bench.kernel_source_hash(["a.cu"], _reader(spaced)) == h0
    assert bench.kernel_source_hash(["a.cu"], _reader(changed)) != h0


def test_measured_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    names = ["kq_gemv.cu", "kq_ptx.cuh"]
    current = bench.kernel_source_hash(names)
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({
        "same": {"source_hash": current, "dram_bytes_per_launch": 1234},
        "stale": {"source_hash": "0" * 16, "dram_bytes_per_launch": 99},
    }))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.measured_traffic("same", names) == 1234.0
    assert bench.measured_traffic("stale", names) is None
    assert bench.measured_traffic("missing", names) is None


def test_committed_traffic_entries_are_well_formed():
    with open(bench.TRAFFIC_FILE) as fh:
        t = json.load(fh)
    for key, e in t.items():
        if key.startswith("_"):
            continue
        assert len(e["source_hash"]) == 16
        assert e["dram_bytes_per_launch"] > 0


def test_reference_arm_prints_one_contract_line(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class A:
        workload = "q4_k_gemv_4096x4096"
        steps, warmup = 1, 0

    bench.run_reference(A())
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    r = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in r
    assert r["impl"] == "reference" and r["value"] > 0 and r["higher_is_better"] is True
    assert r["config"]["workload"] == "q4_k_gemv_4096x4096"
    # the same config object the GPU arm prints for this workload and world size
    wl = bench.synth.WORKLOADS["q4_k_gemv_4096x4096"]
    wbytes = wl.weight_bytes()
    l2 = bench.l2_bytes()
    assert r["config"] == bench.headline_config(wl, wbytes, bench.pool_size(wbytes, l2), l2, 1)
    assert r["config"]["pool_matrices_per_step"] == 57 or l2 != bench.B200_L2_BYTES
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1 and cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": r["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


PEAKS = {"hbm_gbs": 6468.0, "bf16_tflops": 1644.2, "bf16_tflops_sustained": 1385.2}


def test_secondary_entry_figures():
    import synth

    g = bench.secondary_entry(synth.WORKLOADS["q4_k_gemm_512x11008x4096"], 67.2, 0, 0, PEAKS)
    tf = 2 * 512 * 11008 * 4096 / 67.2e-6 / 1e12
    assert g["TFLOP/s"] == round(tf, 1)
    assert g["frac_burst"] == round(tf / 1644.2, 4) and g["frac_sustained"] == round(tf / 1385.2, 4)

    wl = synth.WORKLOADS["moe_q4_k_e64_1408x2048_t32_top6"]
    wbytes = 64 * 1408 * (2048 // 256) * 144
    m = bench.secondary_entry(wl, 83.0, wbytes, 63, PEAKS)
    moved = 63 * 1408 * 8 * 144 + 32 * 2048 * 2 + 32 * 6 * 1408 * 4
    assert moved == 103_399_424
    assert m["GB/s"] == round(moved / 83.0e-6 / 1e9, 1)
    assert m["gate_up_pair_us"] == 166.0 and m["tokens/s"] == round(32 / 83.0e-6, 1)

    v = bench.secondary_entry(synth.WORKLOADS["tq1_g128_gemv_5120x17408"], 17.9, 19_496_960, 0, PEAKS)
    assert v["weight GB/s"] == round(19_496_960 / 17.9e-6 / 1e9, 1)
    assert v["frac_hbm"] == round(19_496_960 / 17.9e-6 / 1e9 / 6468.0, 4)


def test_secondary_metrics_call_site(monkeypatch):
    """The timed loop's bookkeeping (time per call from the graph time) with
    the GPU parts replaced by stand-ins."""
    import types

    class FakeStep:
        def __init__(self, torch, kq, wl, l2, glu=False):
            self.wl, self.pool, self.wbytes = wl, 8, 1_000_000
            if wl.kind == "moe":
                self.hit_experts = 63

        def run(self):
            pass

    monkeypatch.setattr(bench, "PoolStep", FakeStep)
    monkeypatch.setattr(bench, "time_graph", lambda torch, fn, steps, warmup, pg: 0.4)  # ms per 5 steps
    fake_torch = types.SimpleNamespace(cuda=types.SimpleNamespace(empty_cache=lambda: None))
    out = bench.secondary_metrics(fake_torch, None, 0, PEAKS)
    assert set(out) == {"q4_k_gemm_512x11008x4096", "moe_q4_k_e64_1408x2048_t32_top6",
                        "tq1_g128_gemv_5120x17408", "tq1_g128_gemm_512x5120x17408", "q8_0_gemv_256x1024",
                        "moe_q4_k_e64_1408x2048_t32_top6_glu"}
    glu = out["moe_q4_k_e64_1408x2048_t32_top6_glu"]
    assert glu["vs_gate_up_pair_us"] == out["moe_q4_k_e64_1408x2048_t32_top6"]["gate_up_pair_us"]
    us = 0.4 * 1e3 / (5 * 8)
    assert out["q8_0_gemv_256x1024"]["us_per_call"] == round(us, 3)
    assert out["moe_q4_k_e64_1408x2048_t32_top6"]["hit_experts"] == 63


def test_clock_summary_reads_sampled_lines():
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1900, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 800.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 1, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = cs.summary()
    assert s["sm_mhz"] == 1950 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    cs.lines = ["0, 1965, 1965, 700, 0x8, Active, Not Active, Not Active, Not Active"]
    assert cs.summary()["reasons"] == ["hw_slowdown"]
    cs.lines = []
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}


def test_clocks_rejected_rules():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert not bench.clocks_rejected(ok)
    assert not bench.clocks_rejected({"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    assert bench.clocks_rejected({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown"]})
    assert bench.clocks_rejected({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0,
                                  "reasons": ["sw_power_cap", "sw_thermal_slowdown"]})
    assert bench.clocks_rejected({"sm_mhz": 1000.0, "sm_max_mhz": 1965.0, "reasons": []})   # stuck low
    assert not bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]})


def test_clock_summary_skips_idle_samples():
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 345, 1965, 120.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active",
        "0, 1965, 1965, 900.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
    ]
    s = cs.summary()
    assert s["samples"] == 1 and s["sm_mhz"] == 1965
    assert not bench.clocks_rejected(s)


def test_clock_summary_with_idle_samples_only():
    cs = bench.ClockSampler(0)
    cs.lines = ["0, 120, 1965, 100.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active"] * 3
    s = cs.summary()
    assert s["idle_samples_only"] is True and s["sm_mhz"] == 120 and s["samples"] == 3
    assert not bench.clocks_rejected(s)   # idle clocks say nothing about a lock
