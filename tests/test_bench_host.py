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
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1 and cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": r["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
