"""Host-side pieces of bench.py that its reported figures rest on (CPU only):
the algorithmic bytes behind `roofline.achieved`, the rule that a recorded
DRAM-traffic figure is reported only for the sources it was captured from,
and the JSON line of the reference arm (the oracle on the host cores)."""
import importlib.util
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_cast_algorithmic_bytes():
    """Per value of the bf16 8192 x 8192 sweep: 2 bytes read, the code's
    bits / 8 and 1/32 of an E8M0 scale byte written."""
    b = load_bench()
    n = 8192 * 8192
    assert b.cast_alg_bytes("e4m3") == 2 * n + n + n // 32 == 203_423_744
    assert b.cast_alg_bytes("e5m2") == b.cast_alg_bytes("int8") == b.cast_alg_bytes("e4m3")
    assert b.cast_alg_bytes("e2m3") == b.cast_alg_bytes("e3m2") == 2 * n + 3 * n // 4 + n // 32 == 186_646_528
    assert b.cast_alg_bytes("e2m1") == 2 * n + n // 2 + n // 32 == 169_869_312
    assert b.cast_alg_bytes("e4m3", 16384, 4096, in_bytes=4) == 16384 * 4096 * (4 + 1) + 16384 * 4096 // 32


def test_traffic_reported_only_for_the_captured_sources(monkeypatch):
    b = load_bench()
    for kernel, (names, sha, table) in b.MEASURED_TRAFFIC.items():
        workload = next(iter(table))
        monkeypatch.setattr(b, "sources_sha256", lambda names, sha=sha: sha)
        assert b.measured_traffic(kernel, workload) == table[workload]
        assert b.measured_traffic(kernel, "no_such_workload") is None
        monkeypatch.setattr(b, "sources_sha256", lambda names: "0" * 64)
        assert b.measured_traffic(kernel, workload) is None


def test_recorded_cast_traffic_shows_no_rereads():
    """Every recorded row-cast launch moved at most the algorithmic bytes
    (plus a little): reads of the input happen once.  Writes can fall short of
    the codes' bytes (the tail is still in L2 when the launch ends), never far."""
    b = load_bench()
    _, _, table = b.MEASURED_TRAFFIC["cast_rows"]
    for f in ("e4m3", "e5m2", "e2m3", "e3m2", "e2m1", "int8"):
        alg = b.cast_alg_bytes(f)
        assert 0.7 * alg < table[f"{f}_bf16_8192x8192"] <= 1.02 * alg, f


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3
    assert line["config"]["workload"] == "cast_sweep_bf16_8192x8192_6fmt"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
