"""Host-side logic of bench.py that needs no GPU: the clock summary (which
nvidia-smi samples count), the timing statistics and the source hash that
keys the stored ncu traffic."""

import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _line(mhz, active, power=300.0, cap="Not Active"):
    return (f"0, {mhz}, 1965, {power}, 0x{active:016x}, Not Active, Not Active, "
            f"Not Active, {cap}")


def test_clock_summary_keeps_loaded_samples_inside_the_window():
    c = bench.ClockSampler(0)
    c.lines = [
        (0.5, _line(1965, 0x1)),               # before the window
        (1.1, _line(120, 0x1)),                # in the window but idle
        (1.2, _line(1800, 0x0, power=410.0)),
        (1.3, _line(1900, 0x4, cap="Active")),
        (1.4, _line(1700, 0x0)),
        (2.5, _line(1000, 0x0)),               # after the window
    ]
    c.t0, c.t1 = 1.0, 2.0
    s = c.summary()
    assert s["samples"] == 3 and s["idle_samples"] == 1
    assert s["sm_mhz"] == 1800.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["power_w_max"] == 410.0


def test_clock_summary_without_loaded_samples_says_so():
    c = bench.ClockSampler(0)
    c.lines = [(1.5, _line(120, 0x1)), (1.6, "garbled line")]
    c.t0, c.t1 = 1.0, 2.0
    s = c.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and "note" in s
    c.lines = []
    assert c.summary() is None


def test_dist_stats():
    xs = [5.0, 1.0, 3.0, 2.0, 4.0, 10.0, 6.0, 7.0, 8.0, 9.0]
    s = bench.dist_stats(xs)
    assert s == {"median": 5.5, "min": 1.0, "p90": 9.0}
    assert bench.dist_stats([2.0]) == {"median": 2.0, "min": 2.0, "p90": 2.0}


def test_decode_sources_hash_covers_the_decode_sources_only(tmp_path, monkeypatch):
    # the hash changes with a decode source and ignores the GEMM source
    import shutil
    csrc = os.path.join(ROOT, "mla_latent_kv_32_b200", "csrc")
    fake = tmp_path / "mla_latent_kv_32_b200" / "csrc"
    fake.mkdir(parents=True)
    for n in ("decode_pair.cu", "decode_simt.cu", "plan.h", "common.cuh", "gemm_tc.cu"):
        shutil.copy(os.path.join(csrc, n), fake / n)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.decode_sources_hash()
    assert h0 == bench.decode_sources_hash() and len(h0) == 16
    (fake / "gemm_tc.cu").write_text("// changed\n")
    assert bench.decode_sources_hash() == h0
    (fake / "decode_pair.cu").write_text((fake / "decode_pair.cu").read_text() + "\n")
    assert bench.decode_sources_hash() != h0


def test_stored_traffic_figures_are_plausible():
    # every stored ncu traffic figure for v3 lies between the algorithmic
    # bytes of its cache format and 1.1x them plus the outputs written (the
    # decode reads each cache row once from HBM), and the current decode
    # sources have a bf16 figure
    row = {"bf16": bench.ROW_BYTES, "fp8": bench.FP8_TOKEN_BYTES}
    out_bytes = 64 * 128 * (512 * 2 + 4)
    v3 = [(cache, t) for (h, w, cache), t in bench.TRAFFIC.items() if w == "v3"]
    assert v3
    for cache, t in v3:
        cache_bytes = 64 * 4096 * row[cache]
        assert cache_bytes <= t <= math.ceil(1.1 * cache_bytes) + out_bytes
    assert (bench.decode_sources_hash(), "v3", "bf16") in bench.TRAFFIC


def test_reference_arm_line_on_the_host():
    # `bench.py --impl reference` times the oracle on the host cores and
    # prints one JSON line in the contract's shape (its own impl tag, the
    # oracle as cpu_baseline, an e2e object with no host<->device bytes)
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                         timeout=300, cwd=bench.ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
