"""Host-side pieces of bench.py (CPU): the DRAM traffic it takes from a
profile summary only while the kernel source is unchanged, and the summary
of the clocks sampled during the timed region."""
import hashlib

import bench


def _profile(tmp_path, src_text, recorded_hash, traffic):
    src = tmp_path / "kernel.cu"
    src.write_text(src_text)
    prof = tmp_path / "prof.md"
    prof.write_text(f"# capture\n\nsource_sha256_16: {recorded_hash}\n"
                    f"dram_bytes_per_launch_fullsize: {traffic}\n")
    return str(src), str(prof)


def test_traffic_only_for_the_captured_source(tmp_path):
    text = "__global__ void k() {}\n"
    h = hashlib.sha256(text.encode()).hexdigest()[:16]
    src, prof = _profile(tmp_path, text, h, 231358208)
    assert bench.traffic_from_profile(src, prof) == 231358208.0
    # the kernel changed since the capture: no traffic figure
    src, prof = _profile(tmp_path, text + "// changed\n", h, 231358208)
    assert bench.traffic_from_profile(src, prof) is None
    # no summary at all
    assert bench.traffic_from_profile(src, str(tmp_path / "missing.md")) is None


def test_clock_summary(tmp_path):
    c = bench.Clocks(0)
    c.path = str(tmp_path / "clocks.csv")
    c.proc = object()  # as if nvidia-smi had run
    rows = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    (tmp_path / "clocks.csv").write_text("\n".join(rows) + "\n")
    s = c.summary()
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert not (tmp_path / "clocks.csv").exists()  # the sample file is removed


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one
    JSON line with the contract keys (CPU only; tiny workload, one step)."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_fp32_L4k", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny_fp32_L4k"
