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
