"""Host-side logic of bench.py that needs no GPU: the clock-sample summary
behind the "clocks" key, the committed-traffic lookup behind roofline.traffic,
the peak lookup behind roofline.peak, and the GPU id used for sampling."""
import hashlib
import json
import os

import pytest

import bench

# index, clocks.sm, clocks.max.sm, power.draw, reasons.active, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
IDLE = "0, 1965, 1965, 140.10, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"
BUSY = "0, {mhz}, 1965, {w}, 0x0000000000000004, Not Active, Not Active, Not Active, {cap}"


def test_clock_summary_takes_the_loaded_samples():
    lines = [IDLE, BUSY.format(mhz=1800, w=950.0, cap="Active"), BUSY.format(mhz=1900, w=700.5, cap="Not Active"),
             BUSY.format(mhz=1700, w=990.0, cap="Active"), IDLE]
    c = bench.summarize_clock_samples(lines)
    assert c["sm_mhz"] == 1800.0            # median of the three loaded samples, not of all five
    assert c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 5 and c["samples_under_load"] == 3
    assert c["power_w_max"] == 990.0


def test_clock_summary_reports_every_throttle_reason_seen():
    row = "0, 1200, 1965, 800, 0x68, Active, Active, Active, Not Active"
    c = bench.summarize_clock_samples([row, BUSY.format(mhz=1965, w=900, cap="Not Active")])
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_skips_fields_that_are_not_numbers():
    lines = ["0, [N/A], 1965, 900, 0x0, Not Active, Not Active, Not Active, Not Active",
             "0, 1500, [N/A], [N/A], 0x0, Not Active, Not Active, Not Active, Not Active",
             BUSY.format(mhz=1950, w=905, cap="Not Active"),
             "garbage line"]
    c = bench.summarize_clock_samples(lines)
    assert c["samples"] == 3                 # the short line is not a sample
    assert c["samples_under_load"] == 1      # only the row with both a clock and a power draw
    assert c["sm_mhz"] == 1950.0
    assert c["sm_max_mhz"] == 1965.0


def test_clock_summary_without_load_or_rows():
    c = bench.summarize_clock_samples([IDLE, IDLE.replace("1965, 1965", "1500, 1965")])
    assert c["samples_under_load"] == 0 and c["sm_mhz"] == (1965.0 + 1500.0) / 2
    assert bench.summarize_clock_samples([]) is None


def test_traffic_record_follows_the_kernel_source():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for kernel, per_workload in rec.items():
        if not isinstance(per_workload, dict) or kernel not in bench.DOMINANT_SOURCES:
            continue
        src = os.path.join(bench.ROOT, "shared_prefix_kv_fca_b200", "csrc", bench.DOMINANT_SOURCES[kernel])
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()[:16]
        for workload, ent in per_workload.items():
            got = bench.traffic_record(kernel, workload)
            if ent.get("source_sha256_16") == digest:
                assert got == float(ent["dram_bytes_per_launch"])
            else:
                assert got is None          # captured on another version of the kernel
    assert bench.traffic_record("suffix", "no such workload") is None
    assert bench.traffic_record("no such kernel", "llama8b") is None


def test_traffic_record_is_null_once_the_source_changes(monkeypatch):
    # the suffix entry read against another file's digest: as if the kernel had changed
    monkeypatch.setitem(bench.DOMINANT_SOURCES, "suffix", "fca_api.cu")
    assert bench.traffic_record("suffix", "llama8b") is None


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6549.1, "bf16_tflops": 1590.0}))
    assert bench.peaks() == (6549.1, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.peaks() == (bench.FALLBACK_HBM_GBS, "fallback")


@pytest.mark.parametrize("vis,local,want", [(None, 0, "0"), (None, 3, "3"), ("4,5", 1, "5"), ("GPU-abc", 0, "GPU-abc"),
                                            ("2", 1, "1")])
def test_gpu_id_for(monkeypatch, vis, local, want):
    if vis is None:
        monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    else:
        monkeypatch.setenv("CUDA_VISIBLE_DEVICES", vis)
    assert bench.gpu_id_for(local) == want


def test_prefix_flops_counts_each_shared_token_once_per_query_head():
    # two requests whose groups cover 3 and 1 blocks of 16 tokens; 8 query
    # heads of head_dim 128: 4 x 128 flops per (query head, key)
    assert bench.prefix_flops([3, 1], 16, 8, 128) == (3 + 1) * 16 * 8 * 4 * 128
    assert bench.prefix_flops([0, 0], 16, 8, 128) == 0


def test_prefix_roofline_fractions():
    r = bench.prefix_roofline(prefix_bytes=2_000_000_000, flops=4_000_000_000_000, prefix_ms=1.0, hbm_gbs=4000.0,
                              tflops_burst=8000.0, tflops_sustained=5000.0, peak_kind="measured",
                              tensor_pipe_pct=12.5)
    assert abs(r["achieved_gbs"] - 2000.0) < 1e-9 and abs(r["frac_hbm"] - 0.5) < 1e-12
    assert abs(r["achieved_tflops"] - 4000.0) < 1e-9
    assert abs(r["frac_tensor_burst"] - 0.5) < 1e-12 and abs(r["frac_tensor_sustained"] - 0.8) < 1e-12
    assert r["tensor_pipe_pct"] == 12.5 and r["us"] == 1000.0
    # no grouped pass (flat plan, or no group): no roofline
    assert bench.prefix_roofline(0, 0, 1.0, 1.0, 1.0, 1.0, "x") is None
    assert bench.prefix_roofline(10, 10, None, 1.0, 1.0, 1.0, "x") is None
