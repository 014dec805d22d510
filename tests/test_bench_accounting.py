"""bench.py's algorithmic accounting on CPU: the per-kernel byte shares that
the dominant-kernel roofline divides by must add up to the path's bytes, and
the path's bytes and flops must follow their stated per-token-head forms."""
import dataclasses
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_deltanet_linear_chunked_b200 import workloads as wl  # noqa: E402

KERNELS = ("gdn_prep_kernel", "gdn_recur_kernel", "gdn_output_kernel")


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
@pytest.mark.parametrize("dims", [(112, 112), (64, 128), (128, 32)])
def test_kernel_shares_sum_to_the_path(mode, dims):
    w = dataclasses.replace(wl.stream_chunk(mode), Dk=dims[0], Dv=dims[1])
    assert sum(bench.kernel_algorithmic_bytes(k, w) for k in KERNELS) == bench.algorithmic_bytes(w)


def test_path_bytes_of_the_streaming_chunk():
    # q, k, v, out in bf16 (2 bytes), g and beta in fp32, one fp32 state in
    # and one out per head: 2640 x 20 token-heads at d = 112
    w = wl.stream_chunk("fwd")
    token_heads = 2640 * 20
    expect = token_heads * (4 * 112 * 2 + 8) + 2 * 20 * 112 * 112 * 4
    assert bench.algorithmic_bytes(w) == expect


def test_path_flops_forms():
    w = wl.stream_chunk("fwd")
    d, c = 112, 64
    assert bench.algorithmic_flops(w) == 2640 * 20 * (6 * d * d + 8 * c * d)
    assert bench.algorithmic_flops(w, True) == 2 * bench.algorithmic_flops(w)


@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_reference_arm_prints_one_contract_line(mode):
    """``bench.py --impl reference`` (the fp64 oracle on this host's cores)
    prints exactly one JSON line on the same metric, unit, direction and
    workload as the native arm, with its own cpu_baseline and an e2e that
    moves no bytes."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--mode", mode, "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["config"]["workload"] == ("stream_chunk_causal" if mode == "fwd"
                                       else "stream_chunk_bidir")
    assert (d["config"]["T"], d["config"]["Dk"], d["config"]["Dv"]) == (2640, 112, 112)
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["unit"] == d["unit"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_peaks_file_is_read_key_by_key(monkeypatch, tmp_path):
    """The roofline denominators: measured where the peaks file holds a
    positive number, the fallback elsewhere, and the source said truthfully;
    a missing or unreadable file means the fallback throughout."""
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = tmp_path / "MEASURED_PEAKS.json"
    assert bench.load_peaks() == (bench.FALLBACK_PEAKS, "fallback")           # absent
    full = {"hbm_gbs": 6547.2, "bf16_tflops": 1646.1, "bf16_tflops_sustained": 1391.6,
            "clocks": {"sm_mhz": 1965}}
    f.write_text(json.dumps(full))
    peaks, kind = bench.load_peaks()
    assert kind == "measured" and peaks == {k: full[k] for k in bench.FALLBACK_PEAKS}
    f.write_text(json.dumps({"hbm_gbs": "6547.2", "bf16_tflops": 1646.1}))
    peaks, kind = bench.load_peaks()
    assert peaks["hbm_gbs"] == 6547.2 and peaks["bf16_tflops"] == 1646.1
    assert peaks["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    assert kind == "measured, with fallback for bf16_tflops_sustained"
    for bad in ("{not json", "[1, 2]", json.dumps({"hbm_gbs": None, "bf16_tflops": -1})):
        f.write_text(bad)
        assert bench.load_peaks() == (bench.FALLBACK_PEAKS, "fallback"), bad


@pytest.mark.parametrize("mode,bound", [("fwd", "hbm"), ("bidir", "tensor")])
def test_roofline_object_arithmetic(mode, bound):
    """The roofline object on made-up kernel times: the causal chunk is bound
    by HBM and the bidirectional one by the tensor pipe; the dominant kernel
    is the longest; achieved is the path's work per launch over that
    kernel's time, the path figure the same work over the step."""
    w = wl.stream_chunk(mode)
    peaks = dict(bench.FALLBACK_PEAKS)
    kernels = {"gdn_prep_kernel": {"ms_per_launch": 0.03},
               "gdn_recur_kernel": {"ms_per_launch": 0.02},
               "gdn_output_kernel": {"ms_per_launch": 0.04}}
    r = bench.roofline_of(w, kernels, 0.1, peaks, "fallback", mode == "bidir")
    assert r["bound"] == bound and r["kernel"] == "gdn_output_kernel"
    if bound == "hbm":
        work, peak, unit = bench.algorithmic_bytes(w) / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        work, peak = bench.algorithmic_flops(w, True) / 1e12, peaks["bf16_tflops_sustained"]
        unit = "TFLOP/s"
    assert r["unit"] == unit and r["peak"] == peak
    assert r["achieved"] == pytest.approx(work / 0.04e-3)
    assert r["frac"] == pytest.approx(work / 0.04e-3 / peak)
    assert r["path"]["frac"] == pytest.approx(work / 0.1e-3 / peak)
    assert r["peak_source"].startswith("fallback")
    t_hbm, t_tc = bench.roofline_times(w, mode == "bidir", peaks)
    assert r["path"]["roofline_us"] == pytest.approx(1e6 * max(t_hbm, t_tc))


def test_clock_sampler_against_a_fake_nvml(monkeypatch):
    """The clock record of the JSON line, on a fake NVML: clocks sampled
    while the region runs, reason bits decoded by name (idle dropped), the
    median taken; and no NVML at all gives an empty record, not an error."""
    import time
    import types
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: ("gpu", i),
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: 1965,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x1 | 0x4,   # idle, sw_power_cap
    )
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0) as c:
        time.sleep(0.1)
    s = c.summary()
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] >= 5

    def no_nvml():
        raise RuntimeError("NVML unavailable")
    monkeypatch.setattr(fake, "nvmlInit", no_nvml)
    with bench.ClockSampler(0) as c:
        time.sleep(0.01)
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_recorded_traffic_only_while_the_source_matches(monkeypatch, tmp_path):
    """roofline.traffic comes from the committed ncu table only while the
    kernel's source still hashes to the value the capture was taken on;
    after any edit of that source it is null."""
    import hashlib
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# kernel  sha256  bytes\n" f"gdn_output_kernel {digest} 57273344\n"
        f"gdn_prep_kernel {'0' * 64} 1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", {"gdn_output_kernel": "k.cu",
                                                  "gdn_prep_kernel": "k.cu"})
    assert bench.recorded_traffic("gdn_output_kernel") == 57273344
    assert bench.recorded_traffic("gdn_prep_kernel") is None       # taken on another source
    assert bench.recorded_traffic("gdn_recur_kernel") is None      # no source known
    src.write_text("kernel v2\n")
    assert bench.recorded_traffic("gdn_output_kernel") is None      # source changed since

