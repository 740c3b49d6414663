"""bench.py's host-side roofline bookkeeping (CPU): the roofline entry, the per-class table,
the recorded DRAM traffic that follows the kernel sources, and the peak fallback."""
import importlib.util
import json
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "measured"}


def test_summarize_tensor_bound():
    b = _bench()
    kernels = {"gemm": {"launches": 8, "ms": 20.0, "flops": 2.8e13, "bytes": 4e9},
               "mhc": {"launches": 4, "ms": 5.0, "flops": 0.0, "bytes": 1.5e10}}
    roof, table = b.summarize(kernels, steps=2, peaks=PEAKS)
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s" and roof["kernel"] == "gemm"
    assert roof["achieved"] == pytest.approx(2.8e13 / 0.020 / 1e12, rel=1e-6)      # 1400 TFLOP/s
    assert roof["peak"] == 1400.0 and roof["frac"] == pytest.approx(1.0, abs=1e-4)   # sustained peak
    assert roof["algorithmic_per_launch"] == pytest.approx(2.8e13 / 8)
    assert roof["launches"] == 8 and roof["ms_per_launch"] == pytest.approx(2.5)
    assert table["gemm"]["launches"] == 4 and table["gemm"]["ms_per_step"] == pytest.approx(10.0)
    assert table["mhc"]["gbs"] == pytest.approx(1.5e10 / 0.005 / 1e9, rel=1e-3)
    assert sum(v["share"] for v in table.values()) == pytest.approx(1.0, abs=1e-3)
    roof_burst, _ = b.summarize(kernels, steps=2, peaks=PEAKS, sustained=False)
    assert roof_burst["peak"] == 1600.0


def test_summarize_hbm_bound():
    b = _bench()
    kernels = {"attention": {"launches": 28, "ms": 19.5, "flops": 5e11, "bytes": 1.2e11},
               "gemm": {"launches": 224, "ms": 7.7, "flops": 1.4e12, "bytes": 2.1e10}}
    roof, _ = b.summarize(kernels, steps=1, peaks=PEAKS, tensor_bound=())
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and roof["kernel"] == "attention"
    assert roof["achieved"] == pytest.approx(1.2e11 / 0.0195 / 1e9, rel=1e-4)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6000.0, rel=1e-3)
    assert roof["traffic"] is None                     # only the GEMM carries a recorded capture


def _fake_root(tmp_path):
    csrc = tmp_path / "looped_hybrid_attention_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in ("gemm_tc.cu", "gemm_tc2.cu", "tc_common.cuh"):
        shutil.copy(os.path.join(ROOT, "looped_hybrid_attention_b200", "csrc", n), csrc / n)
    (tmp_path / "profiles").mkdir()
    shutil.copy(os.path.join(ROOT, "profiles", "gemm_traffic.json"), tmp_path / "profiles" / "gemm_traffic.json")
    return csrc


def test_recorded_traffic_follows_the_sources(tmp_path):
    b = _bench()
    csrc = _fake_root(tmp_path)
    b.ROOT = str(tmp_path)
    import hashlib
    src = b"".join((csrc / n).read_bytes() for n in ("gemm_tc.cu", "gemm_tc2.cu", "tc_common.cuh"))
    rec = json.loads((tmp_path / "profiles" / "gemm_traffic.json").read_text())
    rec["kernel_sources_sha256"] = hashlib.sha256(src).hexdigest()
    (tmp_path / "profiles" / "gemm_traffic.json").write_text(json.dumps(rec))
    assert b.recorded_traffic("gemm") == rec["traffic_bytes_per_launch_step_average"]
    with open(csrc / "tc_common.cuh", "a") as f:        # a changed kernel source voids the capture
        f.write("\n// changed\n")
    assert b.recorded_traffic("gemm") is None
    assert b.recorded_traffic("attention") is None      # no capture recorded for it


def test_recorded_traffic_is_launch_weighted():
    with open(os.path.join(ROOT, "profiles", "gemm_traffic.json")) as f:
        rec = json.load(f)
    n = sum(rec["launches_per_step"].values())
    tot = sum(rec["launches_per_step"][k] * (s["dram_read"] + s["dram_write"]) for k, s in rec["shapes"].items())
    assert n == 224                                     # GEMM launches in one prefill step
    assert rec["traffic_bytes_per_launch_step_average"] == pytest.approx(tot / n, rel=1e-9)


def test_peaks_fallback(tmp_path):
    b = _bench()
    b.ROOT = str(tmp_path)                              # no MEASURED_PEAKS.json there
    p = b.load_peaks()
    assert p["source"] == "fallback"
    assert p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
