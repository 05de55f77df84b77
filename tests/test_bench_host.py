"""Host-side logic of bench.py (no GPU): the roofline denominators and the
measured-traffic table keyed by a hash of the kernel's sources."""
import json
import os

import pytest

import bench


def _root(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    return tmp_path


def test_peaks_fallback_without_file(tmp_path, monkeypatch):
    _root(tmp_path, monkeypatch)
    peaks, src = bench.load_peaks()
    assert src == "fallback"
    assert peaks == bench.FALLBACK_PEAKS


def test_peaks_from_file_and_partial_file(tmp_path, monkeypatch):
    root = _root(tmp_path, monkeypatch)
    full = {"hbm_gbs": 6452.8, "bf16_tflops": 1662.0, "bf16_tflops_sustained": 1383.8, "note": "x"}
    (root / "MEASURED_PEAKS.json").write_text(json.dumps(full))
    peaks, src = bench.load_peaks()
    assert src == "measured"
    assert peaks["bf16_tflops"] == 1662.0 and peaks["hbm_gbs"] == 6452.8
    (root / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1700}))
    peaks, src = bench.load_peaks()
    assert src == "measured (partly fallback)"
    assert peaks["bf16_tflops"] == 1700.0
    assert peaks["hbm_gbs"] == bench.FALLBACK_PEAKS["hbm_gbs"]
    (root / "MEASURED_PEAKS.json").write_text("not json")
    assert bench.load_peaks()[1] == "fallback"


@pytest.mark.parametrize("region_ms,sustained", [(46.0, False), (249.9, False), (250.0, True), (554.0, True)])
def test_tensor_peak_by_region(region_ms, sustained):
    peaks = {"hbm_gbs": 1.0, "bf16_tflops": 1662.0, "bf16_tflops_sustained": 1383.8}
    peak, name = bench.tensor_peak(peaks, region_ms)
    assert peak == (1383.8 if sustained else 1662.0)
    assert ("sustained" in name) == sustained


def test_traffic_only_while_sources_unchanged(tmp_path, monkeypatch):
    root = _root(tmp_path, monkeypatch)
    srcs = ["a.cu", "b.cuh"]
    (root / "a.cu").write_text("kernel a")
    (root / "b.cuh").write_text("header b")
    table = {"gemm1:mixtral": {"bytes_per_launch": 123, "sources": srcs,
                               "sources_sha256_16": bench.sources_hash(srcs)}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(table))
    assert bench.traffic_for("gemm1", "mixtral") == 123
    assert bench.traffic_for("gemm1", "qwen3_skew") is None
    (root / "b.cuh").write_text("header b, edited")
    assert bench.traffic_for("gemm1", "mixtral") is None
    os.remove(root / "a.cu")
    assert bench.traffic_for("gemm1", "mixtral") is None


def test_traffic_entry_without_sources_is_ignored(tmp_path, monkeypatch):
    root = _root(tmp_path, monkeypatch)
    (root / "profiles" / "traffic.json").write_text(json.dumps({"gemm1:mixtral": {"bytes_per_launch": 1}}))
    assert bench.traffic_for("gemm1", "mixtral") is None


def test_gpus_flag_relaunches_as_ranks_reference_arm():
    """`--gpus 2` outside torchrun runs the script again as two ranks; the
    reference arm needs no GPU, and rank 0 alone prints its one line."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--workload", "tiny_fp32"],
                         capture_output=True, text=True, timeout=240, env=env, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
    assert lines[0]["cpu_baseline"]["kind"] == "oracle" and lines[0]["value"] > 0


def test_gemm1_bound_by_arithmetic_intensity():
    import workloads as W
    peaks = bench.FALLBACK_PEAKS
    for name, bound in (("mixtral", "tensor"), ("qwen3_skew", "tensor"), ("gpt2_moe", "tensor"),
                        ("deepseek_v3", "hbm")):
        wl = W.WORKLOADS[name]
        flops = 2 * (2 if wl.act == "swiglu" else 1) * wl.d_model * wl.d_ff * wl.N * wl.k
        assert bench.gemm1_bound(flops, bench.gemm1_bytes(wl, wl.E), peaks["bf16_tflops"], peaks["hbm_gbs"]) == bound
    wl = W.WORKLOADS["deepseek_v3"]
    # weights of the used experts once, x_sorted in, h out
    assert bench.gemm1_bytes(wl, 256) == 256 * 2 * 7168 * 2048 * 2 + 4096 * 8 * (7168 + 2048) * 2
