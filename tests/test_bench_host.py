"""The benchmark's roofline arithmetic and records, on the host (no GPU):
algorithmic bytes and flops per channel-token as the design states them, the
bound each workload is measured against, and the DRAM-traffic records, which
apply only while the kernel sources they were taken from are unchanged."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_per_channel_token():
    for name, wl in bench.WORKLOADS.items():
        chtok = wl["B"] * wl["L"] * wl["D"]
        if not wl.get("decode"):
            assert bench.algorithmic_bytes(wl) == 8 * chtok, name  # 3 bf16 reads + 1 bf16 write
    assert bench.algorithmic_bytes(bench.WORKLOADS["modal32k"]) == 1073741824  # 1.074 GB per call


def test_flops_per_channel_token():
    assert bench.flops_per_chtok(bench.WORKLOADS["modal32k"]) == 68    # 4N + 4, N = 16
    assert bench.flops_per_chtok(bench.WORKLOADS["cmodal8k"]) == 100   # 12N + 4, N = 8 complex
    assert bench.flops_per_chtok(bench.WORKLOADS["fir128"]) == 260     # 2K + 4
    assert bench.flops_per_chtok(bench.WORKLOADS["fir7"]) == 18


def test_decode_bytes_count_state_and_parameters():
    wl = bench.WORKLOADS["decode_modal"]
    B, D, N, L = wl["B"], wl["D"], wl["N"], wl["L"]
    assert bench.algorithmic_bytes(wl) == L * (B * D * (8 + 8 * N) + D * (8 * N + 4))
    wl = bench.WORKLOADS["decode_fir128"]
    B, D, K, L = wl["B"], wl["D"], wl["K"], wl["L"]
    assert bench.algorithmic_bytes(wl) == L * (B * D * (8 + 8 * (K - 1)) + D * (2 * K + 4))


@pytest.mark.parametrize("name,bound", [("modal32k", "hbm"), ("fir7", "hbm"), ("fir128", "alu"), ("cmodal32k", "alu")])
def test_which_roofline_bounds_each_workload(name, bound):
    # the bound the bench reports: flops at the FP32 SIMT peak against bytes at the copy peak
    wl = bench.WORKLOADS[name]
    chtok = wl["B"] * wl["L"] * wl["D"]
    alu = 148 * 128 * 2 * 1965e6           # FP32 SIMT peak at the maximum SM clock
    hbm = 6532.5e9                          # measured copy bandwidth
    t_flops = bench.flops_per_chtok(wl) * chtok / alu
    t_bytes = bench.algorithmic_bytes(wl) / hbm
    assert ("alu" if t_flops > t_bytes else "hbm") == bound


def test_traffic_records_follow_the_kernel_sources(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for name, r in rec.items():
        assert name in bench.WORKLOADS, name
        assert r["dram_bytes_per_launch"] > 0
        assert os.path.exists(os.path.join(ROOT, r["source"])), r["source"]
    # a record whose hash does not match the current sources is not used
    fake = tmp_path / "profiles"
    fake.mkdir()
    (fake / "traffic.json").write_text(json.dumps(
        {"modal32k": {"dram_bytes_per_launch": 1, "kernel_sources_sha256_16": "0000000000000000"}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind="modal": "ffffffffffffffff")
    assert bench.recorded_traffic("modal32k") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind="modal": "0000000000000000")
    assert bench.recorded_traffic("modal32k") == 1


def test_tensor_core_fir_line():
    # the DFT-as-GEMM FIR: its method's tf32 MMA work per channel-token (the
    # two spectra and the inverse per 64 channels x 128 outputs), no SIMT FMA
    # floor, and a tf32 peak of the bf16 figure times the nominal ratio
    wl = bench.WORKLOADS["fir128_dft"]
    macs = 2 * 128 * 64 * 128 + 2 * 128 * 64 * 256 + 128 * 64 * 256
    assert bench.DFT_FLOPS_PER_CHTOK == 2 * macs // (64 * 128)
    assert bench.kernel_fma_per_chtok(wl) is None
    assert bench.algorithmic_bytes(wl) == bench.algorithmic_bytes(bench.WORKLOADS["fir128"])
    peak, src = bench.tensor_peak_tflops_tf32()
    assert peak > 0 and "tf32/bf16" in src
    assert abs(bench.TF32_PER_BF16 - 1.1 / 2.25) < 1e-12


def test_tensor_core_fir_traffic_follows_its_own_sources(tmp_path, monkeypatch):
    # the DFT path's record is keyed by the hash of fir_dft.cu and the shared
    # headers, not by the SIMT FIR's
    fake = tmp_path / "profiles"
    fake.mkdir()
    (fake / "traffic.json").write_text(json.dumps(
        {"fir128_dft": {"dram_bytes_per_launch": 7, "kernel_sources_sha256_16": "abc"}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind="modal": "abc" if kind == "fir_dft" else "zzz")
    assert bench.recorded_traffic("fir128_dft") == 7
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind="modal": "abc" if kind == "fir" else "zzz")
    assert bench.recorded_traffic("fir128_dft") is None
