"""bench.py's measurement bookkeeping on the host: which tensor peak a timed
region is held to, which workloads get an L2 flush between steps, the
algorithmic byte model of each pass, and the lookup of a committed DRAM
traffic record by kernel, workload and kernel-source hash.  No GPU."""
import json

import pytest

import bench
from moe_fp8_grouped_b200 import synth

PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def test_burst_peak_at_full_clock_sustained_when_capped():
    v, why = bench.tensor_peak(PEAKS, "fallback", 0.13, False, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})
    assert v == pytest.approx(2 * 1590.0) and "burst" in why
    v, why = bench.tensor_peak(PEAKS, "fallback", 0.75, False, {"sm_mhz": 1556.0, "sm_max_mhz": 1965.0})
    assert v == pytest.approx(2 * 1400.0) and "sustained" in why
    # within 10 % of the maximum clock: still the burst figure
    v, _ = bench.tensor_peak(PEAKS, "fallback", 0.5, False, {"sm_mhz": 1780.0, "sm_max_mhz": 1965.0})
    assert v == pytest.approx(2 * 1590.0)


def test_peak_without_clock_samples_follows_region_length_and_bf16_has_no_factor():
    assert bench.tensor_peak(PEAKS, "fallback", 0.5, False)[0] == pytest.approx(3180.0)
    assert bench.tensor_peak(PEAKS, "fallback", 3.0, False)[0] == pytest.approx(2800.0)
    assert bench.tensor_peak(PEAKS, "fallback", 0.5, True)[0] == pytest.approx(1590.0)


def test_l2_flush_only_for_workloads_that_fit_in_l2():
    flushed = {n for n, w in synth.WORKLOADS.items() if bench.needs_l2_flush(w)}
    assert {"tiny", "ep_merged", "ep_separate"} <= flushed
    assert not flushed & {"mixtral", "dsv3_up", "dsv3_down", "ragged", "ragged_bf16"}


def test_algorithmic_bytes_count_inputs_and_outputs_once():
    M, K, N, G = 256, 512, 384, 4
    b = bench.algorithmic_bytes(M, K, N, G, G, "static")
    # fwd: bf16 lhs + E4M3 weights + fp32 [G, N] scales + bf16 out
    assert b["fwd"] == 2 * M * K + G * K * N + 4 * G * N + 2 * M * N
    # dlhs: bf16 dout + its 1 x 128 block scales + weights + scales + bf16 dlhs
    assert b["dlhs"] == 2 * M * N + 4 * M * N // 128 + G * K * N + 4 * G * N + 2 * M * K
    # drhs: bf16 lhs + bf16 dout + fp32 dW
    assert b["drhs"] == 2 * M * K + 2 * M * N + 4 * G * K * N
    d = bench.algorithmic_bytes(M, K, N, G, G, "dynamic")
    assert d["fwd"] - b["fwd"] == 4 * M * K // 128  # the lhs block scales
    bf = bench.algorithmic_bytes(M, K, N, G, G, "none")
    assert bf["fwd"] == 2 * M * K + 2 * G * K * N + 2 * M * N  # bf16 weights, no scales
    # empty groups' weights are not read by the row passes
    assert bench.algorithmic_bytes(M, K, N, G, 1, "static")["fwd"] == b["fwd"] - (G - 1) * K * N


def test_traffic_record_needs_matching_kernel_workload_and_source_hash(tmp_path, monkeypatch):
    key = "mixtral/G8/M16384/K4096/N28672/static"
    rec = {"gemm_drhs": [{"workload_key": key, "bytes_per_launch": 123, "gemm_src_sha256_16": bench.gemm_src_hash()},
                         {"workload_key": "other", "bytes_per_launch": 7, "gemm_src_sha256_16": bench.gemm_src_hash()}],
           "gemm_fwd": [{"workload_key": key, "bytes_per_launch": 9, "gemm_src_sha256_16": "0" * 16}],
           "note": "text"}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.traffic_record("gemm_drhs", key) == 123
    assert bench.traffic_record("gemm_fwd", key) is None  # captured from other kernel sources
    assert bench.traffic_record("gemm_dlhs", key) is None  # no capture of that kernel
    assert bench.traffic_record("gemm_drhs", "dsv3_up/G256/M32768/K7168/N4096/dynamic") is None


def test_committed_traffic_records_match_the_current_kernel_sources():
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    h = bench.gemm_src_hash()
    kernels = [k for k, v in rec.items() if isinstance(v, list)]
    assert kernels
    for k in kernels:
        for r in rec[k]:
            assert r["gemm_src_sha256_16"] == h, f"{k} {r['workload_key']}: captured from other kernel sources"
            assert r["dram_bytes_read"] + r["dram_bytes_write"] == r["bytes_per_launch"]
            assert r["passes"] == 1
