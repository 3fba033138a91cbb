"""Host logic of bench.py on the CPU: the per-layer path, the algorithmic bytes, the roofline's bound and
fraction, the clock summary and the peaks file.  These decide every number the bench line reports."""
import json
import types

import numpy as np
import pytest

import bench
import workloads as wl


def layers(name):
    return wl.workload(name)


def test_layer_paths_follow_the_library_dispatch():
    # LLaMA (2:4, K % 128 == 0, T = 2048, with an index map): the compress grid gathers, then the pair GEMM
    assert {bench.layer_mode(L, "one-call", "auto", L.permuted) for L in layers("llama7b")} == {"combined"}
    # decode (T = 16): the fused prune + GEMM kernel
    assert [bench.layer_mode(L, "one-call", "auto", L.permuted) for L in layers("decode")] == ["fused"]
    # 1:8 ViT, the hybrid, two-call steps and other algorithms: compress, then the GEMM call
    assert {bench.layer_mode(L, "one-call", "auto", L.permuted) for L in layers("vit")} == {"split"}
    assert {bench.layer_mode(L, "one-call", "auto", False) for L in layers("patch_p50")} == {"split"}
    assert {bench.layer_mode(L, "two-calls", "auto", True) for L in layers("llama7b")} == {"split"}
    assert {bench.layer_mode(L, "one-call", "dense", True) for L in layers("llama7b")} == {"split"}
    # without an index map a 2:4 pair shape has nothing to gather: compress, then the GEMM call
    assert {bench.layer_mode(L, "one-call", "auto", False) for L in layers("llama7b")} == {"split"}


def test_gemm_bytes_written_out():
    L = layers("llama7b")[0]  # 4096 x 4096, T = 2048, 2:4 with an index map
    d = types.SimpleNamespace(idx=np.arange(L.K), tmap=None)
    values = 4096 * 2048 * 2          # bf16 survivors
    meta = 4096 * 4096 // 8           # 2 bits per survivor
    x = 4096 * 2048 * 2
    y = 4096 * 2048 * 2
    idx = 4096 * 4
    assert bench.gemm_bytes(L, d) == values + meta + x + y + idx
    V = layers("vit")[0]  # 3072 x 768 at 1:8: 96 survivors per row, ten 3-bit positions per word
    dv = types.SimpleNamespace(idx=None, tmap=None)
    assert bench.gemm_bytes(V, dv) == 3072 * 96 * 2 + 3072 * 10 * 4 + 768 * 50432 * 2 + 3072 * 50432 * 2


def test_gemm_bytes_hybrid_reads_dense_tiles_from_w():
    P = layers("patch_p50")[0]
    tmap = np.zeros((32, 32), np.uint8)
    tmap[:16] = 1  # half the tiles 2:4
    d = types.SimpleNamespace(idx=None, tmap=tmap)
    dense_elems = 16 * 32 * 128 * 128
    all_24 = 4096 * 2048 * 2 + 4096 * 4096 // 8
    expect = all_24 + 2 * 4096 * 4096 * 2 + 2.0 * dense_elems - 1.125 * dense_elems + tmap.size
    assert bench.gemm_bytes(P, d) == expect


def _runner_with(bufs):
    r = bench.Runner.__new__(bench.Runner)
    r.bufs = bufs
    return r


def test_roofline_picks_the_slower_bound():
    tc_peak, hbm_peak = 1630.2, 6534.1  # TFLOP/s, GB/s
    # compute-heavy: 1e12 FLOPs, 1e8 bytes -> tensor time 0.61 ms > HBM time 0.015 ms
    r = _runner_with([{"flops": 1e12, "gemm_bytes": 1e8, "mode": "combined"}])
    roof = r.roofline(1.0, tc_peak, hbm_peak, "burst")
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["achieved"] == pytest.approx(1e12 / 1e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / tc_peak)
    # byte-heavy: 1e9 FLOPs, 1e9 bytes -> HBM time 0.153 ms > tensor time 0.0006 ms
    r = _runner_with([{"flops": 1e9, "gemm_bytes": 1e9, "mode": "fused"}])
    roof = r.roofline(0.5, tc_peak, hbm_peak, "burst")
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["achieved"] == pytest.approx(1e9 / 0.5e-3 / 1e9)
    assert roof["frac"] == pytest.approx(roof["achieved"] / hbm_peak)


def test_clock_summary():
    s = bench.ClockSampler("GPU-1")
    # uuid, sm, max, power, active, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    s.rows = [["GPU-1", "1965", "1965", "800", "0x4", "Not Active", "Not Active", "Not Active", "Active"],
              ["GPU-1", "1800", "1965", "990", "0x4", "Not Active", "Not Active", "Not Active", "Active"],
              ["GPU-1", "1965", "1965", "700", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"],
              ["GPU-2", "300", "1965", "100", "0x0", "Active", "Not Active", "Not Active", "Not Active"]]
    out = s.summary()
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0 and out["samples"] == 3
    assert out["reasons"] == ["sw_power_cap"]  # the other GPU's hw_slowdown is not ours
    assert bench.ClockSampler("GPU-3").summary()["reasons"] == ["unsampled"]


def test_step_config_names_the_step_and_the_l2_rule():
    cfg = bench.step_config("llama7b", layers("llama7b"), "one-call", "auto", False, 1)
    assert cfg["workload"] == "llama7b" and cfg["permuted"] is True
    assert cfg["shapes"] == [[4096, 4096], [11008, 4096], [4096, 11008]] and cfg["T"] == [2048] * 3
    assert cfg["step"].startswith("one nm_prune_spmm call per layer")
    assert cfg["l2"].startswith("inputs larger than L2")
    assert set(cfg["layer_paths"].values()) == {"combined"}
    tiny = bench.step_config("tiny", layers("tiny"), "one-call", "auto", False, 2)
    assert tiny["l2"].startswith("working set below L2") and tiny["parallelism"] == "replicas x2"


def test_peaks_file_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0,
                                                              "bf16_tflops_sustained": 3.0}))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["bf16_tflops_sustained"] == 3.0


def test_reencoded_bound_counts_four_products_per_survivor():
    # ViT 3072x768, T = 50432, at 1:8: 29.7 useful GFLOP; the re-encoded form multiplies 4x as many products,
    # half of the dense GEMM's, at the dense product rate: 73 us per layer at 1630 TFLOP/s, above the HBM term
    V = layers("vit")[0]
    useful = 2.0 * 3072 * (768 // 8) * 50432
    bufs = [{"flops": useful, "gemm_bytes": 388030464.0}]
    t = bench.reencoded_bound_s(bufs, 1630.2, 6534.1)
    assert t == pytest.approx(2.0 * 3072 * 768 * 50432 / 2 / 1630.2e12)
    assert t == pytest.approx(4 * V.useful_flops / 1630.2e12) and 72e-6 < t < 74e-6
    # bytes dominate when the products are few
    assert bench.reencoded_bound_s([{"flops": 1.0, "gemm_bytes": 6534.1e9}], 1630.2, 6534.1) == pytest.approx(1.0)
