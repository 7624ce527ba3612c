"""Host logic of bench.py on CPU: the clock-dependent choice of the tensor
peak, and the chunked oracle the CPU baseline and the reference arm time
(its chunks together must be exactly one block forward of the oracle)."""
import json

import numpy as np
import pytest

import bench
import oracle
import workloads as W

PK = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1300.0, "clocks_under_load": {"sm_mhz_median": 1300.0}}


def test_tensor_peak_follows_the_sampled_clock(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "INT8_PEAK_FILE", str(tmp_path / "absent.json"))
    # full clock -> burst; the sustained figure's own clock -> sustained; between -> linear in the clock
    assert bench.tensor_peak(PK, {"sm_mhz": 1965.0})["peak"] == 1600.0
    assert bench.tensor_peak(PK, {"sm_mhz": 1300.0})["peak"] == 1300.0
    assert bench.tensor_peak(PK, {"sm_mhz": 1400.0})["peak"] == pytest.approx(1400.0)
    assert bench.tensor_peak(PK, {"sm_mhz": 900.0})["peak"] == 1300.0  # never below the sustained figure
    assert bench.tensor_peak(PK, {"sm_mhz": None})["peak"] == 1300.0
    # int8 without a measured pair: the bf16 pair x 2, and its own nominal peak
    p = bench.tensor_peak(PK, {"sm_mhz": 1965.0}, int8=True)
    assert p["peak"] == 3200.0 and p["nominal"] == 4500.0 and "x 2" in p["basis"]
    # with a measured int8 pair it is used as is
    f = tmp_path / "int8.json"
    f.write_text(json.dumps({"int8_tops": 3000.0, "int8_tops_sustained": 2500.0, "sustained_sm_mhz_median": 1250.0}))
    monkeypatch.setattr(bench, "INT8_PEAK_FILE", str(f))
    assert bench.tensor_peak(PK, {"sm_mhz": 1965.0}, int8=True)["peak"] == 3000.0
    assert bench.tensor_peak(PK, {"sm_mhz": 1250.0}, int8=True)["peak"] == 2500.0


def test_fallback_peaks_are_labelled(monkeypatch, tmp_path):
    """Without MEASURED_PEAKS.json the bench falls back to the earlier
    measurement and says so in every basis it prints."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "INT8_PEAK_FILE", str(tmp_path / "absent.json"))
    pk, src = bench.peaks()
    assert src == "fallback" and pk["hbm_gbs"] == 6650.0
    p = bench.tensor_peak(pk, {"sm_mhz": 1965.0})
    assert p["peak"] == 1590.0 and p["basis"].startswith("fallback peaks")
    assert "MEASURED_PEAKS.json (cuBLAS" not in bench.tensor_peak(pk, {"sm_mhz": 1300.0}, int8=True)["basis"]


@pytest.mark.parametrize("name", ["block_d256_s288"])
def test_oracle_chunks_are_one_block(name):
    wl = W.WORKLOADS[name]
    oc = bench.OracleChunks(wl, 8)
    out = np.concatenate([oc.run(i) for i in range(8)], axis=0)
    assert sum(oc.tokens(i) for i in range(8)) == wl.seq
    w, x = bench._oracle_inputs(wl)
    ref = oracle.block_forward(x, w, wl)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_oracle_chunks_int8_reference_uses_dequantised_weights():
    wl = W.WORKLOADS["block_d256_s288"].with_(dtype=W.INT8)
    oc = bench.OracleChunks(wl, 4)
    out = np.concatenate([oc.run(i) for i in range(4)], axis=0)
    w, x = bench._oracle_inputs(wl)
    assert np.allclose(out, oracle.block_forward(x, oracle.dequant_weights(w), wl), rtol=1e-12, atol=1e-12)


def test_measured_traffic_only_for_the_source_it_was_taken_on(monkeypatch, tmp_path):
    """The roofline's `traffic` comes from a committed ncu figure only while
    the kernel's source still hashes to the digest recorded with it; after any
    change to that source the bench reports null rather than a stale number."""
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", {"attention": ["k.cu"], "gemm": ["k.cu"], "mem": ["k.cu"]})
    (tmp_path / "profiles").mkdir()
    rec = {"attention@wl": {"bytes_per_launch": 123, "src": bench.src_digest(["k.cu"])}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.measured_traffic("attention", "wl") == 123
    assert bench.measured_traffic("attention", "other_workload") is None
    src.write_text("kernel v2")
    assert bench.measured_traffic("attention", "wl") is None


def test_committed_traffic_matches_the_current_sources():
    """Every committed traffic figure was taken on the kernel sources as they
    are in this tree (the bench line would otherwise report null)."""
    rec = json.load(open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")))
    assert rec
    for key in rec:
        kernel, wl = key.split("@")
        assert bench.measured_traffic(kernel, wl) == rec[key]["bytes_per_launch"], key
