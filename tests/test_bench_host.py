"""Host logic of the benchmark's roofline: which int8 denominator matches the
sampled clocks, and the DRAM traffic figure read from the committed ncu
summary (null once the GEMM's source no longer matches the capture)."""
import os

import bench


def test_peak_follows_the_sampled_clock():
    burst, sustained = 3435.6, 2848.0
    p, why = bench.pick_int8_peak(burst, sustained, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}, 0.07, 1965.0)
    assert p == burst and why["kind"] == "burst"
    p, why = bench.pick_int8_peak(burst, sustained, {"sm_mhz": 1880.0, "sm_max_mhz": 1965.0}, 0.07, 1965.0)
    assert p == burst  # within 5% of the maximum
    p, why = bench.pick_int8_peak(burst, sustained, {"sm_mhz": 1372.0, "sm_max_mhz": 1965.0}, 4.0, 1965.0)
    assert p == sustained and why["kind"] == "sustained"
    # no clock sample: the length of the timed region decides
    assert bench.pick_int8_peak(burst, sustained, {}, 0.5, 1965.0)[0] == burst
    assert bench.pick_int8_peak(burst, sustained, {}, 3.0, 1965.0)[0] == sustained


def test_recorded_traffic_matches_the_gemm_source():
    """The committed summary was taken on the current GEMM source: its figure
    is reported, per launch, between the algorithmic bytes of the smallest
    BLOOM launch (0.29 GB) and twice those of the largest (1.09 GB)."""
    t = bench.recorded_traffic()
    assert t is not None
    assert 0.29e9 < t < 2 * 1.09e9
    names = [os.path.basename(f) for f in bench.GEMM_SOURCES]
    assert {"gemm.cu", "ptx.cuh", "sched.h"} <= set(names)


def test_recorded_traffic_is_null_for_another_source(tmp_path, monkeypatch):
    src = tmp_path / "k.txt"
    src.write_text(open(bench.TRAFFIC_FILE).read().replace("gemm_source_sha256_16:",
                                                          "gemm_source_sha256_16: 0000000000000000\nold:"))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(src))
    assert bench.recorded_traffic() is None


def test_ops_of_a_linear():
    lin = {l.name: l for l in bench.WORKLOAD.linears}["fc2"]
    assert bench.ops_of(lin) == 2 * 2048 * 14336 * 57344
