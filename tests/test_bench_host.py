"""Host-side checks of the benchmark's bookkeeping (no GPU): the DRAM traffic
it reports next to the roofline belongs to the GEMM sources in the tree, and
the clock record keeps only the samples taken inside the timed window, and
an auxiliary sub-measurement that fails is recorded, not fatal."""
import bench


def test_traffic_constants_match_gemm_sources():
    """roofline.traffic comes from ncu captures of the GEMM kernels; the hash
    of the sources they were taken on must be the current one (else the
    benchmark reports null and the captures must be taken again)."""
    assert bench.NCU_TRAFFIC["kernel_hash"] == bench.gemm_source_hash()
    for name, b in bench.NCU_TRAFFIC["bytes_per_launch"].items():
        # 65,536-token launches move at least the 1 GiB logits / dLogits tensor
        assert 0.9e9 < b < 2.0e9, name


def test_clock_window_filters_samples():
    c = bench.ClockSampler(0)
    # (host time, SM MHz, max MHz, active reasons)
    c.samples = [(0.5, 1200.0, 1965.0, ("sw_power_cap",)),   # before the window
                 (1.1, 1965.0, 1965.0, ()),
                 (1.2, 1950.0, 1965.0, ()),
                 (1.3, 1965.0, 1965.0, ("sw_power_cap",)),
                 (2.5, 900.0, 1965.0, ("hw_slowdown",))]      # after it
    c.t0, c.t1 = 1.0, 2.0  # the window begin() / end() would mark
    s = c.summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_window_empty_reports_why():
    c = bench.ClockSampler(0)
    c.samples = [(0.5, 1965.0, 1965.0, ())]
    c.t0, c.t1 = 1.0, 2.0
    c.nvml_error = "NVMLError: test"
    s = c.summary()
    assert s["samples"] == 0 and s["samples_outside_window"] == 1
    assert s["nvml_error"] == "NVMLError: test"


def test_auxiliary_measurement_records_an_exception():
    """A failing auxiliary sub-measurement leaves its error in the line; a
    working one returns its object unchanged."""
    def boom():
        raise RuntimeError("no such tensor")
    assert bench.auxiliary(boom) == {"error": "RuntimeError: no such tensor"}
    assert bench.auxiliary(lambda: {"value": 1.0}) == {"value": 1.0}
