"""Host-side pieces of bench.py, on CPU: the roofline object of the dominant
kernel and the weak-scaling rate."""
import bench


def test_decode_roofline_when_decode_dominates():
    r = bench.roofline_of(100e-6, 538_865_804, 0.0, 0, 6540.2, 1390.0, "measured",
                          traffic=555_000_000)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - 5388.7) < 0.1
    assert abs(r["frac"] - 5388.66 / 6540.2) < 1e-4
    assert r["traffic"] == 555_000_000
    assert r["algorithmic_bytes_per_launch"] == 538_865_804


def test_prefill_roofline_when_prefill_dominates():
    # the mixed batch: prefill 100.7 us against a 70.8 us decode call
    r = bench.roofline_of(70.8e-6, 300_000_000, 100.7e-6, 63_669_534_720, 6540.2, 1390.0,
                          "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 63_669_534_720 / 100.7e-6 / 1e12) < 0.1
    assert abs(r["frac"] - r["achieved"] / 1390.0) < 1e-3
    assert r["traffic"] is None
    assert r["algorithmic_flops_per_launch"] == 63_669_534_720


def test_decode_roofline_when_prefill_is_shorter():
    r = bench.roofline_of(100e-6, 500_000_000, 50e-6, 10**10, 6540.2, 1390.0, "fallback")
    assert r["bound"] == "hbm" and "fallback" in r["peak_source"]


def test_whole_job_rate_is_weak_scaling():
    assert bench.whole_job_rate(1e9, 1, 1.0) == 1e9
    assert bench.whole_job_rate(1e9, 8, 2.0) == 4e9
