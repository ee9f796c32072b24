"""The timing statistic of bench.py, on the CPU: the interquartile mean of the
5/16 to 11/16 quantiles of the per-replay times."""
import bench


def test_iqm_of_a_sorted_ramp_is_the_middle_mean():
    vals = list(range(16))            # quantiles 5/16 .. 11/16 -> elements 5 .. 10
    assert bench.iqm(vals) == sum(range(5, 11)) / 6


def test_iqm_ignores_order_and_outliers():
    vals = [3.0] * 40 + [1e9, 1e9, -1e9]
    import random
    random.Random(0).shuffle(vals)
    assert bench.iqm(vals) == 3.0


def test_iqm_of_one_and_two_values():
    assert bench.iqm([7.0]) == 7.0
    assert bench.iqm([1.0, 3.0]) in (1.0, 2.0, 3.0)


def test_rooflines():
    r = bench.hbm_roofline(6544e9 * 1e-3, 2e-3, 6544.0, "of measured")
    assert abs(r["frac"] - 0.5) < 1e-9 and r["bound"] == "hbm"
    pk = {"hbm": 1000.0, "bf16": 1000.0, "src": "x"}
    m = bench.mixed_roofline(1e9, 1e15, 2.0, pk)      # 1 ms of HBM, 1 s of tensor work
    assert m["bound"] == "tensor" and abs(m["frac"] - 0.5) < 1e-9
