"""bench.py's clock record: only nvidia-smi rows stamped inside the timed
region are summarised (no GPU needed: the rows are synthetic)."""
import datetime
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _row(t, mhz, power_cap="Not Active", hw="Not Active"):
    stamp = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return (f"{stamp}, 0, {mhz}, 1965, 700.5, 0x0000000000000000, {hw}, Not Active, "
            f"Not Active, {power_cap}")


def test_rows_outside_the_region_are_dropped():
    import bench
    t0 = time.time()
    lines = [_row(t0 - 2.0, 345), _row(t0 + 0.05, 1965), _row(t0 + 0.15, 1950, power_cap="Active"),
             _row(t0 + 3.0, 345), "garbage line", ""]
    rows = bench.ClockSampler.parse(lines, t0, t0 + 0.3)
    assert [r[0] for r in rows] == [1965.0, 1950.0]
    assert rows[1][2][3] == "Active"
    assert len(bench.ClockSampler.parse(lines)) == 4


def test_summary_of_a_sampled_region(tmp_path):
    import bench
    t0 = time.time()
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join([_row(t0 + 0.05, 1965), _row(t0 + 0.15, 1950, hw="Active"),
                               _row(t0 + 0.25, 1965)]) + "\n")
    clk = bench.ClockSampler(0)
    clk.path, clk.t0, clk.t1 = str(path), t0, t0 + 0.3
    s = clk.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_slowdown"]
    assert not path.exists()


def test_summary_without_rows_says_unsampled():
    import bench
    clk = bench.ClockSampler(0)
    assert clk.summary()["reasons"] == ["unsampled"]
