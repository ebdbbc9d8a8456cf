"""Host-side statistics of bench.py (no GPU): the peak it rates a kernel
against, the per-step clock attribution and its bins, the runtime SM count."""
import datetime
import statistics

import pytest

import bench


def test_tensor_peak_takes_the_sustained_figure_for_long_regions():
    peaks = {"bf16_tflops": 1625.3, "bf16_tflops_sustained": 1400.0}
    p, label = bench.tensor_peak(peaks, "measured", 2.3)
    assert p == 1400.0 and "sustained" in label
    p, label = bench.tensor_peak(peaks, "measured", 0.13)
    assert p == 1625.3 and "burst" in label
    # no sustained figure recorded: the burst one, whatever the length
    p, _ = bench.tensor_peak({"bf16_tflops": 1590.0}, "fallback", 5.0)
    assert p == 1590.0


def test_clock_bins_group_steps_by_their_sampled_clock():
    step_ms = [100.0, 101.0, 120.0, 119.0, 118.0, 99.0]
    mhz = [1965.0, 1960.0, 1750.0, None, 1745.0, 1966.0]
    out = bench.clock_bins(step_ms, mhz)
    bins = {b["sm_mhz"]: b for b in out["bins"]}
    assert set(bins) == {1965, 1755, 1740}  # 1750 -> 1755, 1745 -> 1740
    assert bins[1965]["steps"] == 3
    assert bins[1965]["median_step_ms"] == pytest.approx(100.0)
    assert out["steps_with_a_sample"] == 5
    tagged = [100 * 1965, 101 * 1960, 120 * 1750, 118 * 1745, 99 * 1966]
    assert out["median_ms_x_mhz"] == pytest.approx(statistics.median(tagged))


def test_clock_bins_without_samples():
    out = bench.clock_bins([1.0, 2.0], [None, None])
    assert out["bins"] == [] and out["median_ms_x_mhz"] is None


def test_per_step_assigns_samples_to_the_step_that_ran(tmp_path):
    # a fake nvidia-smi log: samples every 50 ms from t0
    t0 = datetime.datetime(2026, 1, 2, 3, 4, 5).timestamp()
    path = tmp_path / "clocks.csv"
    lines = []
    for n in range(10):
        ts = datetime.datetime.fromtimestamp(t0 + 0.05 * n + 0.01)
        mhz = 1965 if n < 4 else 1800
        lines.append(f"{ts.strftime('%Y/%m/%d %H:%M:%S.%f')[:-3]}, {mhz}, 1965, 700.0, 0x0, "
                     "Not Active, Not Active, Not Active, Not Active")
    path.write_text("\n".join(lines) + "\n")

    class FakeProc:
        pass

    s = bench.ClockSampler(0)
    s.proc = FakeProc()
    s.file = open(path)
    try:
        # steps of 100, 100, 250 ms starting at t0: samples 0-1, 2-3, 4-8
        got = s.per_step(t0, [100.0, 100.0, 250.0, 10.0])
    finally:
        s.file.close()
        s.file = None
    assert got[:3] == [1965.0, 1965.0, 1800.0]
    assert got[3] is None  # no sample in its 10 ms


def test_ffma_peak_reads_the_sm_count(monkeypatch):
    monkeypatch.setattr(bench, "sm_count", lambda device=None: 100)
    assert bench.ffma_peak_tflops({"sm_max_mhz": 2000.0}) == pytest.approx(100 * 128 * 2 * 2e9 / 1e12)


def test_default_workload_is_the_largest_single_gpu_config():
    import sys
    src = open(bench.__file__).read()
    assert 'ap.add_argument("--config", default="c5"' in src
    from seeded_inputs import CONFIGS
    big = max((c for c in CONFIGS.values() if not c.name.startswith(("prof", "bob"))),
              key=lambda c: c.bwd_flops)
    assert big.name == "c5"
    assert sys.modules["bench"] is bench


def test_rect_pair_count_is_the_oracle_mask():
    import oracle
    for nq, nk, off in ((300, 1000, 700), (1000, 300, 0), (129, 128, 5000), (5, 8, 3)):
        assert bench.rect_pairs(nq, nk, off) == int(oracle.keep_mask(nq, nk, True, off).sum())
    # the last N positions as queries are the square causal problem
    assert bench.rect_pairs(640, 640, 0) == 640 * 641 // 2
