"""Host-side pieces of bench.py that need no GPU: the clock summary taken
from nvidia-smi samples, the DRAM-traffic record keyed on the kernel source,
and the algorithmic byte count the roofline divides by."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import huffman_decode_df11_b200 as df11  # noqa: E402


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.lines = list(lines)
    return s


def _row(sm, mx=1965, hw="Not Active", hwt="Not Active", swt="Not Active", cap="Not Active"):
    return f"0, {sm}, {mx}, 700.5, 0x0, {hw}, {hwt}, {swt}, {cap}"


def test_clock_summary_median_and_reasons():
    s = _sampler([_row(1965), _row(1950), _row(1900, cap="Active"), "garbage", "",
                  "0, [N/A], 1965, 1, 0, a, b, c, d"])
    out = s.summary()
    assert out["sm_mhz"] == 1950 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3


def test_clock_summary_flags_throttling_and_no_samples():
    out = _sampler([_row(1500, hw="Active"), _row(1400, hwt="Active", swt="Active")]).summary()
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert out["sm_mhz"] == 1450
    empty = _sampler([]).summary()
    assert empty["sm_mhz"] is None and empty["reasons"] == ["unsampled"]


def test_traffic_record_follows_the_source_hash(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("__global__ void k() {}\n")
    h = bench.kernel_hash(str(src))
    rec = tmp_path / "traffic.txt"
    rec.write_text("# comment line\n"
                   f"{h} block/c24/t256 591206912  capture.md\n"
                   f"{h} build/c24/t256 1444705195\n"
                   "0123456789abcdef block/c8/t256 1\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.recorded_traffic("block/c24/t256", str(src)) == 591206912.0
    assert bench.recorded_traffic("build/c24/t256", str(src)) == 1444705195.0
    assert bench.recorded_traffic("block/c8/t256", str(src)) is None   # another source
    assert bench.recorded_traffic("embedding/c24/t256", str(src)) is None
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert bench.recorded_traffic("block/c24/t256", str(src)) is None  # stale once changed
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.txt"))
    assert bench.recorded_traffic("block/c24/t256", str(src)) is None


@pytest.mark.parametrize("C,T,n", [(24, 256, 300_001), (8, 128, 70_000), (16, 512, 1)])
def test_algorithmic_bytes_counts_every_buffer_the_decode_moves(C, T, n):
    rng = np.random.default_rng(n)
    w = (rng.normal(0, 0.02, n).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    h = df11.compress(w, C, T)
    p = h.params
    chunks = int(p.num_blocks) * T
    # the stream up to its last bit, one sign/mantissa byte per element, the
    # packed 5-bit gaps, one count per chunk, the block positions, the
    # tables, the code lengths, and the BF16 output
    want_in = (-(-int(p.total_bits) // 8) + n + -(-5 * chunks // 8) + chunks
               + h.block_out_pos.nbytes + h.luts.nbytes + h.code_lengths.nbytes)
    assert bench.algorithmic_bytes(h) == want_in + 2 * n
    assert bench.algorithmic_bytes(h, counts=False) == want_in - chunks + 2 * n
    # what is stored is the moved input plus paddings only
    assert 0 <= h.compressed_bytes() - want_in < C * T + 64 + 16


def test_measured_peak_reads_the_driver_file_or_falls_back(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6538.2}')
    assert bench.measured_peak() == (6538.2, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text("not json")
    assert bench.measured_peak()[1] == "fallback"


class _FakeEvent:
    """A CUDA event stand-in: records the position in a shared log, and its
    'elapsed time' is the number of step calls between two records."""

    def __init__(self, log):
        self.log, self.at = log, None

    def record(self, stream):
        assert stream == "s"
        self.log.append("rec")
        self.at = self.log.count("step")

    def synchronize(self):
        self.log.append("sync")

    def elapsed_time(self, other):
        return float(other.at - self.at)


class _FakeFlush:
    def __init__(self, log):
        self.log = log

    def fill_(self, v):
        self.log.append(f"flush{v}")


def test_time_steps_back_to_back():
    log = []
    ms = bench.time_steps(lambda: log.append("step"), 4, "s", lambda: _FakeEvent(log))
    assert ms == 1.0
    assert log == ["rec", "step", "step", "step", "step", "rec", "sync"]


def test_time_steps_flushes_before_every_step_and_times_steps_alone():
    log = []
    ms = bench.time_steps(lambda: log.append("step"), 3, "s", lambda: _FakeEvent(log),
                          flush=_FakeFlush(log))
    assert ms == 1.0
    assert log == ["flush1", "rec", "step", "rec", "flush2", "rec", "step", "rec",
                   "flush3", "rec", "step", "rec", "sync"]
    with pytest.raises(ValueError):
        bench.time_steps(lambda: None, 0, "s", lambda: _FakeEvent([]))


def test_flush_rule():
    assert bench.FLUSH_BYTES >= 2 * bench.L2_BYTES
    assert bench.flush_wanted("auto", 3_500_000)             # 1024x1024: fits in L2
    assert not bench.flush_wanted("auto", 646_000_000)       # the block: larger than L2
    assert bench.flush_wanted("on", 646_000_000)
    assert not bench.flush_wanted("off", 3_500_000)


def test_build_hist_launches_follows_the_builder_rule():
    """bench.build_hist_launches (the launch count the build line claims):
    tensors in order, at most 32 per histogram launch, the shortest run of
    last tensors holding a quarter of the tiles in a launch of its own, and
    no kernel for a launch of empty tensors."""
    t = bench.BUILD_TILE
    block = [4096 * 4096, 1024 * 4096, 1024 * 4096, 4096 * 4096] + [12288 * 4096] * 3
    assert bench.build_hist_launches(block) == 2      # six tensors, then the last
    assert bench.build_hist_launches([]) == 0
    assert bench.build_hist_launches([0, 0, 0]) == 0  # nothing to count
    assert bench.build_hist_launches([1]) == 1
    assert bench.build_hist_launches([t] * 4) == 2    # the last tile is a quarter
    assert bench.build_hist_launches([t] * 8) == 2    # the last two
    # forty equal tensors: the last ten in their own launch, thirty before
    assert bench.build_hist_launches([10 * t] * 40) == 2
    # a hundred: the last 25 in their own launch, the 75 before in three
    assert bench.build_hist_launches([t] * 100) == 4
    # at most 32 in the last launch: 32 of 200, the 168 before in six
    assert bench.build_hist_launches([t] * 200) == 7
    # a first launch of empty tensors runs no kernel
    assert bench.build_hist_launches([0, 0, 0, t]) == 1
    assert bench.build_hist_launches([0] * 5 + [t] * 20) == 2
