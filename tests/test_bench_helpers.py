"""Host-side logic of bench.py (CPU): the per-step percentile rule, the clock
record (only samples read after the timed region starts, throttle reasons,
loaded-clock median), the decode-group byte count and the traffic record's
source-hash gate."""
import json
import os

import bench


def test_percentile_nearest_rank():
    xs = [5.0, 1.0, 4.0, 2.0, 3.0]
    assert bench.pct(xs, 50) == 3.0
    assert bench.pct(xs, 95) == 5.0
    assert bench.pct(xs, 0) == 1.0
    assert bench.pct(list(range(1, 41)), 95) == 38
    assert bench.pct([], 50) is None


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        pass


class _Thread:
    def join(self, timeout=None):
        pass


def _line(mhz, watts, reasons=("Not Active",) * 4, bus="00000000:1B:00.0"):
    return ", ".join(["0", bus, str(mhz), "1965", str(watts), "0x0"] + list(reasons))


def test_clock_record_uses_timed_region_only():
    c = bench.ClockSampler("1b:00.0")
    c.proc, c.t = _Proc(), _Thread()
    c.lines = [_line(1965, 120)] * 5                    # idle, before the timed region
    c.mark()
    c.lines += [_line(1800, 900, ("Not Active", "Not Active", "Not Active", "Active"))] * 7
    c.lines += [_line(1700, 950)] * 2
    c.lines += [_line(1500, 950, bus="00000000:2C:00.0")] * 3   # another GPU: ignored
    r = c.stop()
    assert r["samples"] == 9
    assert r["sm_mhz"] == 1800.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    assert r["power_w_max"] == 950.0


def test_clock_record_flags_slowdowns_and_ignores_idle_clocks():
    c = bench.ClockSampler(None)
    c.proc, c.t = _Proc(), _Thread()
    c.mark()
    c.lines = [_line(300, 80)] * 3 + [_line(1900, 800, ("Active", "Not Active", "Active", "Not Active"))] * 3
    r = c.stop()
    assert r["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert r["sm_mhz"] == 1900.0      # samples below half the max clock are not "under load"


def test_decode_group_bytes_formula():
    # one sequence, one kv head with one query head, tiny sizes: every term by hand
    c = dict(B=1, Hq=1, Hkv=1, d=2, L=32, P=16, k=4, layers=2)
    row = 2 * 2                       # d bf16 values
    pt = 1 * (32 // 16) * 4           # page-table words
    scan = 32 * row + 2 * 2 + pt + 4 * 4
    per_layer = 4 * 2 * row + 4 * 4 + 2 * 2 * 2 + pt
    assert bench.decode_group_bytes(c) == scan + 2 * per_layer
    # the bench's decode group
    big = dict(B=32, Hq=32, Hkv=8, d=128, L=65536, P=16, k=4096, layers=4)
    assert bench.decode_group_bytes(big) == 12973768704


def test_traffic_record_requires_matching_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = bench.sources_sha1(bench.TRAFFIC_SOURCES["decode"])
    (prof / "traffic.json").write_text(json.dumps({
        "k_prefill_tc": {"bytes": 5, "src_sha1": "0" * 40},
        "decode": {"bytes": 7, "src_sha1": good}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the kernel sources are read from the real tree, the record from tmp_path
    real_sha = bench.sources_sha1

    def sha(files):
        monkeypatch.setattr(bench, "ROOT", os.path.dirname(os.path.abspath(bench.__file__)))
        try:
            return real_sha(files)
        finally:
            monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "sources_sha1", sha)
    t = bench.load_traffic()
    assert t == {"k_prefill_tc": None, "decode": 7}
