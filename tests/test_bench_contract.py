"""bench.py's output contract on CPU: the reference arm's JSON line carries
every key the contract names, the clock sampler keeps only the samples taken
inside the timed window, and the source hash that guards the committed ncu
traffic covers the tile-kernel sources."""
import datetime
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402

KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config")


def test_reference_line_keys(capsys):
    class A:
        steps, warmup, cpu_rows, gpus = 1, 0, 8, 1

    wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    assert bench.run_reference(A, wl, rank=0, world=1) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for k in KEYS:
        assert k in line, k
    assert line["impl"] == "reference" and line["higher_is_better"] is True
    assert line["config"]["workload"] == wl.name
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


class _FakeProc:
    def __init__(self, text):
        self.text = text

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.text, ""


def _line(ts, sm, reason="Not Active"):
    return f"{ts:%Y/%m/%d %H:%M:%S.%f}"[:-3] + f", 0, {sm}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {reason}"


def test_clock_samples_limited_to_timed_window():
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    ms = datetime.timedelta(milliseconds=1)
    c = bench.Clocks(0)
    c.t0, c.t1 = t0 + 300 * ms, t0 + 600 * ms
    c.proc = _FakeProc("\n".join([_line(t0, 900),                          # idle, before
                                  _line(t0 + 350 * ms, 1965),
                                  _line(t0 + 450 * ms, 1950, "Active"),
                                  _line(t0 + 900 * ms, 800)]))             # after
    r = c.stop()
    assert r["window"] == "timed" and r["samples"] == 2
    assert r["sm_mhz"] == (1965 + 1950) / 2 and r["reasons"] == ["sw_power_cap"]
    # a window too short for a sample: the samples within 0.25 s of it
    c2 = bench.Clocks(0)
    c2.t0, c2.t1 = t0 + 500 * ms, t0 + 510 * ms
    c2.proc = _FakeProc("\n".join([_line(t0, 900), _line(t0 + 400 * ms, 1965),
                                   _line(t0 + 700 * ms, 1960)]))
    r2 = c2.stop()
    assert r2["window"] == "near" and r2["samples"] == 2 and r2["reasons"] == []


def test_traffic_guarded_by_tile_source_hash(tmp_path, monkeypatch):
    h = bench._src_hash()
    assert len(h) == 16
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(
        {"k": {"src_hash": h, "bytes_per_launch_full": 123.0},
         "old": {"src_hash": "0" * 16, "bytes_per_launch_full": 5.0}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "_src_hash", lambda: h)
    assert bench._traffic("k") == 123.0
    assert bench._traffic("old") is None and bench._traffic("missing") is None


def test_source_hash_ignores_comments_only():
    # the hash that ties profiles/traffic.json to the tile sources sees code,
    # not comments or blank lines
    a = "int f(int x) {  // one\n    return x + 1;  /* two\n three */\n}\n"
    b = "int f(int x) {\n\n    return x + 1;\n}  // other words\n"
    c = "int f(int x) {\n    return x + 2;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
