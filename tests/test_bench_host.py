"""Host-side helpers of bench.py (no GPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_source_tag_ignores_comments_and_spacing(tmp_path):
    a = tmp_path / "a.cu"
    a.write_text("int f(int x) {  // doubled\n  return 2 * x; /* fast */\n}\n")
    t0 = bench.source_tag([str(a)])
    a.write_text("// a comment that moved\nint f(int x) {\n\n    return 2 * x;\n}\n")
    assert bench.source_tag([str(a)]) == t0
    a.write_text("int f(int x) { return 3 * x; }\n")
    assert bench.source_tag([str(a)]) != t0


def test_attention_traffic_scales_per_query_part_and_keeps_kv_once():
    cap = bench.ATTN_CAPTURE
    t = bench.attn_traffic(cap["queries"], 65536, 128)
    if t is None:  # sources changed since the capture: nothing to check
        return
    assert abs(t - (cap["read"] + cap["write"])) < 1.0
    kv = 2.0 * 65536 * 128 * 2
    t8 = bench.attn_traffic(8 * cap["queries"], 65536, 128)
    assert abs(t8 - (8 * (cap["read"] + cap["write"] - kv) + kv)) < 8.0


def test_clock_summary_uses_samples_taken_while_timing():
    c = bench.ClockSampler(0)
    idle = "0, 345, 1965, 100.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    busy = "0, 1965, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active"
    c.lines, c.n0 = [idle, busy, busy], 1
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["samples"] == 2 and s["reasons"] == ["sw_power_cap"]
    c.lines, c.n0 = [idle], 1  # nothing arrived during the timed work: the last sample stands in
    assert c.summary()["samples"] == 1
