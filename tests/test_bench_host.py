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


def _tiny(L, Lq, B, m, k, d_idx=4):
    import synth
    return synth.Workload("t", L=L, Lq=Lq, B=B, m=m, k=k, d_idx=d_idx, H=2, d=8)


def test_selection_sizes_match_the_oracle():
    """Kept keys per row (and, with k above every candidate count, the
    candidate tokens per row) from the closed form equal the oracle's counts."""
    import numpy as np
    import oracle
    import synth
    for (L, Lq, B, m, k, seed) in [(64, 64, 4, 3, 5, 1), (97, 40, 8, 2, 11, 2), (128, 128, 16, 4, 24, 3),
                                   (50, 50, 5, 20, 7, 4)]:
        w = _tiny(L, Lq, B, m, k)
        q = synth.int_bf16((Lq, w.d_idx), seed, 0)
        kk = synth.int_bf16((L, w.d_idx), seed, 1)
        t = np.arange(L - Lq, L)
        _, cand, kept = bench.selection_sizes(w, t)
        got = (oracle.index(q, kk, B, m, k, threads=2) >= 0).sum(axis=1)
        assert np.array_equal(got, kept), (L, Lq, B, m, k)
        got_all = (oracle.index(q, kk, B, m, L, threads=2) >= 0).sum(axis=1)
        assert np.array_equal(got_all, cand), (L, Lq, B, m, k)


def test_work_model_closed_forms():
    """64K workload: every token scored by the flat indexer gives d_idx*L*(L+1)
    FLOPs; the hierarchical token stage scores all t + 1 tokens below m*B and
    (m-1)*B + t%B + 1 from there on; block scoring covers blocks 1..nb-2."""
    import synth
    w = synth.WORKLOADS["prefill_64k"]
    L, B, m, d = w.L, w.B, w.m, w.d_idx
    wm = bench.work_model(w)
    assert wm["flat_index_flops"] == d * L * (L + 1)
    mB = m * B
    n_after = L - mB
    cand = mB * (mB + 1) // 2 + n_after * ((m - 1) * B + 1) + (n_after // B) * (B * (B - 1) // 2)
    assert wm["token_score_flops"] == 2 * d * cand
    # blocks b = m .. L/B - 1 hold B queries each, scoring b - 1 blocks
    blocks = sum(B * (b - 1) for b in range(m, L // B))
    assert wm["block_score_flops"] == 2 * d * blocks
    ratio = wm["flat_index_flops"] / (wm["token_score_flops"] + wm["block_score_flops"])
    assert 4.1 < ratio < 4.25  # the complexity paragraph's L / (L/B + m*B) regime
    assert wm["kept_pairs"] == sum(min(w.k, c) for c in
                                   list(range(1, mB + 1)) + [(m - 1) * B + (t % B) + 1 for t in range(mB, L)])


def test_work_model_of_a_query_chunk():
    import synth
    w = synth.WORKLOADS["prefill_1m_last8k"]
    wm = bench.work_model(w)
    L, Lq, d = w.L, w.Lq, w.d_idx
    assert wm["flat_index_flops"] == d * (L * (L + 1) - (L - Lq) * (L - Lq + 1))
    assert wm["kept_pairs"] == Lq * w.k  # far past m*B every row keeps k


def test_parity_rows_and_summary():
    import numpy as np
    rows = bench.parity_rows(65536, [5, 70000 - 10000, 0])
    assert rows[0] == 0 and rows[-1] == 65535 and 5 in rows and 60000 in rows
    assert np.all(np.diff(rows) > 0)
    idx = np.arange(12, dtype=np.int32).reshape(3, 4)
    ref_O = np.array([[[1.0, -2.0]], [[0.5, 0.25]], [[0.0, 3.0]]])
    bits = (ref_O.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)  # exact in bf16
    s = bench.parity_summary(idx, bits, idx.copy(), ref_O)
    assert s["ok"] and s["index_rows_mismatched"] == 0 and s["attn_max_abs"] == 0.0
    bad = idx.copy()
    bad[1, 2] += 1
    s = bench.parity_summary(bad, bits, idx, ref_O + np.array([[[0.0, 0.05]], [[0.0, 0.0]], [[0.0, 0.0]]]))
    assert not s["ok"] and s["index_rows_mismatched"] == 1 and abs(s["attn_max_abs"] - 0.05) < 1e-12
