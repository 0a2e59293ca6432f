"""Benchmark of the HISA hot path on B200.

One step = one pass of the whole path over the 64K prefill workload: the
indexer (block sums, block selection, token selection) followed by sparse
MQA attention, L=65536, B=128, m=64, k=2048, d_idx=d=128, H=64, seed 0.
`value` is prefill tokens/s (queries processed per second, all ranks).
The decode half of the metric (batch 32 at context 131072, one query per
sequence per step) is measured in the same run and reported under "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hsa|reference]

--impl reference times the CPU oracle on a bounded sample of the same
workload (host cores; rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "prefill tokens/s at 64K and decode queries/s at 128K (index + sparse attn)"
PREFILL = synth.WORKLOADS["prefill_64k"]
DECODE = synth.WORKLOADS["decode_128k_b32"]
L2_FLUSH_BYTES = 512 << 20


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: int):
        self.gpu, self.proc, self.lines = gpu, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # the timed region starts once the sampler is producing samples
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0 and self.proc.poll() is None:
                time.sleep(0.01)
            self.n0 = len(self.lines)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        # samples taken while the timed work ran (the one before it if none)
        during = self.lines[getattr(self, "n0", 0):] or self.lines[-1:]
        for ln in during:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- helpers

_INPUTS = {}


def prefill_inputs():
    if "prefill" not in _INPUTS:
        _INPUTS["prefill"] = synth.prefill_inputs(PREFILL)
    return _INPUTS["prefill"]


def dev_bf16(u16, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(device).view(torch.bfloat16)


def pinned_bf16(u16):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory()


# DRAM traffic of the sparse-attention kernel from one ncu capture (the
# 8192-query case of `bench.py --profile-case attn_last8k`, summarised in
# profiles/sparse_attn_tc_prefill64k_last8k.md): dram__bytes_read.sum +
# dram__bytes_write.sum of one launch. Q, O and the index rows scale with the
# queries; the K/V cache (read once) does not. The figure belongs to the
# kernel sources it was captured from and is reported only while they are
# unchanged.
ATTN_CAPTURE = {"queries": 8192, "read": 236.003328e6, "write": 121.259776e6, "sources": "e6bdb399f8fc50cb"}
ATTN_SOURCES = ("csrc/attn_tc.cu", "csrc/tc.cuh", "csrc/common.cuh")


def source_tag(paths):
    """Hash of the code in `paths` with comments and blank space removed, so
    that only a change of the code itself changes the tag."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in paths:
        with open(f) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def attn_traffic(Lq, L, d):
    pkg = os.path.join(ROOT, "hierarchical_sparse_attention_hisa_b200")
    if source_tag([os.path.join(pkg, f) for f in ATTN_SOURCES]) != ATTN_CAPTURE["sources"]:
        return None
    kv = 2.0 * L * d * 2
    per_q = (ATTN_CAPTURE["read"] + ATTN_CAPTURE["write"] - kv) / ATTN_CAPTURE["queries"]
    return per_q * Lq + kv


def prefill_config(world):
    w = PREFILL
    return {"workload": "prefill_64k", "L": w.L, "Lq": w.Lq, "B": w.B, "m": w.m, "k": w.k,
            "d_idx": w.d_idx, "H": w.H, "d": w.d, "needles": w.needles, "batch": 1,
            "seq_len": w.L, "parallelism": f"replicas x{world}",
            "l2": "flushed (512 MiB write) between timed steps"}


def attn_flops(idx_counts, H, d):
    # QK^T and PV: 2 * 2 * H * d multiply-adds per kept (query, key) pair
    return 4.0 * H * d * float(idx_counts)


def selection_sizes(w, t):
    """Sizes of the two selection stages for queries at positions t (array).

    With nb = t // B + 1 causal blocks, nb <= m keeps every block: no block
    score is needed and all t + 1 causal tokens are candidates. Otherwise the
    blocks 1 .. nb - 2 are scored, and the m kept blocks are m - 1 complete
    blocks (block 0 and the m - 2 best) plus the query's own block cut at t,
    so (m - 1) * B + t % B + 1 tokens are candidates. min(k, candidates) keys
    are kept. Returns (scored blocks, candidate tokens, kept keys)."""
    t = np.asarray(t, dtype=np.int64)
    nb = t // w.B + 1
    pruned = nb > w.m
    blocks = np.where(pruned, nb - 2, 0)
    cand = np.where(pruned, (w.m - 1) * w.B + t % w.B + 1, t + 1)
    return blocks, cand, np.minimum(cand, w.k)


def selection_summary(w, kept):
    """The measured number of kept (query, key) pairs beside the one the
    selection sizes fix, and the indexer's algorithmic work against the flat
    token-level indexer's."""
    wm = work_model(w)
    index_flops = wm["block_score_flops"] + wm["token_score_flops"]
    return {"kept_pairs": int(kept), "kept_pairs_expected": wm["kept_pairs"],
            "index_gflop": index_flops / 1e9, "flat_index_gflop": wm["flat_index_flops"] / 1e9,
            "index_work_ratio_flat_over_hisa": wm["flat_index_flops"] / index_flops}


def work_model(w):
    """Algorithmic work of one prefill step of workload w (queries at
    positions L - Lq .. L - 1): FLOPs of block scoring and token scoring (one
    dot product of length d_idx per scored block or token), of the flat
    token-level indexer the method replaces (every causal token scored), and
    of the attention over the kept keys."""
    t = np.arange(w.L - w.Lq, w.L, dtype=np.int64)
    blocks, cand, kept = selection_sizes(w, t)
    per = 2.0 * w.d_idx
    kept_pairs = int(kept.sum())
    return {"block_score_flops": per * float(blocks.sum()),
            "token_score_flops": per * float(cand.sum()),
            "flat_index_flops": per * float((t + 1).sum()),
            "kept_pairs": kept_pairs,
            "attn_flops": attn_flops(kept_pairs, w.H, w.d)}


# ---------------------------------------------------------------- our arm

def bench_hsa(args, rank, world, device):
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa

    hsa.load()
    w = PREFILL
    x = prefill_inputs()
    q_idx, k_idx = dev_bf16(x["q_idx"], device), dev_bf16(x["k_idx"], device)
    Q, K, V = dev_bf16(x["Q"], device), dev_bf16(x["K"], device), dev_bf16(x["V"], device)
    p = hsa.params(B=w.B, m=w.m, k=w.k, d_idx=w.d_idx, H=w.H, d=w.d)
    ws = torch.empty(hsa.hsa_index_workspace_size(p, w.Lq, w.L), dtype=torch.uint8, device=device)
    idx = torch.empty((w.Lq, w.k), dtype=torch.int32, device=device)
    O = torch.empty((w.Lq, w.H, w.d), dtype=torch.bfloat16, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        hsa.hsa_index(p, w.Lq, w.L, q_idx, k_idx, idx, ws, stream)
        if ev:
            ev[1].record(stream)
        hsa.hsa_sparse_attn(p, w.Lq, w.L, Q, K, V, idx, O, stream)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    kept = int((idx >= 0).sum().item())
    # diagnostic: the planted needles (query i, key j with k_idx[j] = q_idx[i])
    # whose key the selection kept
    needles = x.get("needles", [])
    if needles:
        rows = idx[torch.tensor([i for i, _ in needles], device=device)].cpu().numpy()
        needle_recall = float(np.mean([j in set(r.tolist()) for (_, j), r in zip(needles, rows)]))
    else:
        needle_recall = None

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    launches0 = hsa.kernel_launches()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for s in range(args.steps):
            flush.zero_()          # evict L2 between timed steps (outside the events)
            step(evs[s])
        torch.cuda.synchronize()
    launches = hsa.kernel_launches() - launches0
    if world > 1:
        torch.distributed.barrier()
    t_index = [e[0].elapsed_time(e[1]) for e in evs]
    t_attn = [e[1].elapsed_time(e[2]) for e in evs]
    ms_step = sum(a + b for a, b in zip(t_index, t_attn)) / args.steps
    ms_step = max_over_ranks(ms_step, world, device)
    attn_ms = sum(t_attn) / args.steps
    # rows the CPU-baseline leg checks against the oracle: evenly spaced rows
    # and every needle row, taken from the timed steps' results
    prow = parity_rows(w.Lq, [i for i, _ in needles])
    prow_t = torch.from_numpy(prow).to(device)
    parity_gpu = {"rows": prow, "idx": idx[prow_t].cpu().numpy(),
                  "O": O[prow_t].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)}

    # the indexer's two stages on their own, for the workload's configs entry
    t_block, t_token = time_index_stages(args, w, p, q_idx, k_idx, ws, idx, flush, stream)
    wmh = work_model(w)
    hbm_, tf_, _, src_ = peaks()
    attn_tf_ = wmh["attn_flops"] / (attn_ms / 1e3) / 1e12
    configs_headline = {
        "L": w.L, "Lq": w.Lq, "B": w.B, "m": w.m, "k": w.k, "d_idx": w.d_idx, "H": w.H, "d": w.d,
        "ms_index": sum(t_index) / args.steps, "ms_attn": attn_ms,
        "ms_index_block_stage": t_block, "ms_index_token_stage": t_token,
        "kept_pairs": kept, "kept_pairs_expected": wmh["kept_pairs"],
        "roofline": {"attention": {"bound": "tensor", "achieved": attn_tf_, "peak": tf_, "unit": "TFLOP/s",
                                   "frac": attn_tf_ / tf_, "peak_source": f"{src_} bf16 burst"},
                     **index_rooflines(w, t_block, t_token)},
        "l2": "flushed between steps", "note": "the headline workload: the line's own figures"}

    # end to end through the public API: pinned host inputs -> device, results -> host
    e2e = None
    if not args.skip_e2e:
        hq, hk = pinned_bf16(x["q_idx"]), pinned_bf16(x["k_idx"])
        hQ, hK, hV = pinned_bf16(x["Q"]), pinned_bf16(x["K"]), pinned_bf16(x["V"])
        hO = torch.empty(O.shape, dtype=torch.bfloat16).pin_memory()
        hidx = torch.empty(idx.shape, dtype=torch.int32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hQ, hK, hV))
        d2h = hO.numel() * 2 + hidx.numel() * 4
        O_dev, idx_dev = O.cpu(), idx.cpu()  # the device path's results, to check the host path's

        def timed(fn, n):
            fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / n

        def e2e_copies():
            # the inputs copied in, the two device calls, the results copied out, in turn
            for dst, src in ((q_idx, hq), (k_idx, hk), (Q, hQ), (K, hK), (V, hV)):
                dst.copy_(src, non_blocking=True)
            hsa.hsa_index(p, w.Lq, w.L, q_idx, k_idx, idx, ws, stream)
            hsa.hsa_sparse_attn(p, w.Lq, w.L, Q, K, V, idx, O, stream)
            hO.copy_(O, non_blocking=True)
            hidx.copy_(idx, non_blocking=True)

        n_e2e = max(1, min(args.steps, 3))
        try:
            # one C-ABI call with the host buffers: the copies overlap the kernels
            ws_host = torch.empty(hsa.hsa_prefill_host_workspace_size(p, w.Lq, w.L), dtype=torch.uint8,
                                  device=device)
            ms = timed(lambda: hsa.hsa_prefill_host(p, w.Lq, w.L, hq, hk, hQ, hK, hV, hO, hidx, ws_host,
                                                     stream), n_e2e)
            if not (torch.equal(hO.view(torch.int16), O_dev.view(torch.int16)) and torch.equal(hidx, idx_dev)):
                raise RuntimeError("its results differ from the device path's")
            form = "hsa_prefill_host (host buffers in and out, copies overlapped with the kernels)"
            del ws_host
        except Exception as ex:  # report the serial form rather than no end-to-end number
            ws_host = None
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            ms = timed(e2e_copies, n_e2e)
            form = f"serial copies around hsa_index + hsa_sparse_attn (hsa_prefill_host: {ex})"
        ms = max_over_ranks(ms, world, device)
        e2e = {"value": w.Lq * world / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms, "form": form}
        del hQ, hK, hV, hO, O_dev, idx_dev

    del Q, K, V, O, flush
    torch.cuda.empty_cache()
    dec = None if args.skip_decode else bench_decode(args, world, device)

    hbm, tf, tf_sus, src = peaks()
    flops = attn_flops(kept, w.H, w.d)
    achieved = flops / (attn_ms / 1e3) / 1e12
    res = {
        "metric": METRIC,
        "value": w.Lq * world / (ms_step / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": prefill_config(world),
        "breakdown_ms": {"hsa_index": sum(t_index) / args.steps, "hsa_sparse_attn": attn_ms},
        "needle_recall": needle_recall,
        "selection": selection_summary(PREFILL, kept),
        "roofline": {"kernel": "sparse attention", "bound": "tensor", "achieved": achieved,
                     "peak": tf, "unit": "TFLOP/s", "frac": achieved / tf,
                     "traffic": attn_traffic(w.Lq, w.L, w.d),
                     "peak_source": f"{src} bf16 burst",
                     "flops_per_launch": flops},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "e2e": e2e,
        "decode": dec,
        "_parity_gpu": parity_gpu,  # taken out before the line is printed
        "configs_headline": configs_headline,  # becomes the headline's entry of `configs`
    }
    return res


def bench_decode(args, world, device, w=None):
    """Decode: batch 32 sequences at context 131072 (or workload w's batch and
    context), one query each per step."""
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa

    w = DECODE if w is None else w
    steps = max(2, min(args.decode_steps, w.decode_steps))
    warm = min(args.warmup, 8)
    cap = w.decode_ctx + warm + steps + w.B
    cap = (cap + w.B - 1) // w.B * w.B
    x = synth.decode_inputs(w, w.decode_ctx, cap, warm + steps)
    p = hsa.params(B=w.B, m=w.m, k=w.k, d_idx=w.d_idx, H=w.H, d=w.d)
    kc, Kc, Vc = (dev_bf16(x[n], device) for n in ("k_idx_cache", "K_cache", "V_cache"))
    ksum = torch.zeros((w.batch, cap // w.B, w.d_idx), dtype=torch.float32, device=device)
    for b in range(w.batch):
        hsa.hsa_block_sums(p, w.decode_ctx, kc[b], ksum[b])
    ctx = torch.full((w.batch,), w.decode_ctx, dtype=torch.int32, device=device)
    new = {n: dev_bf16(x[n], device) for n in ("q_idx_new", "k_idx_new", "Q_new", "K_new", "V_new")}
    ws = torch.empty(hsa.hsa_decode_workspace_size(p, w.batch, cap), dtype=torch.uint8, device=device)
    O = torch.empty((w.batch, w.H, w.d), dtype=torch.bfloat16, device=device)
    idx = torch.empty((w.batch, w.k), dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()

    def step(s):
        # launched on the current stream: the capture stream inside the graph
        hsa.hsa_decode_step(p, w.batch, cap, ctx, kc, Kc, Vc, ksum, new["q_idx_new"][s],
                            new["k_idx_new"][s], new["Q_new"][s], new["K_new"][s], new["V_new"][s],
                            O, idx, ws, None)

    for s in range(warm):
        step(s)
    torch.cuda.synchronize()
    # the timed steps run twice over fresh input rows: as direct launches (the
    # step's kernels are programmatic dependent launches, so each launch
    # overlaps its predecessor) and captured once into a CUDA graph that is
    # replayed, as a serving loop would; the faster form is the reported value
    half = max(1, steps // 2)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = hsa.kernel_launches()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    a.record(stream)
    for s in range(warm, warm + half):
        step(s)
    b.record(stream)
    torch.cuda.synchronize()
    launches = hsa.kernel_launches() - launches0
    ms_direct = max_over_ranks(a.elapsed_time(b) / half, world, device)
    warm += half
    steps -= half
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for s in range(warm, warm + steps):
            step(s)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    stream = torch.cuda.current_stream()
    a.record(stream)
    graph.replay()
    b.record(stream)
    torch.cuda.synchronize()
    ms_graph = max_over_ranks(a.elapsed_time(b) / steps, world, device)
    del graph
    # every step ran: each sequence grew by one token per step
    assert int(ctx.min().item()) == int(ctx.max().item()) == w.decode_ctx + warm + steps, "decode steps did not all run"
    ms = min(ms_direct, ms_graph)
    timing = "direct launches, CUDA events" if ms_direct <= ms_graph else "CUDA graph replay, CUDA events"
    hbm, _, _, src = peaks()
    # algorithmic bytes per query: block sums read + kept blocks' index keys +
    # kept K/V rows + Q and O rows
    per_q = (w.decode_ctx // w.B) * w.d_idx * 4 + w.m * w.B * w.d_idx * 2 + w.k * w.d * 2 * 2 \
        + 2 * w.H * w.d * 2
    gbs = per_q * w.batch / (ms / 1e3) / 1e9
    label = "decode queries/s at 128K" if w is DECODE else \
        f"decode queries/s ({w.name}: batch {w.batch}, context {w.decode_ctx})"
    return {"metric": label, "value": w.batch * world / (ms / 1e3),
            "unit": "queries/s", "ms_per_step": ms, "steps_direct": half, "steps_graph": steps,
            "batch": w.batch,
            "ctx": w.decode_ctx, "timing": timing,
            "ms_per_step_direct_launch": ms_direct, "ms_per_step_graph": ms_graph,
            "gpu_launches_per_step": int(launches) // half,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm,
                                              "unit": "GB/s", "frac": gbs / hbm,
                                              "peak_source": src,
                                              "bytes_per_query": per_q}}


def max_over_ranks(v, world, device):
    if world <= 1:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- oracle arm

def parity_rows(Lq, extra=(), n=64):
    """n evenly spaced query rows of [0, Lq) plus the rows in `extra`, ascending."""
    r = set(np.linspace(0, Lq - 1, n).astype(np.int64).tolist()) | {int(i) for i in extra}
    return np.array(sorted(r), dtype=np.int64)


def parity_summary(idx_gpu, O_gpu_bits, idx_ref, O_ref, max_abs=2e-2, mean_abs=2e-3):
    """Rows whose indices differ at all, and the attention error of bf16 O
    (bit patterns) against the oracle's fp64 O, with the pass/fail verdict."""
    mism = int(np.sum(np.any(np.asarray(idx_gpu) != np.asarray(idx_ref), axis=1)))
    got = (np.asarray(O_gpu_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    err = np.abs(got - np.asarray(O_ref, dtype=np.float64))
    return {"rows": int(np.asarray(idx_gpu).shape[0]), "index_rows_mismatched": mism,
            "attn_max_abs": float(err.max()), "attn_mean_abs": float(err.mean()),
            "tolerance": {"max_abs": max_abs, "mean_abs": mean_abs},
            "ok": bool(mism == 0 and err.max() <= max_abs and err.mean() <= mean_abs)}


def parity_check(gpu):
    """The oracle on the rows bench_hsa kept from the timed steps, compared
    with what the GPU computed for them."""
    import oracle
    w = PREFILL
    x = prefill_inputs()
    threads = oracle.default_threads()
    idx = oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, w.k, rows=gpu["rows"], threads=threads)
    O = oracle.sparse_attn(x["Q"], x["K"], x["V"], idx, rows=gpu["rows"], threads=threads)
    return parity_summary(gpu["idx"], gpu["O"], idx, O)


def oracle_sample(target_s=15.0, w=None, x=None):
    """Time the oracle (index + attention) on a bounded sample of query rows
    of the 64K workload (or workload w with inputs x); returns (tokens/s,
    threads, description)."""
    import oracle
    if w is None:
        w, x = PREFILL, prefill_inputs()
    threads = oracle.default_threads()
    rows = np.linspace(0, w.Lq - 1, 8 * threads).astype(np.int64)
    t0 = time.perf_counter()
    idx = oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, w.k, rows=rows, threads=threads)
    oracle.sparse_attn(x["Q"], x["K"], x["V"], idx, rows=rows, threads=threads)
    dt = time.perf_counter() - t0
    n = len(rows)
    if dt < target_s:   # grow the sample towards the target duration
        n = int(min(w.Lq, max(n, n * target_s / max(dt, 1e-3))))
        rows = np.linspace(0, w.Lq - 1, n).astype(np.int64)
        t0 = time.perf_counter()
        idx = oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, w.k, rows=rows, threads=threads)
        oracle.sparse_attn(x["Q"], x["K"], x["V"], idx, rows=rows, threads=threads)
        dt = time.perf_counter() - t0
    return n / dt, threads, f"{n} evenly spaced query rows of {w.name} (index + attention), {dt:.1f} s"


def bench_reference(args, rank, world):
    if rank != 0:
        return None
    vals = []
    desc = threads = None
    for s in range(args.warmup + args.steps):
        # each step a bounded sample: the whole run stays near two and a half minutes
        per_step = min(10.0, 150.0 / max(1, args.warmup + args.steps))
        v, threads, desc = oracle_sample(target_s=float(os.environ.get("HSA_ORACLE_SECONDS", str(per_step))))
        if s >= args.warmup:
            vals.append(v)
    v = statistics.mean(vals)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            # the time a whole 65,536-query step would take at the sampled rate
            "ms_per_step": PREFILL.Lq / v * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64",
            "data": "synthetic", "config": prefill_config(world),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- every workload

def time_index_stages(args, w, p, q_idx, k_idx, ws, idx, flush, stream):
    """The indexer's two selection stages timed on their own through the
    stage entry points hsa_index chains (L2 flushed before each pass):
    block stage = block sums + block scoring + top-m, token stage = token
    scoring + top-k. Returns their mean times in ms."""
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa

    device = q_idx.device
    ksum = torch.empty((max(w.L // w.B, 1), w.d_idx), dtype=torch.float32, device=device)
    blocks = torch.empty((w.Lq, w.m), dtype=torch.int32, device=device)
    steps = max(1, args.steps)
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for s in range(args.warmup + steps):
        ev = sev[s - args.warmup] if s >= args.warmup else None
        flush.zero_()
        if ev:
            ev[0].record(stream)
        hsa.hsa_block_sums(p, w.L, k_idx, ksum, stream)
        hsa.hsa_select_blocks(p, w.Lq, w.L, q_idx, ksum, blocks, ws, stream)
        if ev:
            ev[1].record(stream)
        hsa.hsa_select_tokens(p, w.Lq, w.L, q_idx, k_idx, blocks, idx, ws, stream)
        if ev:
            ev[2].record(stream)
    torch.cuda.synchronize()
    return (statistics.mean(e[0].elapsed_time(e[1]) for e in sev),
            statistics.mean(e[1].elapsed_time(e[2]) for e in sev))


def index_rooflines(w, t_block, t_token):
    """Roofline entries of the indexer's two stages (see time_index_stages)."""
    hbm, tf, _, src = peaks()
    wm = work_model(w)
    block_tf = 3 * wm["block_score_flops"] / (t_block / 1e3) / 1e12
    # token scoring's algorithmic bytes: the d_idx bf16 values of every
    # candidate key each query scores (one dot product per candidate, so the
    # same count as its FLOPs); reuse through L2 can carry this past HBM peak
    token_gbs = wm["token_score_flops"] / (t_token / 1e3) / 1e9
    return {
        "block_stage": {"bound": "tensor", "achieved": block_tf, "peak": tf, "unit": "TFLOP/s",
                        "frac": block_tf / tf, "peak_source": f"{src} bf16 burst",
                        "note": "three bf16 planes of the fp32 block sums, so 3x the block-score FLOPs; "
                                "the stage time includes the block sums and the top-m"},
        "token_stage": {"bound": "hbm", "achieved": token_gbs, "peak": hbm, "unit": "GB/s",
                        "frac": token_gbs / hbm, "peak_source": f"{src} copy",
                        "note": "effective: candidate keys' bytes / stage time (MMA reuse through L2 "
                                "can carry it past HBM peak); the stage time includes the top-k"}}


def time_prefill(args, w, x, device, flush, stream):
    """One prefill workload timed as index + attention steps (L2 flushed
    between steps), plus the index's two selection stages timed on their own
    (block stage: block sums + block scoring + top-m; token stage: token
    scoring + top-k, through the stage entry points hsa_index chains).
    Returns the workload's entry of the bench line's `configs` object."""
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa

    hbm, tf, _, src = peaks()
    q_idx, k_idx = dev_bf16(x["q_idx"], device), dev_bf16(x["k_idx"], device)
    Q, K, V = (dev_bf16(x[n], device) for n in ("Q", "K", "V"))
    p = hsa.params(B=w.B, m=w.m, k=w.k, d_idx=w.d_idx, H=w.H, d=w.d)
    ws = torch.empty(hsa.hsa_index_workspace_size(p, w.Lq, w.L), dtype=torch.uint8, device=device)
    idx = torch.empty((w.Lq, w.k), dtype=torch.int32, device=device)
    O = torch.empty((w.Lq, w.H, w.d), dtype=torch.bfloat16, device=device)
    steps = max(1, args.steps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for s in range(args.warmup + steps):
        ev = evs[s - args.warmup] if s >= args.warmup else None
        flush.zero_()
        if ev:
            ev[0].record(stream)
        hsa.hsa_index(p, w.Lq, w.L, q_idx, k_idx, idx, ws, stream)
        if ev:
            ev[1].record(stream)
        hsa.hsa_sparse_attn(p, w.Lq, w.L, Q, K, V, idx, O, stream)
        if ev:
            ev[2].record(stream)
    torch.cuda.synchronize()
    t_index = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_attn = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    wm = work_model(w)
    kept = int((idx >= 0).sum().item())
    attn_tf = wm["attn_flops"] / (t_attn / 1e3) / 1e12
    index_flops = wm["block_score_flops"] + wm["token_score_flops"]
    t_block, t_token = time_index_stages(args, w, p, q_idx, k_idx, ws, idx, flush, stream)
    res = {
        "L": w.L, "Lq": w.Lq, "B": w.B, "m": w.m, "k": w.k, "d_idx": w.d_idx, "H": w.H, "d": w.d,
        "value": w.Lq / ((t_index + t_attn) / 1e3), "unit": "tokens/s",
        "ms_per_step": t_index + t_attn, "ms_index": t_index, "ms_attn": t_attn,
        "ms_index_block_stage": t_block, "ms_index_token_stage": t_token,
        "kept_pairs": kept, "kept_pairs_expected": wm["kept_pairs"],
        "roofline": {
            "attention": {"bound": "tensor", "achieved": attn_tf, "peak": tf, "unit": "TFLOP/s",
                          "frac": attn_tf / tf, "peak_source": f"{src} bf16 burst"},
            **index_rooflines(w, t_block, t_token)},
        "index_gflop": index_flops / 1e9, "flat_index_gflop": wm["flat_index_flops"] / 1e9,
        "index_work_ratio_flat_over_hisa": wm["flat_index_flops"] / index_flops,
        "l2": "flushed between steps"}
    del q_idx, k_idx, Q, K, V, ws, idx, O
    torch.cuda.empty_cache()
    return res


def bench_configs(args, device, headline=None):
    """Every workload but the headline one, timed on its own: the prefill
    workloads (2K, 16K, the last 8192 queries of the 1M context) as index +
    attention steps, then the 64 batch-1 decode steps after the 1M context.
    Each entry also checks its number of kept (query, key) pairs against the
    selection sizes the method fixes, and carries a bounded oracle sample of
    the same workload (host cores). Returns {workload: entry}."""
    import torch

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    out = {}
    for name in ("tiny_prefill_2k", "prefill_16k", "prefill_64k", "prefill_1m_last8k"):
        if name == PREFILL.name and headline is not None:
            out[name] = headline
            continue
        w = synth.WORKLOADS[name]
        x = synth.prefill_inputs(w)
        res = time_prefill(args, w, x, device, flush, stream)
        if not args.skip_cpu_baseline:  # the oracle on a bounded sample of the same workload
            v, threads, desc = oracle_sample(target_s=float(os.environ.get("HSA_ORACLE_SECONDS_CFG", "5")), w=w, x=x)
            res["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                   "sample": desc}
        out[name] = res
        del x
    del flush
    torch.cuda.empty_cache()
    out["prefill_1m_last8k_decode"] = bench_decode(args, 1, device, synth.WORKLOADS["prefill_1m_last8k"])
    out["flat_indexer_64k"] = bench_flat_indexer(args, device, headline)
    return out


def bench_flat_indexer(args, device, headline=None):
    """The token-level indexer the method replaces (the pages' comparison):
    the same library with every causal block kept (m = all 512 blocks of the
    64K workload), so every causal token of a query is scored and the top-k
    taken over all of them. Timed like the hierarchical indexer (L2 flushed
    between calls) and reported beside it."""
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa

    w = PREFILL
    x = synth.prefill_inputs(w, with_attn=False)
    q_idx, k_idx = dev_bf16(x["q_idx"], device), dev_bf16(x["k_idx"], device)
    m_flat = w.L // w.B
    p = hsa.params(B=w.B, m=m_flat, k=w.k, d_idx=w.d_idx, H=w.H, d=w.d)
    ws = torch.empty(hsa.hsa_index_workspace_size(p, w.Lq, w.L), dtype=torch.uint8, device=device)
    idx = torch.empty((w.Lq, w.k), dtype=torch.int32, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    steps = max(1, min(args.steps, 3))
    ts = []
    for s in range(args.warmup + steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        hsa.hsa_index(p, w.Lq, w.L, q_idx, k_idx, idx, ws, stream)
        b.record(stream)
        torch.cuda.synchronize()
        if s >= args.warmup:
            ts.append(a.elapsed_time(b))
    ms = statistics.mean(ts)
    wm = work_model(w)
    res = {"m": m_flat, "ms_index": ms, "index_gflop": wm["flat_index_flops"] / 1e9,
           "workspace_bytes": int(ws.numel())}
    if headline is not None and headline.get("ms_index"):
        res["ms_index_hisa"] = headline["ms_index"]
        res["speedup_hisa_over_flat"] = ms / headline["ms_index"]
    res["note"] = ("context, not a target: the HISA page reports up to 3.75x over the DSA indexer at 64K "
                   "(hardware not stated)")
    del ws, idx, q_idx, k_idx, flush
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- variants

def bench_variants(device):
    """The comparisons the pages draw, as parameter settings of the same
    path, one JSON line each (not the headline line):
    - the flat token-level indexer (every causal block kept, m = all blocks)
      against the hierarchical one, at 16K where every block fits the
      candidate limit;
    - pure block-sparse attention: every token of the top-m blocks (k = m*B,
      so the token stage keeps all candidates);
    - a (B, m) sweep of the indexer at 64K with k = 2048.
    Times are CUDA-event means of three calls after two warm-up calls."""
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa

    hsa.load()
    stream = torch.cuda.current_stream()

    def timed(fn, n=3):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    def run(name, w, x, B, m, k, attn, comment):
        p = hsa.params(B=B, m=m, k=k, d_idx=w.d_idx, H=w.H, d=w.d)
        q_idx, k_idx = dev_bf16(x["q_idx"], device), dev_bf16(x["k_idx"], device)
        ws = torch.empty(max(16, hsa.hsa_index_workspace_size(p, w.Lq, w.L)), dtype=torch.uint8, device=device)
        idx = torch.empty((w.Lq, k), dtype=torch.int32, device=device)
        t_index = timed(lambda: hsa.hsa_index(p, w.Lq, w.L, q_idx, k_idx, idx, ws, stream))
        res = {"variant": name, "workload": w.name, "L": w.L, "Lq": w.Lq, "B": B, "m": m, "k": k,
               "index_ms": t_index, "note": comment}
        if x.get("needles"):
            rows = idx[torch.tensor([i for i, _ in x["needles"]], device=device)].cpu().numpy()
            res["needle_recall"] = float(np.mean([j in set(r.tolist()) for (_, j), r in zip(x["needles"], rows)]))
        del ws
        if attn:
            Q, K, V = (dev_bf16(x[n], device) for n in ("Q", "K", "V"))
            O = torch.empty((w.Lq, w.H, w.d), dtype=torch.bfloat16, device=device)
            res["attn_ms"] = timed(lambda: hsa.hsa_sparse_attn(p, w.Lq, w.L, Q, K, V, idx, O, stream))
            res["tokens_per_s"] = w.Lq / ((t_index + res["attn_ms"]) / 1e3)
            del Q, K, V, O
        del idx, q_idx, k_idx
        torch.cuda.empty_cache()
        print(json.dumps(res), flush=True)

    w16 = synth.WORKLOADS["prefill_16k"]
    x16 = synth.prefill_inputs(w16, with_attn=False)
    nb16 = w16.L // w16.B
    run("hierarchical_16k", w16, x16, w16.B, w16.m, w16.k, False, "HISA indexer, m = 32 of 128 blocks")
    run("flat_16k", w16, x16, w16.B, nb16, w16.k, False, "flat token-level indexer: every block kept")
    del x16
    w = PREFILL
    x = prefill_inputs()
    run("hierarchical_64k", w, x, w.B, w.m, w.k, True, "the headline configuration")
    run("block_sparse_64k", w, x, w.B, w.m, w.m * w.B, True, "every token of the top-m blocks, no token stage")
    for B, m in ((64, 16), (64, 32), (64, 64), (64, 128), (128, 16), (128, 32), (128, 64), (128, 128),
                 (256, 32), (256, 64)):
        run(f"sweep_B{B}_m{m}", w, x, B, m, w.k, False, "(B, m) sweep of the indexer")


# ---------------------------------------------------------------- profiling cases

def profile_case(name):
    """Small cases for ncu captures: the last 8192 queries of the 64K workload
    (inputs larger than L2), run three times untimed and once timed; or
    decode_128k: 12 steps of the batch-32 decode at context 131072 (the
    caches, about 3.3 GB, far larger than L2)."""
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa
    hsa.load()
    if name == "decode_128k":
        class A:  # the decode bench's arguments
            decode_steps, warmup = 4, 8
        torch.cuda.set_device(0)
        dec = bench_decode(A(), 1, torch.device("cuda", 0))
        print(json.dumps({"profile_case": name, "ms_per_step": dec["ms_per_step"]}))
        return
    w = PREFILL
    lq = 8192
    x = synth.prefill_inputs(w, with_attn=(name == "attn_last8k"))
    dev = lambda u: dev_bf16(u, "cuda")  # noqa: E731
    q_idx, k_idx = dev(x["q_idx"][-lq:]), dev(x["k_idx"])
    p = hsa.params(B=w.B, m=w.m, k=w.k, d_idx=w.d_idx, H=w.H, d=w.d)
    ws = torch.empty(hsa.hsa_index_workspace_size(p, lq, w.L), dtype=torch.uint8, device="cuda")
    idx = torch.empty((lq, w.k), dtype=torch.int32, device="cuda")
    if name == "attn_last8k":
        Q, K, V = dev(x["Q"][-lq:]), dev(x["K"]), dev(x["V"])
        O = torch.empty_like(Q)
        hsa.hsa_index(p, lq, w.L, q_idx, k_idx, idx, ws)
        run = lambda: hsa.hsa_sparse_attn(p, lq, w.L, Q, K, V, idx, O)  # noqa: E731
    else:
        run = lambda: hsa.hsa_index(p, lq, w.L, q_idx, k_idx, idx, ws)  # noqa: E731
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    run()
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "ms": a.elapsed_time(b)}))


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="hsa", choices=["hsa", "reference"])
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-configs", action="store_true",
                    help="leave out the other workloads' entries (configs) of the line")
    ap.add_argument("--variants", action="store_true",
                    help="time the flat indexer, block-sparse attention and a (B, m) sweep, then exit")
    ap.add_argument("--configs", action="store_true",
                    help="time every workload (2K, 16K, 64K, 1M-context chunk and its decode), then exit")
    ap.add_argument("--profile-case", choices=["attn_last8k", "index_last8k", "decode_128k"],
                    help="run one small case for an ncu capture and exit")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if args.variants:
        import torch
        bench_variants(torch.device("cuda", 0))
        return
    if args.configs:
        import torch
        torch.cuda.set_device(0)
        import hierarchical_sparse_attention_hisa_b200 as hsa
        hsa.load()
        for name, entry in bench_configs(args, torch.device("cuda", 0)).items():
            print(json.dumps(dict(entry, workload=name)), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = bench_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    res = bench_hsa(args, rank, world, device)
    parity_gpu = res.pop("_parity_gpu", None)
    import hierarchical_sparse_attention_hisa_b200 as hsa
    # A bounded device wait that gave up leaves its launch's work undone, so
    # the line says whether every wait of the run (on every rank) completed.
    try:
        status = float(hsa.hsa_device_status(reset=True) != 0)
    except hsa.HSAError as ex:  # the check itself failed: say so, keep the line
        status, res["device_waits_error"] = -1.0, str(ex)
    gave_up = max_over_ranks(status, world, device)
    res["device_waits"] = ("a bounded wait gave up: outputs incomplete" if gave_up > 0 else
                           "all completed" if gave_up == 0 else "not checked")
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        v, threads, desc = oracle_sample(target_s=float(os.environ.get("HSA_ORACLE_SECONDS", "15")))
        res["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                               "sample": desc}
        if parity_gpu is not None:
            # the timed steps' results against the oracle on a fixed set of rows
            try:
                res["parity_sample"] = parity_check(parity_gpu)
            except Exception as ex:  # the line is still printed, saying why the check is missing
                res["parity_sample"] = {"error": f"{type(ex).__name__}: {ex}"}
    if world == 1 and not args.skip_configs:
        # the other workloads, each on its own (one GPU only: the headline
        # numbers above are what the replicas of a multi-GPU run measure)
        head = {k: res[k] for k in ("value", "unit", "ms_per_step")}
        head.update(res.get("configs_headline", {}))
        res["configs"] = bench_configs(args, device, headline=head)
    res.pop("configs_headline", None)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
