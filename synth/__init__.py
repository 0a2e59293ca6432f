"""Seeded synthetic inputs for hierarchical indexed sparse attention (HISA).

This module is shared by the CPU oracle's tests and by the GPU benchmark. It
holds only random-number generation, bf16 encoding and the workload table;
none of the method's arithmetic (pooling, scoring, selection, softmax) lives
here.

Workloads follow the shapes the HISA page describes (page "HISA: Hierarchical
Indexed Sparse Attention", sections 第一步 / 第二步: blocks of B=128 tokens,
m=64 kept blocks, k kept tokens, 64K-1M contexts). The pages evaluate on
LongBench and needle-in-a-haystack with trained DeepSeek-V3.2 / GLM-5 weights;
none of that is available, so these seeded synthetic tensors stand in:

* indexer queries / keys: integers uniform in [-8, 8] stored as bf16, so every
  fp32 score is an exact integer and selected indices are bit-comparable;
* attention Q / K / V: N(0, 1) rounded to bf16 (round-to-nearest-even);
* optional planted "needles": a key row set equal to a later query row.

Every tensor is generated in fixed-size chunks, each chunk from its own
``numpy.random.SeedSequence((seed, tensor_id, chunk))`` stream, so the values do
not depend on how many threads fill them.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK = 1 << 22  # elements per independently seeded chunk

# Stable tensor ids: the stream a tensor draws from never changes.
T_Q_IDX, T_K_IDX, T_Q, T_K, T_V, T_NEEDLE = 1, 2, 3, 4, 5, 6
T_DEC_Q_IDX, T_DEC_K_IDX, T_DEC_Q, T_DEC_K, T_DEC_V = 11, 12, 13, 14, 15


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
    return (b >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _fill(shape, seed: int, tensor_id: int, kind: str, threads: int = 8) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nchunks = (n + CHUNK - 1) // CHUNK

    def work(c):
        lo, hi = c * CHUNK, min(n, (c + 1) * CHUNK)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence((seed, tensor_id, c))))
        if kind == "int":
            v = rng.integers(-8, 9, size=hi - lo, dtype=np.int32).astype(np.float32)
        else:
            v = rng.standard_normal(size=hi - lo, dtype=np.float32)
        out[lo:hi] = f32_to_bf16_bits(v)

    if nchunks <= 1 or threads <= 1:
        for c in range(nchunks):
            work(c)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def int_bf16(shape, seed: int, tensor_id: int) -> np.ndarray:
    """Integers uniform in [-8, 8], as bf16 bit patterns (exact)."""
    return _fill(shape, seed, tensor_id, "int")


def normal_bf16(shape, seed: int, tensor_id: int) -> np.ndarray:
    """Standard normal values rounded to bf16, as bit patterns."""
    return _fill(shape, seed, tensor_id, "normal")


def plant_needles(q_idx: np.ndarray, k_idx: np.ndarray, Lk: int, B: int, m: int,
                  count: int, seed: int):
    """Copy ``count`` query rows onto earlier key rows (in place on ``k_idx``).

    Needle query positions i are distinct and drawn uniformly from [B*m, Lk);
    each gets a distinct key position j drawn uniformly from [0, i-1], and
    k_idx[j] := q_idx[i]. Queries are assumed to be positions 0..Lk-1.
    Returns the list of (i, j) pairs.
    """
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence((seed, T_NEEDLE))))
    lo = min(B * m, Lk - 1)
    qs = rng.choice(np.arange(lo, Lk), size=count, replace=False)
    used, pairs = set(), []
    for i in sorted(int(v) for v in qs):
        while True:
            j = int(rng.integers(0, i))
            if j not in used:
                break
        used.add(j)
        k_idx[j] = q_idx[i]
        pairs.append((i, j))
    return pairs


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    L: int            # context length (keys) for prefill
    Lq: int           # number of queries (the last Lq positions)
    B: int
    m: int
    k: int
    d_idx: int
    H: int
    d: int
    needles: int = 0
    batch: int = 1
    decode_ctx: int = 0    # decode: cached tokens per sequence before step 0
    decode_steps: int = 0
    seed: int = 0


# The five workloads: a tiny prefill, 16K and 64K prefill, batch-32 decode at
# 128K, and the last 8192 queries of a 1M context (plus 64 decode steps there).
WORKLOADS = {
    "tiny_prefill_2k": Workload("tiny_prefill_2k", L=2048, Lq=2048, B=64, m=8, k=256,
                                d_idx=64, H=4, d=64),
    "prefill_16k": Workload("prefill_16k", L=16384, Lq=16384, B=128, m=32, k=2048,
                            d_idx=128, H=16, d=128),
    "prefill_64k": Workload("prefill_64k", L=65536, Lq=65536, B=128, m=64, k=2048,
                            d_idx=128, H=64, d=128, needles=32),
    "decode_128k_b32": Workload("decode_128k_b32", L=131072, Lq=1, B=128, m=64, k=2048,
                                d_idx=128, H=64, d=128, batch=32, decode_ctx=131072,
                                decode_steps=256),
    "prefill_1m_last8k": Workload("prefill_1m_last8k", L=1 << 20, Lq=8192, B=128, m=64,
                                  k=2048, d_idx=128, H=64, d=128, batch=1,
                                  decode_ctx=1 << 20, decode_steps=64),
}


def prefill_inputs(w: Workload, seed: int | None = None, with_attn: bool = True):
    """Indexer and attention inputs of a prefill workload, as bf16 bit arrays.

    Returns a dict with q_idx [Lq][d_idx], k_idx [L][d_idx] and, if with_attn,
    Q [Lq][H][d], K [L][d], V [L][d]; plus 'needles' (list of (i, j)).
    """
    s = w.seed if seed is None else seed
    q_full_rows = w.L if w.needles else w.Lq
    q_idx = int_bf16((q_full_rows, w.d_idx), s, T_Q_IDX)
    k_idx = int_bf16((w.L, w.d_idx), s, T_K_IDX)
    needles = []
    if w.needles:
        needles = plant_needles(q_idx, k_idx, w.L, w.B, w.m, w.needles, s)
        q_idx = q_idx[w.L - w.Lq:]
    out = {"q_idx": np.ascontiguousarray(q_idx), "k_idx": k_idx, "needles": needles}
    if with_attn:
        out["Q"] = normal_bf16((w.Lq, w.H, w.d), s, T_Q)
        out["K"] = normal_bf16((w.L, w.d), s, T_K)
        out["V"] = normal_bf16((w.L, w.d), s, T_V)
    return out


def decode_inputs(w: Workload, ctx: int, capacity: int, steps: int, seed: int | None = None):
    """Decode caches (first ``ctx`` rows filled) and per-step new-token rows.

    Caches: k_idx [batch][capacity][d_idx], K/V [batch][capacity][d].
    New tokens for every step: q_idx_new/k_idx_new [steps][batch][d_idx],
    Q_new [steps][batch][H][d], K_new/V_new [steps][batch][d].
    """
    s = w.seed if seed is None else seed
    bt = w.batch
    kc = np.zeros((bt, capacity, w.d_idx), dtype=np.uint16)
    Kc = np.zeros((bt, capacity, w.d), dtype=np.uint16)
    Vc = np.zeros((bt, capacity, w.d), dtype=np.uint16)
    for b in range(bt):
        kc[b, :ctx] = int_bf16((ctx, w.d_idx), s * 1000 + b, T_K_IDX)
        Kc[b, :ctx] = normal_bf16((ctx, w.d), s * 1000 + b, T_K)
        Vc[b, :ctx] = normal_bf16((ctx, w.d), s * 1000 + b, T_V)
    return {
        "k_idx_cache": kc, "K_cache": Kc, "V_cache": Vc,
        "q_idx_new": int_bf16((steps, bt, w.d_idx), s, T_DEC_Q_IDX),
        "k_idx_new": int_bf16((steps, bt, w.d_idx), s, T_DEC_K_IDX),
        "Q_new": normal_bf16((steps, bt, w.H, w.d), s, T_DEC_Q),
        "K_new": normal_bf16((steps, bt, w.d), s, T_DEC_K),
        "V_new": normal_bf16((steps, bt, w.d), s, T_DEC_V),
    }
