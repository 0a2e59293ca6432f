"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Selected indices and block lists must match bit for bit (integer-valued
indexer inputs make every fp32 score exact); attention outputs must be within
max-abs 2e-2 / mean-abs 2e-3 of the oracle's fp64 result.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_attn_close, dev, host_bits, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hsa():
    import torch
    import hierarchical_sparse_attention_hisa_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.build()
    m.load()
    return m


def run_index(hsa, q, k, B, m, kk):
    import torch
    out = hsa.index(dev(q), dev(k), B, m, kk)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def run_attn(hsa, Q, K, V, idx_np, scale=0.0):
    import torch
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    O = hsa.sparse_attn(dev(Q), dev(K), dev(V), idx, scale=scale)
    torch.cuda.synchronize()
    return host_bits(O)


# ------------------------------------------------------------------ stages

@pytest.mark.parametrize("Lk,B,d", [(2048, 64, 64), (5037, 128, 128), (999, 7, 64), (64, 64, 128)])
def test_block_sums_bit_exact(hsa, Lk, B, d):
    import torch
    k = synth.int_bf16((Lk, d), 11, 2)
    ks = torch.empty((Lk // B, d), dtype=torch.float32, device="cuda")
    p = hsa.params(B=B, m=8, k=16, d_idx=d)
    hsa.hsa_block_sums(p, Lk, dev(k), ks)
    torch.cuda.synchronize()
    assert np.array_equal(ks.cpu().numpy(), oracle.block_sums(k, B))


@pytest.mark.parametrize("Lq,Lk,B,m,d", [(2048, 2048, 64, 8, 64), (700, 5037, 128, 6, 128),
                                         (300, 300, 4, 2, 64), (4096, 4096, 16, 40, 128)])
def test_select_blocks_bit_exact(hsa, Lq, Lk, B, m, d):
    import torch
    q, k = synth.int_bf16((Lq, d), 12, 1), synth.int_bf16((Lk, d), 12, 2)
    p = hsa.params(B=B, m=m, k=16, d_idx=d)
    ks = torch.empty((max(Lk // B, 1), d), dtype=torch.float32, device="cuda")
    hsa.hsa_block_sums(p, Lk, dev(k), ks)
    blocks = torch.empty((Lq, m), dtype=torch.int32, device="cuda")
    ws = torch.empty(hsa.hsa_index_workspace_size(p, Lq, Lk), dtype=torch.uint8, device="cuda")
    hsa.hsa_select_blocks(p, Lq, Lk, dev(q), ks, blocks, ws)
    torch.cuda.synchronize()
    want = oracle.select_blocks(q, oracle.block_sums(k, B), Lk, B, m)
    assert np.array_equal(blocks.cpu().numpy(), want)
    # token stage on the same blocks, through its own entry point
    kk = 3 * B
    p.k = kk
    ws = torch.empty(hsa.hsa_index_workspace_size(p, Lq, Lk), dtype=torch.uint8, device="cuda")
    idx = torch.empty((Lq, kk), dtype=torch.int32, device="cuda")
    hsa.hsa_select_tokens(p, Lq, Lk, dev(q), dev(k), blocks, idx, ws)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), oracle.select_tokens(q, k, want, B, kk))


# ------------------------------------------------------------------ indexer

def test_index_tiny_prefill_all_rows(hsa):
    w = synth.WORKLOADS["tiny_prefill_2k"]
    x = synth.prefill_inputs(w, with_attn=False)
    got = run_index(hsa, x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    assert np.array_equal(got, oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, w.k))


def test_index_prefill_16k_all_rows(hsa):
    w = synth.WORKLOADS["prefill_16k"]
    x = synth.prefill_inputs(w, with_attn=False)
    got = run_index(hsa, x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    want = oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    bad = np.nonzero((got != want).any(axis=1))[0]
    assert len(bad) == 0, f"{len(bad)} rows differ, first {bad[:5]}"


@pytest.mark.parametrize("Lq,Lk,B,m,k,d", [
    (777, 5037, 64, 8, 256, 128),     # chunk of queries, ragged last block
    (1, 1, 64, 8, 256, 64),           # a single token
    (1, 9000, 128, 16, 2048, 128),    # one query at the end of a long prefix
    (512, 512, 16, 2, 7, 64),         # m = 2: forced blocks only
    (600, 600, 32, 4, 1, 64),         # k = 1
    (400, 400, 8, 5, 40, 128),        # k = m*B: every candidate of a full row kept
    (333, 1000, 10, 12, 100, 64),     # B not a power of two
    (3000, 9000, 64, 16, 300, 128),   # tensor-core path, B = 64, chunk of queries
    (2500, 2500, 64, 10, 200, 64),    # tensor-core path, d_idx = 64
    (129, 20000, 128, 24, 1000, 128), # one M tile plus one row
])
def test_index_shapes_bit_exact(hsa, Lq, Lk, B, m, k, d):
    q, kk = synth.int_bf16((Lq, d), 13, 1), synth.int_bf16((Lk, d), 13, 2)
    got = run_index(hsa, q, kk, B, m, k)
    assert np.array_equal(got, oracle.index(q, kk, B, m, k))


def test_index_all_ties_goes_to_lowest_indices(hsa):
    Lq = Lk = 1500
    q = np.zeros((Lq, 64), dtype=np.uint16)     # every score is 0
    kk = synth.int_bf16((Lk, 64), 14, 2)
    got = run_index(hsa, q, kk, 32, 6, 50)
    assert np.array_equal(got, oracle.index(q, kk, 32, 6, 50))


@pytest.mark.parametrize("probs,k", [
    ({1.0: 0.5}, 512),            # two score values: the threshold bin holds ~1000 tied keys
    ({3.0: 0.2, 2.0: 0.02}, 430),  # the threshold usually falls among ~40 tied keys of value 2
])
def test_index_few_score_values_ties_exact(hsa, probs, k):
    # every score is k[:, 0] (q is all ones, the other key dims are 0), so most
    # candidates tie and selection inside the tied group goes by lowest index
    rng = np.random.default_rng(16)
    Lq = Lk = 4096
    q = synth.f32_to_bf16_bits(np.ones((Lq, 64), np.float32))
    vals = np.zeros((Lk, 64), np.float32)
    u = rng.random(Lk)
    lo = 0.0
    for v, pr in probs.items():
        vals[(u >= lo) & (u < lo + pr), 0] = v
        lo += pr
    kk = synth.f32_to_bf16_bits(vals)
    got = run_index(hsa, q, kk, 128, 16, k)
    assert np.array_equal(got, oracle.index(q, kk, 128, 16, k))


def test_index_infinite_scores_exact(hsa):
    # one key row whose products with every query overflow fp32 to +inf: its
    # token score and its block's score are +inf in every row that sees it, so
    # the top-k cannot use value-linear bins and runs on the key bits alone
    rng = np.random.default_rng(17)
    Lq = Lk = 3072
    q = synth.int_bf16((Lq, 64), 17, 1)
    q[:, 0] = synth.f32_to_bf16_bits(np.full(Lq, 2.0 ** 64, np.float32))
    kk = synth.int_bf16((Lk, 64), 17, 2)
    kk[:, 0] = synth.f32_to_bf16_bits(rng.integers(0, 9, Lk).astype(np.float32))
    kk[700, 0] = synth.f32_to_bf16_bits(np.array([2.0 ** 65], np.float32))[0]
    got = run_index(hsa, q, kk, 128, 8, 512)
    want = oracle.index(q, kk, 128, 8, 512)
    assert np.array_equal(got, want)
    assert (got[1000:] == 700).any(axis=1).all()  # the +inf key is always kept once visible


def test_index_extreme_magnitudes_exact(hsa):
    # all entries +-8: token scores reach +-8192 and block scores +-2^20
    rng = np.random.default_rng(15)
    Lq = Lk = 4096
    q = synth.f32_to_bf16_bits(rng.choice([-8.0, 8.0], size=(Lq, 128)).astype(np.float32))
    kk = synth.f32_to_bf16_bits(rng.choice([-8.0, 8.0], size=(Lk, 128)).astype(np.float32))
    kk[:128] = synth.f32_to_bf16_bits(np.full((128, 128), 8.0, np.float32))
    q[-1] = synth.f32_to_bf16_bits(np.full(128, 8.0, np.float32))
    got = run_index(hsa, q, kk, 128, 8, 512)
    assert np.array_equal(got, oracle.index(q, kk, 128, 8, 512))


def test_index_prefill_64k_all_rows_and_needles(hsa):
    w = synth.WORKLOADS["prefill_64k"]
    x = synth.prefill_inputs(w, with_attn=False)
    got = run_index(hsa, x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    want = oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, w.k)  # every one of the 65,536 rows
    bad = np.flatnonzero(np.any(got != want, axis=1))
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:8].tolist()}"
    # structural checks on every row: ascending, causal, -1 only as tail padding
    t = np.arange(w.Lq)[:, None]
    valid = got >= 0
    assert (got <= t).all()
    nvalid = valid.sum(axis=1)
    assert (valid == (np.arange(w.k)[None, :] < nvalid[:, None])).all()  # -1 only as a tail
    assert (nvalid == np.minimum(np.arange(w.Lq) + 1, w.k)).all()
    inc = np.diff(got, axis=1) > 0
    assert (inc | ~valid[:, 1:]).all()  # strictly ascending over the valid prefix
    recall = np.mean([j in set(got[i].tolist()) for i, j in x["needles"]])
    print(f"needle recall {recall:.3f}")


def test_index_long_context_chunk_all_rows(hsa):
    w = synth.WORKLOADS["prefill_1m_last8k"]
    x = synth.prefill_inputs(w, with_attn=False)
    got = run_index(hsa, x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    want = oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, w.k)  # all 8192 rows
    bad = np.flatnonzero(np.any(got != want, axis=1))
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:8].tolist()}"


@pytest.mark.parametrize("Lq,Lk,B,m,k,seed", [
    (16384, 16384, 128, 128, 2048, 50),  # the flat token-level indexer at 16K: every causal block kept
    (1000, 12000, 128, 80, 1000, 52),    # 10,240 candidates, many rows: one warp per row
    (400, 20000, 64, 200, 3000, 53),     # 12,800 candidates at B = 64
    (200, 40000, 64, 256, 2048, 51),     # 16,384 candidates, few rows: a 1024-thread CTA per row
    (100, 30000, 128, 100, 4096, 54),    # 12,800 candidates, few rows, k above the block count * 32
])
def test_index_long_candidate_rows_bit_exact(hsa, Lq, Lk, B, m, k, seed):
    # rows of more than 8192 candidates (m*B > 8192) leave the shared-memory
    # row kernel of the top-k for the longer-row kernels
    q, kk = synth.int_bf16((Lq, 128), seed, 1), synth.int_bf16((Lk, 128), seed, 2)
    got = run_index(hsa, q, kk, B, m, k)
    want = oracle.index(q, kk, B, m, k)
    bad = np.flatnonzero(np.any(got != want, axis=1))
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:8].tolist()}"


@pytest.mark.parametrize("Lq,Lk,B,m,k,seed", [
    (2000, 20000, 256, 16, 1000, 55),    # B = 256 on tensor cores
    (500, 30000, 256, 64, 2048, 56),     # B = 256, 16,384 candidates, one warp per row
    (100, 30000, 256, 40, 3000, 57),     # B = 256, few rows: a 1024-thread CTA per row
    (300, 40000, 64, 512, 4096, 58),     # m = 512 (32,768 candidates), blocks pruned
    (120, 70000, 128, 512, 2048, 59),    # m = 512 at B = 128: 65,536 candidates, few rows
])
def test_index_wide_rows_bit_exact(hsa, Lq, Lk, B, m, k, seed):
    q, kk = synth.int_bf16((Lq, 128), seed, 1), synth.int_bf16((Lk, 128), seed, 2)
    got = run_index(hsa, q, kk, B, m, k)
    want = oracle.index(q, kk, B, m, k)
    bad = np.flatnonzero(np.any(got != want, axis=1))
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:8].tolist()}"


def test_index_flat_64k_sampled(hsa):
    # the flat token-level indexer at 64K: m = 512 keeps every causal block, so
    # every causal token of a query is a candidate (up to 65,536 per row)
    w = synth.WORKLOADS["prefill_64k"]
    x = synth.prefill_inputs(w, with_attn=False)
    m = w.L // w.B
    got = run_index(hsa, x["q_idx"], x["k_idx"], w.B, m, w.k)
    rows = sample_rows(w.Lq, 1024, 60, always=[0, w.k - 1, w.k, w.Lq // 2, w.Lq - 1])
    want = oracle.index(x["q_idx"], x["k_idx"], w.B, m, w.k, rows=rows)
    bad = np.flatnonzero(np.any(got[rows] != want, axis=1))
    assert bad.size == 0, f"{bad.size} rows differ, first {rows[bad[:8]].tolist()}"
    # structure of every row: ascending, causal, min(t + 1, k) valid entries
    valid = got >= 0
    assert (valid.sum(axis=1) == np.minimum(np.arange(w.Lq) + 1, w.k)).all()


# ------------------------------------------------------------------ attention

def test_attention_tiny_prefill_all_rows(hsa):
    w = synth.WORKLOADS["tiny_prefill_2k"]
    x = synth.prefill_inputs(w)
    idx = oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    got = run_attn(hsa, x["Q"], x["K"], x["V"], idx)
    ref = oracle.sparse_attn(x["Q"], x["K"], x["V"], idx)
    print("tiny max/mean abs err", assert_attn_close(got, ref, "tiny"))


def test_attention_prefill_16k_sampled(hsa):
    w = synth.WORKLOADS["prefill_16k"]
    x = synth.prefill_inputs(w)
    idx = run_index(hsa, x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    got = run_attn(hsa, x["Q"], x["K"], x["V"], idx)
    rows = sample_rows(w.Lq, 512, 18, always=[0, 1, 100, 2047, 2048, w.Lq - 1])
    ref = oracle.sparse_attn(x["Q"], x["K"], x["V"], idx[rows], rows=rows)
    print("16k max/mean abs err", assert_attn_close(got[rows], ref, "16k"))


@pytest.mark.parametrize("H,d,k", [(1, 64, 5), (16, 128, 1), (64, 128, 300), (128, 64, 130),
                                   (8, 128, 2048)])
def test_attention_shapes(hsa, H, d, k):
    Lq, Lk = 70, 3000
    rng = np.random.default_rng(H * 1000 + k)
    Q, K, V = (synth.normal_bf16(s, 19, i) for i, s in enumerate([(Lq, H, d), (Lk, d), (Lk, d)]))
    idx = np.full((Lq, k), -1, dtype=np.int32)
    for i in range(Lq):
        n = int(rng.integers(0, k + 1)) if i % 7 else k   # ragged rows, some empty
        idx[i, :n] = np.sort(rng.choice(Lk, size=n, replace=False))
    got = run_attn(hsa, Q, K, V, idx)
    ref = oracle.sparse_attn(Q, K, V, idx)
    assert_attn_close(got, ref, f"H={H} d={d} k={k}")


@pytest.mark.parametrize("k", [4096, 8192])
def test_attention_long_index_rows(hsa, k):
    # k above 2048 (up to the 8192 the API accepts): 32 or 64 tiles per query,
    # ragged and empty rows among them
    Lq, Lk, H, d = 40, 12000, 64, 128
    rng = np.random.default_rng(k)
    Q, K, V = (synth.normal_bf16(s, 26, i) for i, s in enumerate([(Lq, H, d), (Lk, d), (Lk, d)]))
    idx = np.full((Lq, k), -1, dtype=np.int32)
    for i in range(Lq):
        n = k if i % 3 == 0 else int(rng.integers(0, k + 1))
        idx[i, :n] = np.sort(rng.choice(Lk, size=n, replace=False))
    got = run_attn(hsa, Q, K, V, idx)
    assert_attn_close(got, oracle.sparse_attn(Q, K, V, idx), f"k={k}")


def test_attention_pure_block_sparse_64k_sampled(hsa):
    # the pure block-sparse setting of the 64K workload: k = m*B keeps every
    # candidate of the top-m blocks (8192 keys per query)
    w = synth.WORKLOADS["prefill_64k"]
    x = synth.prefill_inputs(w)
    k = w.m * w.B
    idx = run_index(hsa, x["q_idx"], x["k_idx"], w.B, w.m, k)
    rows = sample_rows(w.Lq, 256, 27, always=[0, w.B * w.m, w.Lq - 1])
    assert np.array_equal(idx[rows], oracle.index(x["q_idx"], x["k_idx"], w.B, w.m, k, rows=rows))
    got = run_attn(hsa, x["Q"], x["K"], x["V"], idx)
    ref = oracle.sparse_attn(x["Q"], x["K"], x["V"], idx[rows], rows=rows)
    print("64k block-sparse max/mean abs err", assert_attn_close(got[rows], ref, "64k k=8192"))


def test_attention_large_logits_stable(hsa):
    # Q, K of magnitude 4..8: scaled logits in the hundreds; exact softmax must hold.
    Lq, Lk, H, d, k = 16, 512, 4, 128, 256
    rng = np.random.default_rng(20)
    Q = synth.f32_to_bf16_bits((rng.choice([-1, 1], size=(Lq, H, d)) * 6.0).astype(np.float32))
    K = synth.f32_to_bf16_bits((rng.choice([-1, 1], size=(Lk, d)) * 4.0).astype(np.float32))
    V = synth.normal_bf16((Lk, d), 20, 5)
    idx = np.stack([np.sort(rng.choice(Lk, size=k, replace=False)) for _ in range(Lq)]).astype(np.int32)
    got = run_attn(hsa, Q, K, V, idx)
    assert_attn_close(got, oracle.sparse_attn(Q, K, V, idx), "large logits")


def test_attention_explicit_scale(hsa):
    Lq, Lk, H, d, k = 20, 400, 4, 64, 64
    Q, K, V = (synth.normal_bf16(s, 21, i) for i, s in enumerate([(Lq, H, d), (Lk, d), (Lk, d)]))
    rng = np.random.default_rng(21)
    idx = np.stack([np.sort(rng.choice(Lk, size=k, replace=False)) for _ in range(Lq)]).astype(np.int32)
    got = run_attn(hsa, Q, K, V, idx, scale=0.3)
    assert_attn_close(got, oracle.sparse_attn(Q, K, V, idx, scale=0.3), "scale")


def test_attention_explicit_scale_d128(hsa):
    Lq, Lk, H, d, k = 33, 900, 64, 128, 257
    Q, K, V = (synth.normal_bf16(s, 23, i) for i, s in enumerate([(Lq, H, d), (Lk, d), (Lk, d)]))
    rng = np.random.default_rng(23)
    idx = np.stack([np.sort(rng.choice(Lk, size=k, replace=False)) for _ in range(Lq)]).astype(np.int32)
    got = run_attn(hsa, Q, K, V, idx, scale=0.05)
    assert_attn_close(got, oracle.sparse_attn(Q, K, V, idx, scale=0.05), "scale d128")


def test_attention_holes_and_out_of_range_entries(hsa):
    # -1 entries anywhere in a row (not only as a tail) are skipped
    Lq, Lk, H, d, k = 40, 2000, 16, 128, 700
    Q, K, V = (synth.normal_bf16(s, 24, i) for i, s in enumerate([(Lq, H, d), (Lk, d), (Lk, d)]))
    rng = np.random.default_rng(24)
    idx = np.stack([np.sort(rng.choice(Lk, size=k, replace=False)) for _ in range(Lq)]).astype(np.int32)
    idx[rng.random(idx.shape) < 0.3] = -1
    idx[5, :] = -1            # an empty row
    idx[6, 130:] = -1         # only the first tile valid
    idx[7, :600] = -1         # only the last tiles valid
    got = run_attn(hsa, Q, K, V, idx)
    ref = oracle.sparse_attn(Q, K, V, idx)
    assert (got[5] == 0).all()
    assert_attn_close(got, ref, "holes")


@pytest.mark.parametrize("H", [64, 16, 5])
def test_attention_running_max_rescales(hsa, H):
    # scores grow by ~8 (log2 units) from one 128-key tile to the next, so the
    # running maximum is raised and the accumulator rescaled on every tile
    Lq, Lk, d, k = 12, 2048, 128, 2048
    Q = synth.f32_to_bf16_bits(np.ones((Lq, H, d), np.float32)
                               * (1.0 + np.arange(H, dtype=np.float32) / 64)[None, :, None])
    K = synth.f32_to_bf16_bits(np.repeat(0.5 * (np.arange(Lk) // 128), d).reshape(Lk, d).astype(np.float32))
    V = synth.normal_bf16((Lk, d), 25, 5)
    idx = np.tile(np.arange(k, dtype=np.int32), (Lq, 1))
    idx[1, 1000:] = -1
    idx[2] = idx[2][::-1].copy()  # descending order: the first tile holds the maximum
    got = run_attn(hsa, Q, K, V, idx)
    assert_attn_close(got, oracle.sparse_attn(Q, K, V, idx), "rescale")


def test_attention_prefill_64k_sampled(hsa):
    w = synth.WORKLOADS["prefill_64k"]
    x = synth.prefill_inputs(w)
    idx = run_index(hsa, x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    got = run_attn(hsa, x["Q"], x["K"], x["V"], idx)
    rows = sample_rows(w.Lq, 4096, 22, always=[0, 1, 2047, w.Lq - 1])
    ref = oracle.sparse_attn(x["Q"], x["K"], x["V"], idx[rows], rows=rows)
    print("64k max/mean abs err", assert_attn_close(got[rows], ref, "64k"))


def test_attention_long_context_chunk_sampled(hsa):
    w = synth.WORKLOADS["prefill_1m_last8k"]
    x = synth.prefill_inputs(w)
    idx = run_index(hsa, x["q_idx"], x["k_idx"], w.B, w.m, w.k)
    got = run_attn(hsa, x["Q"], x["K"], x["V"], idx)
    rows = sample_rows(w.Lq, 4096, 23, always=[0, w.Lq - 1])
    ref = oracle.sparse_attn(x["Q"], x["K"], x["V"], idx[rows], rows=rows)
    print("1m chunk max/mean abs err", assert_attn_close(got[rows], ref, "1m chunk"))


def test_attention_second_pass_many_rows(hsa):
    # Rows whose later tiles outgrow the first tile's maximum (by ~8 log2
    # units a tile) are flagged by the first pass and taken again with the
    # per-tile rescale; more rows than SMs, every head group's warpgroups
    # flagging the same rows, flat rows (descending order) and short rows
    # among them.
    Lq, Lk, H, d, k = 400, 2048, 64, 128, 1024
    Q = synth.f32_to_bf16_bits(np.ones((Lq, H, d), np.float32)
                               * (1.0 + np.arange(H, dtype=np.float32) / 64)[None, :, None])
    K = synth.f32_to_bf16_bits(np.repeat(0.5 * (np.arange(Lk) // 128), d).reshape(Lk, d).astype(np.float32))
    V = synth.normal_bf16((Lk, d), 28, 5)
    rng = np.random.default_rng(28)
    idx = np.full((Lq, k), -1, dtype=np.int32)
    for i in range(Lq):
        n = k if i % 5 else int(rng.integers(1, k + 1))
        row = np.sort(rng.choice(Lk, size=n, replace=False)).astype(np.int32)
        idx[i, :n] = row[::-1] if i % 2 else row
    got = run_attn(hsa, Q, K, V, idx)
    assert_attn_close(got, oracle.sparse_attn(Q, K, V, idx), "second pass")


# ------------------------------------------------------------------ decode

def decode_case(hsa, B, m, k, d_idx, H, d, ctx0, capacity, steps, seed, check_seqs=None):
    """Run `steps` decode steps on the GPU and compare every step with the
    oracle evaluated on the host copy of each sequence's cache."""
    import torch
    batch = len(ctx0)
    rng = np.random.default_rng(seed)
    kc = synth.int_bf16((batch, capacity, d_idx), seed, 2)
    Kc = synth.normal_bf16((batch, capacity, d), seed, 4)
    Vc = synth.normal_bf16((batch, capacity, d), seed, 5)
    new = {n: synth.int_bf16((steps, batch, d_idx), seed, 30 + i) for i, n in enumerate(["q", "k"])}
    newQ = synth.normal_bf16((steps, batch, H, d), seed, 33)
    newK = synth.normal_bf16((steps, batch, d), seed, 34)
    newV = synth.normal_bf16((steps, batch, d), seed, 35)
    p = hsa.params(B=B, m=m, k=k, d_idx=d_idx, H=H, d=d)
    g_kc, g_Kc, g_Vc = dev(kc), dev(Kc), dev(Vc)
    ksum = torch.zeros((batch, capacity // B, d_idx), dtype=torch.float32, device="cuda")
    for b in range(batch):
        hsa.hsa_block_sums(p, int(ctx0[b]), g_kc[b], ksum[b])
    ctx = torch.tensor(ctx0, dtype=torch.int32, device="cuda")
    ws = torch.empty(hsa.hsa_decode_workspace_size(p, batch, capacity), dtype=torch.uint8, device="cuda")
    O = torch.empty((batch, H, d), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((batch, k), dtype=torch.int32, device="cuda")
    lens = np.array(ctx0, dtype=np.int64)
    check = range(batch) if check_seqs is None else check_seqs
    for s in range(steps):
        hsa.hsa_decode_step(p, batch, capacity, ctx, g_kc, g_Kc, g_Vc, ksum, dev(new["q"][s]),
                            dev(new["k"][s]), dev(newQ[s]), dev(newK[s]), dev(newV[s]), O, idx, ws)
        torch.cuda.synchronize()
        got_idx, got_O = idx.cpu().numpy(), host_bits(O)
        for b in check:
            t = int(lens[b])
            if t >= capacity:
                assert (got_idx[b] == -1).all() and (got_O[b] == 0).all()
                continue
            kc[b, t], Kc[b, t], Vc[b, t] = new["k"][s, b], newK[s, b], newV[s, b]
            want = oracle.index(new["q"][s, b][None], kc[b, : t + 1], B, m, k)
            assert np.array_equal(got_idx[b], want[0]), (s, b)
            ref = oracle.sparse_attn(newQ[s, b][None], Kc[b, : t + 1], Vc[b, : t + 1], want)
            assert_attn_close(got_O[b][None], ref, f"decode step {s} seq {b}")
        lens = np.minimum(lens + 1, capacity)
        assert np.array_equal(ctx.cpu().numpy(), np.minimum(np.array(ctx0) + s + 1, capacity))
    # block sums written by the steps match the oracle's for every complete block
    for b in check:
        n = int(lens[b]) // B
        assert np.array_equal(ksum[b, :n].cpu().numpy(), oracle.block_sums(kc[b, : n * B], B))


def test_decode_small_all_sequences(hsa):
    # ragged lengths, block completions during the run, one sequence hitting capacity
    decode_case(hsa, B=64, m=8, k=256, d_idx=64, H=4, d=64, ctx0=[1, 63, 500, 1000, 1020],
                capacity=1024, steps=70, seed=40)


def test_decode_wide_rows(hsa):
    # 19,200 candidates per query: the long-row top-k kernels on decode rows
    decode_case(hsa, B=64, m=300, k=1000, d_idx=64, H=4, d=64, ctx0=[30000, 20000, 20095],
                capacity=32768, steps=3, seed=43)


def test_decode_128k_all_sequences(hsa):
    # the 128K decode workload's shape, every sequence checked: the contexts
    # start one token short of 1024 full blocks, so step 0 completes block
    # 1023 of every sequence (its block sum is written and then compared) and
    # step 1 scores it as a candidate block
    decode_case(hsa, B=128, m=64, k=2048, d_idx=128, H=64, d=128, ctx0=[131071] * 32,
                capacity=131072 + 256, steps=2, seed=41)


def test_decode_after_1m_context(hsa):
    # the decode steps of the 1M-context workload: one sequence at 1,048,576 cached tokens
    decode_case(hsa, B=128, m=64, k=2048, d_idx=128, H=64, d=128, ctx0=[1 << 20],
                capacity=(1 << 20) + 256, steps=2, seed=42)
