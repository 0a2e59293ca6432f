"""Pins for the CPU oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: hand-worked
examples (tests/golden), brute-force subset enumeration in exact integer
arithmetic, the flat top-k invariant (m >= number of blocks), closed forms of
the softmax, and torch's textbook scaled-dot-product attention.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from synth import bf16_bits_to_f32, f32_to_bf16_bits, int_bf16, normal_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- hand examples

@pytest.mark.parametrize("name", ["hand_example_a.json", "hand_example_b.json"])
def test_hand_examples_indices(name):
    g = load(name)
    p = g["params"]
    q, k = bf(g["q_idx"]), bf(g["k_idx"])
    out, blocks = oracle.index(q, k, p["B"], p["m"], p["k"], with_blocks=True)
    for t, exp in g["expected_indices"].items():
        assert out[int(t)].tolist() == exp, (name, t)
    for t, exp in g.get("expected_blocks", {}).items():
        assert blocks[int(t)].tolist() == exp, (name, t)


def test_hand_example_b_differs_from_flat():
    g = load("hand_example_b.json")
    p = g["params"]
    q, k = bf(g["q_idx"]), bf(g["k_idx"])
    flat = oracle.index(q, k, p["B"], 100, p["k"])  # m above every block count
    assert flat[7].tolist() == g["flat_top2_t7"]
    hier = oracle.index(q, k, p["B"], p["m"], p["k"])
    assert hier[7].tolist() != flat[7].tolist()


def test_hand_example_a_uniform_attention():
    g = load("hand_example_a.json")
    p = g["params"]
    q, k = bf(g["q_idx"]), bf(g["k_idx"])
    idx = oracle.index(q, k, p["B"], p["m"], p["k"])
    rng = np.random.default_rng(1)
    V = bf(rng.standard_normal((8, 8)))
    K = bf(rng.standard_normal((8, 8)))
    Q = np.zeros((8, 2, 8), dtype=np.uint16)  # Q = 0: every kept key weighs the same
    O = oracle.sparse_attn(Q, K, V, idx)
    Vf = bf16_bits_to_f32(V).astype(np.float64)
    want = (Vf[2] + Vf[5] + Vf[6]) / 3.0
    for h in range(2):
        np.testing.assert_allclose(O[7, h], want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O[0, 0], Vf[0], rtol=0, atol=1e-12)  # single key


# ---------------------------------------------------------------- block sums

def test_block_sums_closed_form():
    # k_idx[j][c] = (j mod 7) - 3 + c; the sum over a block of B rows has a closed form.
    Lk, B, d = 45, 5, 3
    vals = np.array([[(j % 7) - 3 + c for c in range(d)] for j in range(Lk)], dtype=np.float32)
    ks = oracle.block_sums(bf(vals), B)
    assert ks.shape == (Lk // B, d)  # partial tail block is not produced
    for b in range(Lk // B):
        for c in range(d):
            want = sum((j % 7) - 3 + c for j in range(b * B, b * B + B))
            assert ks[b, c] == want


# ---------------------------------------------------------------- brute force

def brute_blocks(q, kv, t, B, m):
    """Kept blocks by exhaustive search: the forced pair plus the (m-2)-subset
    of blocks 1..nb-2 with the largest total score, the lexicographically
    smallest such subset on ties (== 'ties go to the lowest index')."""
    nb = t // B + 1
    if nb <= m:
        return list(range(nb))
    def score(b):
        return sum(int(q[c]) * sum(int(kv[j][c]) for j in range(b * B, b * B + B))
                   for c in range(len(q)))
    best, best_s = None, None
    for comb in itertools.combinations(range(1, nb - 1), m - 2):
        s = sum(score(b) for b in comb)
        if best_s is None or s > best_s:
            best, best_s = comb, s
    return sorted([0, nb - 1, *best])


def brute_tokens(q, kv, t, B, blocks, k):
    cand = [j for b in blocks for j in range(b * B, b * B + B) if j <= t]
    if len(cand) <= k:
        keep = cand
    else:
        def score(j):
            return sum(int(q[c]) * int(kv[j][c]) for c in range(len(q)))
        best, best_s = None, None
        for comb in itertools.combinations(sorted(cand), k):
            s = sum(score(j) for j in comb)
            if best_s is None or s > best_s:
                best, best_s = comb, s
        keep = list(best)
    keep = sorted(keep)
    return keep + [-1] * (k - len(keep))


@pytest.mark.parametrize("seed", range(40))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(2, 4))
    m = int(rng.integers(2, 5))
    k = int(rng.integers(1, 4))
    d = int(rng.integers(1, 4))
    Lk = int(rng.integers(1, 7 * B + 1))
    Lq = int(rng.integers(1, Lk + 1))
    kv = rng.integers(-2, 3, size=(Lk, d))
    qv = rng.integers(-2, 3, size=(Lq, d))
    out, blocks = oracle.index(bf(qv), bf(kv), B, m, k, with_blocks=True)
    for i in range(Lq):
        t = Lk - Lq + i
        bb = brute_blocks(qv[i], kv, t, B, m)
        assert blocks[i].tolist() == bb + [-1] * (m - len(bb)), (seed, i)
        assert out[i].tolist() == brute_tokens(qv[i], kv, t, B, bb, k), (seed, i)


# ---------------------------------------------------------------- invariants

def flat_topk(qf, kf, t, k):
    s = kf[: t + 1] @ qf
    order = np.lexsort((np.arange(t + 1), -s))[:k]
    keep = np.sort(order)
    return np.concatenate([keep, -np.ones(k - len(keep), dtype=np.int64)])


@pytest.mark.parametrize("Lq,Lk,B,k", [(200, 200, 8, 16), (64, 300, 16, 40), (97, 97, 4, 5)])
def test_all_blocks_equals_flat_topk(Lq, Lk, B, k):
    q = int_bf16((Lq, 16), 3, 1)
    kk = int_bf16((Lk, 16), 3, 2)
    m = Lk // B + 2  # m >= number of causal blocks for every query
    out = oracle.index(q, kk, B, m, k)
    qf, kf = bf16_bits_to_f32(q).astype(np.float64), bf16_bits_to_f32(kk).astype(np.float64)
    for i in range(Lq):
        t = Lk - Lq + i
        assert out[i].tolist() == flat_topk(qf[i], kf, t, k).tolist(), i


def test_forced_blocks_and_count():
    Lq = Lk = 2048
    B, m, k = 32, 6, 64
    q, kk = int_bf16((Lq, 32), 5, 1), int_bf16((Lk, 32), 5, 2)
    out, blocks = oracle.index(q, kk, B, m, k, with_blocks=True)
    for t in range(Lk):
        nb = t // B + 1
        row = blocks[t]
        valid = row[row >= 0]
        assert len(valid) == min(nb, m)
        assert valid[0] == 0 and valid[-1] == nb - 1
        assert np.all(np.diff(valid) > 0)
        sel = out[t][out[t] >= 0]
        assert np.all(np.diff(sel) > 0) and sel.max() <= t
        assert np.all(np.isin(sel // B, valid))
        ncand = sum(min(B, t + 1 - b * B) for b in valid)
        assert len(sel) == min(ncand, k)


def test_rows_subset_matches_full():
    Lq, Lk = 300, 700
    q, kk = int_bf16((Lq, 16), 9, 1), int_bf16((Lk, 16), 9, 2)
    full = oracle.index(q, kk, 16, 5, 30)
    rows = np.array([0, 7, 150, 299])
    assert np.array_equal(oracle.index(q, kk, 16, 5, 30, rows=rows), full[rows])


# ---------------------------------------------------------------- attention

def sdpa_reference(Q, K, V, idx, Lk):
    """torch's scaled_dot_product_attention in fp64 with a boolean mask built
    from the kept indices (MQA: the single K/V head is shared by all heads)."""
    Lq, H, d = Q.shape
    q = torch.from_numpy(bf16_bits_to_f32(Q).astype(np.float64)).permute(1, 0, 2)  # H, Lq, d
    kf = torch.from_numpy(bf16_bits_to_f32(K).astype(np.float64))
    vf = torch.from_numpy(bf16_bits_to_f32(V).astype(np.float64))
    mask = torch.zeros(Lq, Lk, dtype=torch.bool)
    for i in range(Lq):
        sel = idx[i][idx[i] >= 0]
        mask[i, torch.from_numpy(sel.astype(np.int64))] = True
    o = torch.nn.functional.scaled_dot_product_attention(
        q, kf.expand(H, Lk, d), vf.expand(H, Lk, d), attn_mask=mask)
    return o.permute(1, 0, 2).numpy()


def test_attention_equals_dense_causal_when_k_covers_all():
    L, H, d = 96, 3, 16
    Q, K, V = normal_bf16((L, H, d), 4, 3), normal_bf16((L, d), 4, 4), normal_bf16((L, d), 4, 5)
    q, kk = int_bf16((L, 8), 4, 1), int_bf16((L, 8), 4, 2)
    # m covers every block and k >= L: every causal key is a kept candidate
    idx = oracle.index(q, kk, 8, L // 8 + 1, L)
    for t in range(L):
        assert idx[t].tolist() == list(range(t + 1)) + [-1] * (L - t - 1)
    O = oracle.sparse_attn(Q, K, V, idx)
    qt = torch.from_numpy(bf16_bits_to_f32(Q).astype(np.float64)).permute(1, 0, 2)
    kt = torch.from_numpy(bf16_bits_to_f32(K).astype(np.float64)).expand(H, L, d)
    vt = torch.from_numpy(bf16_bits_to_f32(V).astype(np.float64)).expand(H, L, d)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    np.testing.assert_allclose(O, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_attention_matches_masked_sdpa_on_sparse_sets():
    Lq, Lk, H, d = 40, 120, 4, 32
    Q, K, V = normal_bf16((Lq, H, d), 6, 3), normal_bf16((Lk, d), 6, 4), normal_bf16((Lk, d), 6, 5)
    q, kk = int_bf16((Lq, 16), 6, 1), int_bf16((Lk, 16), 6, 2)
    idx = oracle.index(q, kk, 8, 4, 20)
    O = oracle.sparse_attn(Q, K, V, idx)
    np.testing.assert_allclose(O, sdpa_reference(Q, K, V, idx, Lk), rtol=0, atol=1e-12)


def test_attention_two_key_closed_form():
    # Two kept keys: weights are a logistic function of scale * q.(K0 - K1).
    d = 64
    rng = np.random.default_rng(2)
    Q = bf(rng.standard_normal((1, 1, d)))
    K = bf(rng.standard_normal((2, d)))
    V = bf(rng.standard_normal((2, d)))
    idx = np.array([[0, 1, -1]], dtype=np.int32)
    O = oracle.sparse_attn(Q, K, V, idx)
    qf, kf, vf = (bf16_bits_to_f32(a).astype(np.float64) for a in (Q, K, V))
    delta = (qf[0, 0] @ (kf[0] - kf[1])) / math.sqrt(d)
    w0 = 1.0 / (1.0 + math.exp(-delta))
    np.testing.assert_allclose(O[0, 0], w0 * vf[0] + (1 - w0) * vf[1], rtol=0, atol=1e-12)
    # An explicit scale replaces 1/sqrt(d).
    O2 = oracle.sparse_attn(Q, K, V, idx, scale=0.5)
    w0 = 1.0 / (1.0 + math.exp(-0.5 * (qf[0, 0] @ (kf[0] - kf[1]))))
    np.testing.assert_allclose(O2[0, 0], w0 * vf[0] + (1 - w0) * vf[1], rtol=0, atol=1e-12)


def test_attention_single_index_returns_value_row():
    Q, K, V = normal_bf16((3, 2, 16), 8, 3), normal_bf16((10, 16), 8, 4), normal_bf16((10, 16), 8, 5)
    idx = np.array([[4, -1], [9, -1], [0, -1]], dtype=np.int32)
    O = oracle.sparse_attn(Q, K, V, idx)
    Vf = bf16_bits_to_f32(V).astype(np.float64)
    for r, j in enumerate([4, 9, 0]):
        for h in range(2):
            np.testing.assert_array_equal(O[r, h], Vf[j])


def test_attention_large_scores_are_stable():
    # Scores of a few hundred must not overflow: the max is subtracted first.
    d = 16
    Q = bf(np.full((1, 1, d), 8.0))
    K = bf(np.stack([np.full(d, 4.0), np.full(d, 3.0)]))
    V = bf(np.stack([np.arange(d), -np.arange(d)]).astype(np.float32))
    O = oracle.sparse_attn(Q, K, V, np.array([[0, 1]], dtype=np.int32), scale=1.0)
    # scores 512 and 384: weight of key 1 is exp(-128) ~ 2.6e-56
    Vf = bf16_bits_to_f32(V).astype(np.float64)
    np.testing.assert_allclose(O[0, 0], Vf[0], rtol=1e-15, atol=1e-40)
