"""The seeded synthetic inputs follow their stated recipe: bf16 rounding to
nearest-even (checked against torch's conversion), integer indexer values
uniform in [-8, 8], N(0, 1) attention values, streams that depend only on
(seed, tensor id, chunk) and not on the thread count, and needles planted
as described (distinct query rows i >= B*m, distinct earlier key rows j,
k_idx[j] = q_idx[i])."""
import numpy as np
import pytest

import synth


def test_bf16_rounding_is_nearest_even():
    import torch
    ulp = 2.0 ** -7
    # ties: halfway between neighbouring bf16 values (the bf16 spacing is ulp in [1, 2), 2 ulp in [2, 4))
    halfway = np.array([1 + ulp / 2, 1 + 3 * ulp / 2, -(1 + ulp / 2), 3.0 + ulp], dtype=np.float32)
    want = np.array([1.0, 1 + 2 * ulp, -1.0, 3.0], dtype=np.float32)  # ties go to the even mantissa
    assert np.array_equal(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(halfway)), want)
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(200_000) * np.exp(rng.uniform(-20, 20, 200_000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f32_to_bf16_bits(x), ref)


def test_bf16_widening_is_exact():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = synth.bf16_bits_to_f32(bits)
    finite = np.isfinite(f)
    assert np.array_equal(synth.f32_to_bf16_bits(f[finite]), bits[finite])


def test_streams_depend_only_on_seed_tensor_and_chunk():
    n = synth.CHUNK * 2 + 12345
    a = synth._fill((n,), 3, 7, "int", threads=1)
    b = synth._fill((n,), 3, 7, "int", threads=8)
    assert np.array_equal(a, b)
    # a longer tensor starts with the same chunks
    c = synth._fill((n + synth.CHUNK,), 3, 7, "int", threads=4)
    assert np.array_equal(c[: 2 * synth.CHUNK], a[: 2 * synth.CHUNK])
    assert not np.array_equal(synth.int_bf16((1000,), 3, 7), synth.int_bf16((1000,), 3, 8))
    assert not np.array_equal(synth.int_bf16((1000,), 3, 7), synth.int_bf16((1000,), 4, 7))


def test_indexer_values_are_uniform_integers_in_range():
    v = synth.bf16_bits_to_f32(synth.int_bf16((170_000,), 0, 1)).astype(np.float64)
    assert np.all(v == np.round(v)) and v.min() == -8 and v.max() == 8
    counts = np.bincount((v + 8).astype(np.int64), minlength=17)
    assert counts.min() > 0.9 * 10_000 and counts.max() < 1.1 * 10_000


def test_attention_values_are_standard_normal():
    v = synth.bf16_bits_to_f32(synth.normal_bf16((1_000_000,), 0, 3)).astype(np.float64)
    assert abs(v.mean()) < 5e-3 and abs(v.std() - 1.0) < 5e-3
    assert abs(np.mean(np.abs(v) < 1.0) - 0.6827) < 3e-3


@pytest.mark.parametrize("Lk,B,m,count", [(4096, 64, 8, 32), (300, 16, 4, 10)])
def test_needles_are_planted_as_described(Lk, B, m, count):
    q = synth.int_bf16((Lk, 8), 1, synth.T_Q_IDX)
    k = synth.int_bf16((Lk, 8), 1, synth.T_K_IDX)
    k0 = k.copy()
    pairs = synth.plant_needles(q, k, Lk, B, m, count, seed=1)
    assert len(pairs) == count
    qi = [i for i, _ in pairs]
    kj = [j for _, j in pairs]
    assert len(set(qi)) == count and len(set(kj)) == count
    assert all(min(B * m, Lk - 1) <= i < Lk and 0 <= j < i for i, j in pairs)
    for i, j in pairs:
        assert np.array_equal(k[j], q[i])
    untouched = np.setdiff1d(np.arange(Lk), kj)
    assert np.array_equal(k[untouched], k0[untouched])


def test_prefill_workload_shapes():
    w = synth.WORKLOADS["tiny_prefill_2k"]
    x = synth.prefill_inputs(w)
    assert x["q_idx"].shape == (w.Lq, w.d_idx) and x["k_idx"].shape == (w.L, w.d_idx)
    assert x["Q"].shape == (w.Lq, w.H, w.d) and x["K"].shape == (w.L, w.d) and x["V"].shape == (w.L, w.d)
    assert x["needles"] == []
    y = synth.prefill_inputs(w)
    assert all(np.array_equal(x[n], y[n]) for n in ("q_idx", "k_idx", "Q", "K", "V"))
