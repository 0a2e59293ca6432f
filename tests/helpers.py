"""Shared test helpers: moving seeded synthetic inputs onto the GPU and
comparing GPU results with the oracle."""
import numpy as np

ATOL_MAX = 2e-2   # attention tolerance: max-abs error of bf16 O (fp32 accumulate)
ATOL_MEAN = 2e-3  # attention tolerance: mean-abs error


def dev(u16, device="cuda"):
    """bf16 bit array (uint16) -> torch bf16 tensor on the device."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).to(device).view(torch.bfloat16)


def host_bits(t):
    """torch bf16 tensor -> uint16 bit array on the host."""
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(u16):
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_attn_close(gpu_bits, ref, what=""):
    got = bf16_to_f64(gpu_bits)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= ATOL_MAX, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= ATOL_MEAN, f"{what}: mean-abs {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def sample_rows(Lq, n, seed, always=()):
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in always if 0 <= r < Lq)
    rows |= set(int(r) for r in rng.choice(Lq, size=min(n, Lq), replace=False))
    return np.array(sorted(rows), dtype=np.int64)
