"""hsa_decode_step_noalloc against hsa_decode_step.

Some callers cannot allocate device memory at the point where they decode: a
framework that owns every allocation, or a serving loop that may not call
cudaMalloc once it runs. hsa_decode_step_noalloc serves them from a static
scratch array inside the library instead of a caller workspace. Here the two
entry points run two decode steps in a row on identical caches; their
outputs must agree within the attention tolerance of the other GPU tests,
and their indices, lengths and caches exactly. A step that needs more
scratch than the static array holds must be refused before anything runs.
"""
import numpy as np
import pytest

import synth
from helpers import ATOL_MAX, ATOL_MEAN, bf16_to_f64, dev, host_bits

pytestmark = pytest.mark.gpu


def make_state(hsa, p, batch, capacity, ctx0, seed):
    import torch
    kc = dev(synth.int_bf16((batch, capacity, p.d_idx), seed, 2))
    Kc = dev(synth.normal_bf16((batch, capacity, p.d), seed, 4))
    Vc = dev(synth.normal_bf16((batch, capacity, p.d), seed, 5))
    ksum = torch.zeros((batch, capacity // p.B, p.d_idx), dtype=torch.float32, device="cuda")
    for b in range(batch):
        hsa.hsa_block_sums(p, int(ctx0[b]), kc[b], ksum[b])
    ctx = torch.tensor(ctx0, dtype=torch.int32, device="cuda")
    return {"k": kc, "K": Kc, "V": Vc, "ksum": ksum, "ctx": ctx}


def test_noalloc_decode_matches_workspace_decode():
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa
    assert torch.cuda.is_available()
    hsa.build()
    hsa.load()
    p = hsa.params(B=64, m=8, k=256, d_idx=128, H=16, d=128)
    batch, capacity, seed = 4, 2048, 50
    ctx0 = [63, 500, 1000, 1500]  # the first step completes a block of sequence 0
    a = make_state(hsa, p, batch, capacity, ctx0, seed)
    b = make_state(hsa, p, batch, capacity, ctx0, seed)
    ws = torch.empty(hsa.hsa_decode_workspace_size(p, batch, capacity), dtype=torch.uint8, device="cuda")
    steps = 2
    new = {
        "q": dev(synth.int_bf16((steps, batch, p.d_idx), seed, 30)),
        "k": dev(synth.int_bf16((steps, batch, p.d_idx), seed, 31)),
        "Q": dev(synth.normal_bf16((steps, batch, p.H, p.d), seed, 33)),
        "K": dev(synth.normal_bf16((steps, batch, p.d), seed, 34)),
        "V": dev(synth.normal_bf16((steps, batch, p.d), seed, 35)),
    }
    for s in range(steps):
        Oa = torch.empty((batch, p.H, p.d), dtype=torch.bfloat16, device="cuda")
        Ob = torch.empty_like(Oa)
        ia = torch.empty((batch, p.k), dtype=torch.int32, device="cuda")
        ib = torch.empty_like(ia)
        hsa.hsa_decode_step(p, batch, capacity, a["ctx"], a["k"], a["K"], a["V"], a["ksum"],
                            new["q"][s], new["k"][s], new["Q"][s], new["K"][s], new["V"][s], Oa, ia, ws)
        hsa.hsa_decode_step_noalloc(p, batch, capacity, b["ctx"], b["k"], b["K"], b["V"], b["ksum"],
                                    new["q"][s], new["k"][s], new["Q"][s], new["K"][s], new["V"][s],
                                    Ob, ib)
        torch.cuda.synchronize()
        oa, ob = bf16_to_f64(host_bits(Oa)), bf16_to_f64(host_bits(Ob))
        err = np.abs(oa - ob)
        assert np.isfinite(ob).all()
        assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (s, err.max(), err.mean())
        assert np.array_equal(ia.cpu().numpy(), ib.cpu().numpy()), s
        assert np.array_equal(a["ctx"].cpu().numpy(), b["ctx"].cpu().numpy()), s
        for name in ("k", "K", "V", "ksum"):
            assert torch.equal(a[name], b[name]), (s, name)
    assert b["ctx"].cpu().tolist() == [c + steps for c in ctx0]


def test_noalloc_refuses_more_scratch_than_the_static_array():
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa
    from hierarchical_sparse_attention_hisa_b200._lib import HSA_ERR_WORKSPACE
    hsa.load()
    p = hsa.params(B=64, m=8, k=256, d_idx=128, H=16, d=128)
    capacity = 256
    batch = 9000  # batch * (m + k) * 4 bytes of scratch > 8 MiB
    assert hsa.hsa_decode_workspace_size(p, batch, capacity) > (8 << 20)
    ctx = torch.zeros(batch, dtype=torch.int32, device="cuda")
    with pytest.raises(hsa.HSAError) as e:
        hsa.hsa_decode_step_noalloc(p, batch, capacity, ctx, None, None, None, None, None, None,
                                    None, None, None, None, None)
    assert e.value.status == HSA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(ctx.sum().item()) == 0
