"""Out-of-bounds writes: every output and workspace of hsa_index,
hsa_sparse_attn and hsa_decode_step sits between two 4 KiB guard regions
filled with a known byte; after the calls the guards must be untouched and
the outputs must equal those written into plain buffers. Cases: the tiny
prefill, a ragged chunk of the 16K prefill (Lq = 1000, not a multiple of
the 128-query tile) and two decode steps at batch 3.
"""
import numpy as np
import pytest

import synth
from helpers import dev

pytestmark = pytest.mark.gpu

GUARD = 4096
FILL = 0xA5


class Guarded:
    """A device buffer of `nbytes` between two guard regions of FILL bytes."""

    def __init__(self, nbytes):
        import torch
        self.n = nbytes
        self.buf = torch.full((2 * GUARD + nbytes,), FILL, dtype=torch.uint8, device="cuda")
        self.inner = self.buf[GUARD:GUARD + nbytes]

    def view(self, dtype, shape):
        return self.inner.view(dtype).view(shape)

    def guards_intact(self):
        head, tail = self.buf[:GUARD], self.buf[GUARD + self.n:]
        return bool((head == FILL).all().item()) and bool((tail == FILL).all().item())


@pytest.mark.parametrize("name,Lq", [("tiny_prefill_2k", None), ("prefill_16k", 1000)])
def test_prefill_writes_stay_inside_their_buffers(name, Lq):
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa
    hsa.build()
    w = synth.WORKLOADS[name]
    x = synth.prefill_inputs(w)
    Lq = w.Lq if Lq is None else Lq
    q_idx, k_idx = dev(x["q_idx"][w.Lq - Lq:]), dev(x["k_idx"])
    Q, K, V = dev(x["Q"][w.Lq - Lq:]), dev(x["K"]), dev(x["V"])
    p = hsa.params(B=w.B, m=w.m, k=w.k, d_idx=w.d_idx, H=w.H, d=w.d)
    nws = hsa.hsa_index_workspace_size(p, Lq, w.L)
    ws = Guarded(nws)
    idx = Guarded(Lq * w.k * 4)
    O = Guarded(Lq * w.H * w.d * 2)
    hsa.hsa_index(p, Lq, w.L, q_idx, k_idx, idx.view(torch.int32, (Lq, w.k)), ws.view(torch.uint8, (nws,)))
    hsa.hsa_sparse_attn(p, Lq, w.L, Q, K, V, idx.view(torch.int32, (Lq, w.k)),
                        O.view(torch.bfloat16, (Lq, w.H, w.d)))
    torch.cuda.synchronize()
    assert ws.guards_intact() and idx.guards_intact() and O.guards_intact()
    # the same results as in plain buffers
    idx_ref = hsa.index(q_idx, k_idx, w.B, w.m, w.k)
    O_ref = hsa.sparse_attn(Q, K, V, idx_ref)
    torch.cuda.synchronize()
    assert torch.equal(idx.view(torch.int32, (Lq, w.k)), idx_ref)
    assert torch.equal(O.view(torch.int16, (Lq, w.H, w.d)), O_ref.view(torch.int16))


def test_decode_writes_stay_inside_their_buffers():
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa
    hsa.build()
    p = hsa.params(B=64, m=8, k=256, d_idx=128, H=16, d=128)
    batch, capacity, steps, seed = 3, 1024, 2, 61
    ctx0 = [63, 500, 1000]  # the first step completes a block of sequence 0
    kc = Guarded(batch * capacity * p.d_idx * 2)
    Kc = Guarded(batch * capacity * p.d * 2)
    Vc = Guarded(batch * capacity * p.d * 2)
    ksum = Guarded(batch * (capacity // p.B) * p.d_idx * 4)
    ctx = Guarded(batch * 4)
    kc_t = kc.view(torch.bfloat16, (batch, capacity, p.d_idx))
    Kc_t = Kc.view(torch.bfloat16, (batch, capacity, p.d))
    Vc_t = Vc.view(torch.bfloat16, (batch, capacity, p.d))
    ks_t = ksum.view(torch.float32, (batch, capacity // p.B, p.d_idx))
    kc_t.copy_(dev(synth.int_bf16((batch, capacity, p.d_idx), seed, 2)))
    Kc_t.copy_(dev(synth.normal_bf16((batch, capacity, p.d), seed, 4)))
    Vc_t.copy_(dev(synth.normal_bf16((batch, capacity, p.d), seed, 5)))
    ks_t.zero_()
    for b in range(batch):
        hsa.hsa_block_sums(p, ctx0[b], kc_t[b], ks_t[b])
    ctx_t = ctx.view(torch.int32, (batch,))
    ctx_t.copy_(torch.tensor(ctx0, dtype=torch.int32))
    new = {
        "q": dev(synth.int_bf16((steps, batch, p.d_idx), seed, 30)),
        "k": dev(synth.int_bf16((steps, batch, p.d_idx), seed, 31)),
        "Q": dev(synth.normal_bf16((steps, batch, p.H, p.d), seed, 33)),
        "K": dev(synth.normal_bf16((steps, batch, p.d), seed, 34)),
        "V": dev(synth.normal_bf16((steps, batch, p.d), seed, 35)),
    }
    nws = hsa.hsa_decode_workspace_size(p, batch, capacity)
    ws = Guarded(nws)
    O = Guarded(batch * p.H * p.d * 2)
    idx = Guarded(batch * p.k * 4)
    for s in range(steps):
        hsa.hsa_decode_step(p, batch, capacity, ctx_t, kc_t, Kc_t, Vc_t, ks_t, new["q"][s], new["k"][s],
                            new["Q"][s], new["K"][s], new["V"][s], O.view(torch.bfloat16, (batch, p.H, p.d)),
                            idx.view(torch.int32, (batch, p.k)), ws.view(torch.uint8, (nws,)))
    torch.cuda.synchronize()
    for g in (kc, Kc, Vc, ksum, ctx, ws, O, idx):
        assert g.guards_intact()
    assert ctx_t.cpu().tolist() == [c + steps for c in ctx0]
