"""hsa_prefill_host (host tensors in and out, the copies overlapped with the
kernels chunk by chunk) against hsa_index + hsa_sparse_attn on device tensors:
the same indices and the same O bits, on page-locked and pageable buffers, for
a whole prefill and for a ragged chunk of queries (Lq < Lk, Lq not a multiple
of the 128-query tile). It runs after the other GPU tests (file name order)
and checks the device wait flags itself.
"""
import numpy as np
import pytest

import synth
from helpers import dev

pytestmark = pytest.mark.gpu


def host_bf16(u16, pin):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pin else t


@pytest.mark.parametrize("name,Lq,pin,with_idx", [
    ("tiny_prefill_2k", None, True, True),
    ("tiny_prefill_2k", None, False, True),
    ("prefill_16k", None, True, False),
    ("prefill_16k", 1000, True, True),
])
def test_prefill_host_matches_the_device_path(name, Lq, pin, with_idx):
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa
    from hierarchical_sparse_attention_hisa_b200._lib import HSA_OK
    hsa.build()
    w = synth.WORKLOADS[name]
    x = synth.prefill_inputs(w)
    L = w.L
    Lq = w.Lq if Lq is None else Lq
    q_idx, Q = x["q_idx"][w.Lq - Lq:], x["Q"][w.Lq - Lq:]
    # the device path
    idx_d = hsa.index(dev(q_idx), dev(x["k_idx"]), w.B, w.m, w.k)
    O_d = hsa.sparse_attn(dev(Q), dev(x["K"]), dev(x["V"]), idx_d)
    torch.cuda.synchronize()
    # the host path
    p = hsa.params(B=w.B, m=w.m, k=w.k, d_idx=w.d_idx, H=w.H, d=w.d)
    ws = torch.empty(hsa.hsa_prefill_host_workspace_size(p, Lq, L), dtype=torch.uint8, device="cuda")
    O_h = torch.full((Lq, w.H, w.d), 7.0, dtype=torch.bfloat16)
    idx_h = torch.full((Lq, w.k), -7, dtype=torch.int32) if with_idx else None
    if pin:
        O_h = O_h.pin_memory()
        idx_h = idx_h.pin_memory() if idx_h is not None else None
    hsa.hsa_prefill_host(p, Lq, L, host_bf16(q_idx, pin), host_bf16(x["k_idx"], pin), host_bf16(Q, pin),
                         host_bf16(x["K"], pin), host_bf16(x["V"], pin), O_h, idx_h, ws)
    torch.cuda.synchronize()
    assert torch.equal(O_h.view(torch.int16), O_d.cpu().view(torch.int16))
    if with_idx:
        assert torch.equal(idx_h, idx_d.cpu())
    assert hsa.hsa_device_status(reset=False) == HSA_OK
