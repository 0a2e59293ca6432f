"""Failure detection without a GPU fault: a producer hand-off that never comes.

The tensor-core kernels bound every mbarrier wait. With the library's test
hook on (hsa_debug_inject_lost_arrival), each of them loses one producer
hand-off in its first CTA (the scoring kernels never produce their first
tile; the attention's first K-tile arrival is not made) and its waits give up
after about a millisecond. The launch must then return on its own, nothing
may fault, hsa_device_status must report HSA_ERR_TIMEOUT, and once the hook is
off and the flag cleared the same calls must give the same results as before.
Runs after the check that no wait gave up during the other GPU tests.
"""
import time

import numpy as np
import pytest

import synth
from helpers import dev

pytestmark = pytest.mark.gpu


def test_lost_arrival_times_out_and_recovers():
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa
    from hierarchical_sparse_attention_hisa_b200._lib import HSA_ERR_TIMEOUT, HSA_OK
    assert torch.cuda.is_available()
    hsa.build()
    hsa.load()
    w = synth.WORKLOADS["tiny_prefill_2k"]   # block and token scoring and attention on tensor cores
    x = synth.prefill_inputs(w)
    q, k = dev(x["q_idx"]), dev(x["k_idx"])
    Q, K, V = dev(x["Q"]), dev(x["K"]), dev(x["V"])
    idx_ref = hsa.index(q, k, w.B, w.m, w.k)
    O_ref = hsa.sparse_attn(Q, K, V, idx_ref)
    torch.cuda.synchronize()
    assert hsa.hsa_device_status(reset=True) == HSA_OK
    try:
        hsa.hsa_debug_inject_lost_arrival(True)
        t0 = time.time()
        hsa.index(q, k, w.B, w.m, w.k)
        st_index = hsa.hsa_device_status(reset=True)
        hsa.sparse_attn(Q, K, V, idx_ref)
        st_attn = hsa.hsa_device_status(reset=True)
        elapsed = time.time() - t0
    finally:
        hsa.hsa_debug_inject_lost_arrival(False)
        hsa.hsa_device_status(reset=True)
    assert st_index == HSA_ERR_TIMEOUT, "the scoring kernels' lost tile went unnoticed"
    assert st_attn == HSA_ERR_TIMEOUT, "the attention's lost arrival went unnoticed"
    assert elapsed < 30.0, f"the shortened waits took {elapsed:.1f} s"
    # the context is still usable: a clean rerun gives the same results
    idx2 = hsa.index(q, k, w.B, w.m, w.k)
    O2 = hsa.sparse_attn(Q, K, V, idx2)
    torch.cuda.synchronize()
    assert hsa.hsa_device_status(reset=False) == HSA_OK
    assert torch.equal(idx2, idx_ref)
    assert torch.equal(O2.view(torch.int16), O_ref.view(torch.int16))
