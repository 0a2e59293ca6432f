"""No bounded device wait gave up during the GPU tests.

The tensor-core kernels bound every mbarrier wait; one that runs out sets a
sticky per-device flag and the launch skips the work behind it, so its outputs
would be incomplete. pytest runs test files in name order, so this file runs
after every other GPU test of the session and reads the flag once for all of
them through hsa_device_status.
"""
import pytest


@pytest.mark.gpu
def test_no_bounded_wait_gave_up():
    import torch
    import hierarchical_sparse_attention_hisa_b200 as hsa
    from hierarchical_sparse_attention_hisa_b200._lib import HSA_OK
    assert torch.cuda.is_available()
    hsa.build()
    assert hsa.hsa_device_status(reset=False) == HSA_OK
