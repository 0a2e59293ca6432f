"""B200-native hierarchical indexed sparse attention (HISA).

Two-stage selection (blocks of B keys scored by their summed representative,
top-m kept with the first and the query's own block forced; then the tokens
of those blocks scored and the top-k kept) followed by exact sparse softmax
attention over the k kept tokens, shared by the H heads of a multi-query
layer. The work runs in libhsa.so (hand-written sm_100a CUDA behind a C ABI,
see include/hsa.h); this package marshals torch tensors into it.

    import hierarchical_sparse_attention_hisa_b200 as hsa
    idx = hsa.index(q_idx, k_idx, B=128, m=64, k=2048)
    O = hsa.sparse_attn(Q, K, V, idx)
"""
from __future__ import annotations

from ._lib import (EXPORTS, HSAError, hsa_block_sums, hsa_decode_step,  # noqa: F401
                   hsa_debug_inject_lost_arrival, hsa_decode_step_noalloc, hsa_device_status,
                   hsa_prefill_host,
                   hsa_prefill_host_workspace_size,
                   hsa_decode_workspace_size, hsa_index, hsa_index_workspace_size, hsa_params,
                   hsa_select_blocks, hsa_select_tokens, hsa_sparse_attn, kernel_launches, lib_path, load,
                   params, status_string)
from .build import build  # noqa: F401


def _check_bf16(name, t, ndim):
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != ndim:
        raise ValueError(f"{name}: expected a contiguous {ndim}-d bf16 CUDA tensor")


def index(q_idx, k_idx, B: int, m: int, k: int, stream=None):
    """indices [Lq][k] int32 for queries at positions Lk-Lq .. Lk-1."""
    import torch
    _check_bf16("q_idx", q_idx, 2)
    _check_bf16("k_idx", k_idx, 2)
    Lq, d_idx = q_idx.shape
    Lk = k_idx.shape[0]
    p = params(B=B, m=m, k=k, d_idx=d_idx)
    ws = torch.empty(max(hsa_index_workspace_size(p, Lq, Lk), 16), dtype=torch.uint8,
                     device=q_idx.device)
    out = torch.empty((Lq, k), dtype=torch.int32, device=q_idx.device)
    hsa_index(p, Lq, Lk, q_idx, k_idx, out, ws, stream)
    return out


def sparse_attn(Q, K, V, indices, scale: float = 0.0, stream=None):
    """O [Lq][H][d] bf16 = softmax attention of Q over the indexed rows of K/V."""
    import torch
    _check_bf16("Q", Q, 3)
    _check_bf16("K", K, 2)
    _check_bf16("V", V, 2)
    Lq, H, d = Q.shape
    p = params(k=indices.shape[1], H=H, d=d, scale=scale)
    O = torch.empty_like(Q)
    hsa_sparse_attn(p, Lq, K.shape[0], Q, K, V, indices, O, stream)
    return O
