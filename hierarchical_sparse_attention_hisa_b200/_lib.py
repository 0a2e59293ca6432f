"""ctypes binding of libhsa.so (declared in include/hsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Tensors are torch CUDA tensors (used for device memory and streams);
their data pointers and the current CUDA stream are handed to the C ABI.
The library must have been built (``build.build()``); a missing library is an
ImportError, never a silent fallback.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

HSA_OK, HSA_ERR_ARG, HSA_ERR_WORKSPACE, HSA_ERR_CUDA, HSA_ERR_TIMEOUT, HSA_ERR_DEVICE = range(6)

# Every entry point declared in include/hsa.h.
EXPORTS = (
    "hsa_status_string", "hsa_index_workspace_size", "hsa_block_sums", "hsa_select_blocks",
    "hsa_select_tokens", "hsa_index", "hsa_sparse_attn", "hsa_decode_workspace_size",
    "hsa_decode_step", "hsa_kernel_launches", "hsa_decode_step_noalloc", "hsa_device_status",
    "hsa_prefill_host_workspace_size", "hsa_prefill_host", "hsa_debug_inject_lost_arrival",
)


class hsa_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("m", ctypes.c_int32), ("k", ctypes.c_int32),
                ("d_idx", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
                ("scale", ctypes.c_float)]


class HSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")
        self.status = status


_lib = None


def lib_path() -> str:
    return _build.LIB


def load():
    """Load libhsa.so (raises ImportError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise ImportError(f"libhsa.so not built at {path}; run build() first")
    L = ctypes.CDLL(path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    PP = ctypes.POINTER(hsa_params)
    L.hsa_status_string.argtypes, L.hsa_status_string.restype = [ctypes.c_int], ctypes.c_char_p
    L.hsa_index_workspace_size.argtypes = [PP, I64, I64, ctypes.POINTER(SZ)]
    L.hsa_block_sums.argtypes = [PP, I64, P, P, P]
    L.hsa_select_blocks.argtypes = [PP, I64, I64, P, P, P, P, SZ, P]
    L.hsa_select_tokens.argtypes = [PP, I64, I64, P, P, P, P, P, SZ, P]
    L.hsa_index.argtypes = [PP, I64, I64, P, P, P, P, SZ, P]
    L.hsa_sparse_attn.argtypes = [PP, I64, I64, P, P, P, P, P, P]
    L.hsa_decode_workspace_size.argtypes = [PP, I32, I64, ctypes.POINTER(SZ)]
    L.hsa_decode_step.argtypes = [PP, I32, I64, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    L.hsa_decode_step_noalloc.argtypes = [PP, I32, I64, P, P, P, P, P, P, P, P, P, P, P, P, P]
    L.hsa_kernel_launches.argtypes, L.hsa_kernel_launches.restype = [], ctypes.c_uint64
    L.hsa_device_status.argtypes = [ctypes.c_int]
    L.hsa_debug_inject_lost_arrival.argtypes = [ctypes.c_int]
    L.hsa_prefill_host_workspace_size.argtypes = [PP, I64, I64, ctypes.POINTER(SZ)]
    L.hsa_prefill_host.argtypes = [PP, I64, I64, P, P, P, P, P, P, P, P, SZ, P]
    for name in EXPORTS:
        if name not in ("hsa_status_string", "hsa_kernel_launches"):
            getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def kernel_launches() -> int:
    """Kernels launched by libhsa.so in this process so far."""
    return int(load().hsa_kernel_launches())


def hsa_device_status(reset: bool = True) -> int:
    """HSA_OK, or HSA_ERR_TIMEOUT if a bounded device wait gave up (synchronises the device)."""
    st = int(load().hsa_device_status(1 if reset else 0))
    if st not in (HSA_OK, HSA_ERR_TIMEOUT):
        raise HSAError("hsa_device_status", st)
    return st


def hsa_debug_inject_lost_arrival(on: bool) -> None:
    """Test hook: short bounded waits and one lost producer hand-off per tensor-core kernel."""
    _check("hsa_debug_inject_lost_arrival", int(load().hsa_debug_inject_lost_arrival(1 if on else 0)))


def status_string(status: int) -> str:
    return load().hsa_status_string(int(status)).decode()


def params(B=128, m=64, k=2048, d_idx=128, H=64, d=128, scale=0.0) -> hsa_params:
    return hsa_params(int(B), int(m), int(k), int(d_idx), int(H), int(d), float(scale))


def _p(t):
    """Data pointer of a tensor (None -> NULL); 0-size tensors pass NULL."""
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr()) if t.numel() else None


def _s(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn, status):
    if status != HSA_OK:
        raise HSAError(fn, status)


# ----------------------------------------------------------------- raw entry points
# Same names and argument order as the C ABI; tensors in place of pointers.

def hsa_index_workspace_size(p: hsa_params, Lq: int, Lk: int) -> int:
    n = ctypes.c_size_t(0)
    _check("hsa_index_workspace_size", load().hsa_index_workspace_size(ctypes.byref(p), Lq, Lk, ctypes.byref(n)))
    return n.value


def hsa_block_sums(p, Lk, k_idx, ksum, stream=None):
    _check("hsa_block_sums", load().hsa_block_sums(ctypes.byref(p), Lk, _p(k_idx), _p(ksum), _s(stream)))


def hsa_select_blocks(p, Lq, Lk, q_idx, ksum, blocks, workspace=None, stream=None):
    ws = _p(workspace)
    _check("hsa_select_blocks", load().hsa_select_blocks(
        ctypes.byref(p), Lq, Lk, _p(q_idx), _p(ksum), _p(blocks), ws,
        workspace.numel() * workspace.element_size() if workspace is not None else 0, _s(stream)))


def hsa_select_tokens(p, Lq, Lk, q_idx, k_idx, blocks, indices, workspace=None, stream=None):
    _check("hsa_select_tokens", load().hsa_select_tokens(
        ctypes.byref(p), Lq, Lk, _p(q_idx), _p(k_idx), _p(blocks), _p(indices), _p(workspace),
        workspace.numel() * workspace.element_size() if workspace is not None else 0, _s(stream)))


def hsa_index(p, Lq, Lk, q_idx, k_idx, indices, workspace, stream=None):
    _check("hsa_index", load().hsa_index(
        ctypes.byref(p), Lq, Lk, _p(q_idx), _p(k_idx), _p(indices), _p(workspace),
        workspace.numel() * workspace.element_size(), _s(stream)))


def hsa_sparse_attn(p, Lq, Lk, Q, K, V, indices, O, stream=None):
    _check("hsa_sparse_attn", load().hsa_sparse_attn(
        ctypes.byref(p), Lq, Lk, _p(Q), _p(K), _p(V), _p(indices), _p(O), _s(stream)))


def hsa_prefill_host_workspace_size(p, Lq, Lk) -> int:
    n = ctypes.c_size_t(0)
    _check("hsa_prefill_host_workspace_size",
           load().hsa_prefill_host_workspace_size(ctypes.byref(p), Lq, Lk, ctypes.byref(n)))
    return n.value


def hsa_prefill_host(p, Lq, Lk, q_idx_h, k_idx_h, Q_h, K_h, V_h, O_h, indices_h, workspace, stream=None):
    """Index + attention with host tensors in and out (page-locked for overlap); device workspace."""
    _check("hsa_prefill_host", load().hsa_prefill_host(
        ctypes.byref(p), Lq, Lk, _p(q_idx_h), _p(k_idx_h), _p(Q_h), _p(K_h), _p(V_h), _p(O_h),
        _p(indices_h), _p(workspace), workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _s(stream)))


def hsa_decode_workspace_size(p, batch, capacity) -> int:
    n = ctypes.c_size_t(0)
    _check("hsa_decode_workspace_size", load().hsa_decode_workspace_size(ctypes.byref(p), batch, capacity, ctypes.byref(n)))
    return n.value


def hsa_decode_step(p, batch, capacity, ctx_len, k_idx_cache, K_cache, V_cache, ksum_cache,
                    q_idx_new, k_idx_new, Q_new, K_new, V_new, O, indices_out, workspace,
                    stream=None):
    _check("hsa_decode_step", load().hsa_decode_step(
        ctypes.byref(p), batch, capacity, _p(ctx_len), _p(k_idx_cache), _p(K_cache),
        _p(V_cache), _p(ksum_cache), _p(q_idx_new), _p(k_idx_new), _p(Q_new), _p(K_new),
        _p(V_new), _p(O), _p(indices_out), _p(workspace),
        workspace.numel() * workspace.element_size(), _s(stream)))


def hsa_decode_step_noalloc(p, batch, capacity, ctx_len, k_idx_cache, K_cache, V_cache, ksum_cache,
                            q_idx_new, k_idx_new, Q_new, K_new, V_new, O, indices_out, stream=None):
    """hsa_decode_step with its scratch in the library's static device array."""
    _check("hsa_decode_step_noalloc", load().hsa_decode_step_noalloc(
        ctypes.byref(p), batch, capacity, _p(ctx_len), _p(k_idx_cache), _p(K_cache),
        _p(V_cache), _p(ksum_cache), _p(q_idx_new), _p(k_idx_new), _p(Q_new), _p(K_new),
        _p(V_new), _p(O), _p(indices_out), _s(stream)))
