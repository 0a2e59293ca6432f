"""CPU oracle for hierarchical indexed sparse attention -- TEST INFRASTRUCTURE.

Thin numpy/ctypes front end to ``hsa_oracle.cpp`` (plain C++ loops, fp32
indexer scores, fp64 attention). Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this package; the product library
never does. See ``hsa_oracle.cpp`` for the method's steps and the readings of
points the pages leave open.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hsa_oracle.cpp")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libhsa_oracle.so")
# A prebuilt library in place of the one built here: the mutation tests use it
# to run the pins against copies of the oracle with a planted mistake.
_LIB_OVERRIDE = os.environ.get("HSA_ORACLE_LIB")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (no fused multiply-add contraction)."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fPIC",
                               "-shared", "-pthread", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_block_sums.argtypes = [P, I64, I32, I32, P]
        lib.oracle_select_blocks.argtypes = [P, P, I64, I64, I32, I32, I32, P, I64, P, I32]
        lib.oracle_select_tokens.argtypes = [P, P, P, I64, I64, I32, I32, I32, I32, P, I64, P, I32]
        lib.oracle_index.argtypes = [P, P, I64, I64, I32, I32, I32, I32, P, I64, P, P, I32]
        lib.oracle_sparse_attn.argtypes = [P, P, P, P, I64, I64, I32, I32, I32, D, P, I64, P, I32]
        _lib = lib
    return _lib


def default_threads() -> int:
    return os.cpu_count() or 1


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 inputs are passed as uint16 bit patterns"
    return a


def _rows(rows, n):
    if rows is None:
        return None, n
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, len(r)


def _ptr(a):
    return None if a is None else a.ctypes.data


def block_sums(k_idx, B: int) -> np.ndarray:
    k = _u16(k_idx)
    Lk, d_idx = k.shape
    out = np.zeros((Lk // B, d_idx), dtype=np.float32)
    assert _load().oracle_block_sums(_ptr(k), Lk, d_idx, B, _ptr(out)) == 0
    return out


def select_blocks(q_idx, ksum, Lk: int, B: int, m: int, rows=None, threads=None) -> np.ndarray:
    q = _u16(q_idx)
    ks = np.ascontiguousarray(ksum, dtype=np.float32)
    Lq, d_idx = q.shape
    r, n = _rows(rows, Lq)
    out = np.empty((n, m), dtype=np.int32)
    assert _load().oracle_select_blocks(_ptr(q), _ptr(ks), Lq, Lk, d_idx, B, m, _ptr(r), n,
                                        _ptr(out), threads or default_threads()) == 0
    return out


def select_tokens(q_idx, k_idx, blocks, B: int, k: int, rows=None, threads=None) -> np.ndarray:
    q, kk = _u16(q_idx), _u16(k_idx)
    bl = np.ascontiguousarray(blocks, dtype=np.int32)
    Lq, d_idx = q.shape
    Lk = kk.shape[0]
    r, n = _rows(rows, Lq)
    assert bl.shape[0] == n
    out = np.empty((n, k), dtype=np.int32)
    assert _load().oracle_select_tokens(_ptr(q), _ptr(kk), _ptr(bl), Lq, Lk, d_idx, B,
                                        bl.shape[1], k, _ptr(r), n, _ptr(out),
                                        threads or default_threads()) == 0
    return out


def index(q_idx, k_idx, B: int, m: int, k: int, rows=None, threads=None, with_blocks=False):
    """Both HISA stages: indices [n][k] (ascending, -1 padded)."""
    q, kk = _u16(q_idx), _u16(k_idx)
    Lq, d_idx = q.shape
    Lk = kk.shape[0]
    r, n = _rows(rows, Lq)
    out = np.empty((n, k), dtype=np.int32)
    blk = np.empty((n, m), dtype=np.int32) if with_blocks else None
    assert _load().oracle_index(_ptr(q), _ptr(kk), Lq, Lk, d_idx, B, m, k, _ptr(r), n,
                                _ptr(out), _ptr(blk), threads or default_threads()) == 0
    return (out, blk) if with_blocks else out


def sparse_attn(Q, K, V, indices, scale=None, rows=None, threads=None) -> np.ndarray:
    """fp64 softmax attention over the selected keys: O [n][H][d]."""
    Qa, Ka, Va = _u16(Q), _u16(K), _u16(V)
    idx = np.ascontiguousarray(indices, dtype=np.int32)
    Lq, H, d = Qa.shape
    Lk = Ka.shape[0]
    k = idx.shape[1]
    r, n = _rows(rows, Lq)
    assert idx.shape[0] == n
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((n, H, d), dtype=np.float64)
    assert _load().oracle_sparse_attn(_ptr(Qa), _ptr(Ka), _ptr(Va), _ptr(idx), Lq, Lk, H, d, k,
                                      float(scale), _ptr(r), n, _ptr(out),
                                      threads or default_threads()) == 0
    return out
