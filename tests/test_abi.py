"""CPU checks of the C-ABI library: it loads, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from hierarchical_sparse_attention_hisa_b200 import build, load
    build()
    return load()


def header_functions():
    text = open(os.path.join(ROOT, "include", "hsa.h")).read()
    return sorted(set(re.findall(r"HSA_API\s+[\w\s\*]+?\b(hsa_\w+)\s*\(", text)))


def test_header_lists_entry_points():
    names = header_functions()
    assert "hsa_index" in names and "hsa_sparse_attn" in names and "hsa_decode_step" in names
    from hierarchical_sparse_attention_hisa_b200._lib import EXPORTS
    assert sorted(EXPORTS) == names


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_only_declared_symbols_are_exported(lib):
    import subprocess
    from hierarchical_sparse_attention_hisa_b200 import lib_path
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path()], capture_output=True,
                         text=True).stdout
    exported = sorted(set(re.findall(r"\bT (hsa_\w+)", out)))
    assert exported == header_functions()


C_CALLER = r"""
#include <string.h>
#include "hsa.h"
int main(void) {
  hsa_params p = {128, 64, 2048, 128, 64, 128, 0.0f};
  size_t n = 0;
  if (hsa_index_workspace_size(&p, 65536, 65536, &n) != HSA_OK || n == 0) return 1;
  if (hsa_prefill_host_workspace_size(&p, 65536, 65536, &n) != HSA_OK || n == 0) return 2;
  if (strcmp(hsa_status_string(HSA_OK), "ok") != 0) return 3;
  p.m = 1;
  if (hsa_index_workspace_size(&p, 100, 200, &n) != HSA_ERR_ARG) return 4;
  return 0;
}
"""


def test_header_is_plain_c_and_links_from_c(lib, tmp_path):
    """include/hsa.h compiles as strict C99 and a C program links libhsa.so and calls it."""
    import shutil
    import subprocess
    from hierarchical_sparse_attention_hisa_b200 import lib_path
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(lib_path())
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), "-isystem", cuda_inc, str(src), "-L", libdir, "-lhsa",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0


def test_status_strings(lib):
    from hierarchical_sparse_attention_hisa_b200 import status_string
    assert status_string(0) == "ok"
    for s in range(1, 6):
        assert status_string(s) and status_string(s) != "unknown status"
    assert status_string(99) == "unknown status"


def test_workspace_sizes_on_host(lib):
    import hierarchical_sparse_attention_hisa_b200 as hsa
    p = hsa.params(B=128, m=64, k=2048, d_idx=128, H=64, d=128)
    n = hsa.hsa_index_workspace_size(p, 65536, 65536)
    assert n >= 512 * 128 * 4 + 65536 * 64 * 4
    assert hsa.hsa_decode_workspace_size(p, 32, 131072 + 256) > 0


@pytest.mark.parametrize("field,value", [("B", 0), ("m", 1), ("k", 0), ("d_idx", 96),
                                         ("m", 513), ("B", 2048)])
def test_bad_index_params_rejected(lib, field, value):
    import hierarchical_sparse_attention_hisa_b200 as hsa
    p = hsa.params(B=128, m=64, k=2048, d_idx=128)
    setattr(p, field, value)
    n = ctypes.c_size_t(0)
    assert lib.hsa_index_workspace_size(ctypes.byref(p), 100, 200, ctypes.byref(n)) == 1
    # the full call is rejected on the host as well (no pointers needed)
    assert lib.hsa_index(ctypes.byref(p), 100, 200, None, None, None, None, 0, None) == 1


@pytest.mark.parametrize("B,m,ok", [(128, 512, True), (256, 256, True), (256, 257, False),
                                    (96, 170, True), (96, 171, False)])
def test_candidate_limits(lib, B, m, ok):
    # at most 65,536 candidates per row (m * B) when B is 64, 128 or 256, else 16,384
    import hierarchical_sparse_attention_hisa_b200 as hsa
    p = hsa.params(B=B, m=m, k=256, d_idx=128)
    n = ctypes.c_size_t(0)
    assert (lib.hsa_index_workspace_size(ctypes.byref(p), 100, 200, ctypes.byref(n)) == 0) == ok


def test_bad_lengths_and_pointers_rejected(lib):
    import hierarchical_sparse_attention_hisa_b200 as hsa
    p = hsa.params(B=64, m=8, k=256, d_idx=64, H=4, d=64)
    n = ctypes.c_size_t(0)
    assert lib.hsa_index_workspace_size(ctypes.byref(p), 300, 200, ctypes.byref(n)) == 1  # Lq > Lk
    # null pointers
    assert lib.hsa_index(ctypes.byref(p), 10, 20, None, None, None, None, 0, None) == 1
    assert lib.hsa_sparse_attn(ctypes.byref(p), 10, 20, None, None, None, None, None, None) == 1
    # misaligned pointer
    bad = ctypes.c_void_p(0x1001)
    assert lib.hsa_sparse_attn(ctypes.byref(p), 10, 20, bad, bad, bad, bad, bad, None) == 1
    p.d = 96
    assert lib.hsa_sparse_attn(ctypes.byref(p), 10, 20, None, None, None, None, None, None) == 1
    p.d, p.H = 64, 0
    assert lib.hsa_sparse_attn(ctypes.byref(p), 10, 20, None, None, None, None, None, None) == 1


def test_prefill_host_checks_on_the_host(lib):
    import hierarchical_sparse_attention_hisa_b200 as hsa
    from hierarchical_sparse_attention_hisa_b200._lib import HSA_ERR_ARG, HSA_ERR_WORKSPACE
    p = hsa.params(B=128, m=64, k=2048, d_idx=128, H=64, d=128)
    n = hsa.hsa_prefill_host_workspace_size(p, 65536, 65536)
    copies = 65536 * 128 * 2 * 4 + 2 * 65536 * 64 * 128 * 2 + 65536 * 2048 * 4
    assert n >= hsa.hsa_index_workspace_size(p, 65536, 65536) + copies
    sz = ctypes.c_size_t(0)
    bad = hsa.params(B=128, m=64, k=2048, d_idx=128, H=0, d=128)  # an attention argument
    assert lib.hsa_prefill_host_workspace_size(ctypes.byref(bad), 100, 200, ctypes.byref(sz)) == HSA_ERR_ARG
    q = hsa.params(B=64, m=8, k=256, d_idx=64, H=4, d=64)
    host = ctypes.c_void_p(0x1000)
    # missing host buffers, then a misaligned workspace: refused before anything is enqueued
    assert lib.hsa_prefill_host(ctypes.byref(q), 100, 200, None, None, None, None, None, None, None,
                                None, 0, None) == HSA_ERR_ARG
    assert lib.hsa_prefill_host(ctypes.byref(q), 100, 200, host, host, host, host, host, host, None,
                                ctypes.c_void_p(0x1010), 1 << 30, None) == HSA_ERR_WORKSPACE
    assert lib.hsa_prefill_host(ctypes.byref(q), 0, 200, None, None, None, None, None, None, None,
                                None, 0, None) == 0


def test_device_status_without_a_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: covered by test_zz_wait_status")
    from hierarchical_sparse_attention_hisa_b200._lib import HSA_ERR_CUDA
    assert lib.hsa_device_status(0) == HSA_ERR_CUDA


def test_zero_queries_is_a_no_op(lib):
    import hierarchical_sparse_attention_hisa_b200 as hsa
    p = hsa.params(B=64, m=8, k=256, d_idx=64, H=4, d=64)
    assert lib.hsa_index(ctypes.byref(p), 0, 20, None, None, None, None, 0, None) == 0
    assert lib.hsa_sparse_attn(ctypes.byref(p), 0, 20, None, None, None, None, None, None) == 0


def test_product_path_has_no_oracle_or_cpu_fallback():
    pkg = os.path.join(ROOT, "hierarchical_sparse_attention_hisa_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "hsa_oracle" not in src, f
