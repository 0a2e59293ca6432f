"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C++ source (a dropped
forced block, a flipped tie rule, a wrong causal bound or query position, a
block sum short of a row, a wrong range of scored blocks or block tokens, a
missing softmax scale, maximum shift or normalisation, unsorted or
zero-padded output, V swapped for K), builds it, and runs the oracle's
own pin tests (tests/test_oracle.py) against it: at least one pin must
fail. The unmodified source, built the same way, must pass them all.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hsa_oracle.cpp")

BLOCK_SORT = "      return x.second < y.second;\n    });\n    std::vector<int64_t> kept = {0, nb - 1};"
TOKEN_SORT = "        return x.second < y.second;\n      });\n      for (int s = 0; s < k; ++s) kept.push_back(sc[s].second);"

# name -> (text in the source, its replacement)
MUTATIONS = {
    "own block not forced": (
        "std::vector<int64_t> kept = {0, nb - 1};\n    for (int s = 0; s < m - 2; ++s)",
        "std::vector<int64_t> kept = {0};\n    for (int s = 0; s < m - 1 && s < int(cand.size()); ++s)"),
    "first block not forced": (
        "std::vector<int64_t> kept = {0, nb - 1};\n    for (int s = 0; s < m - 2; ++s)",
        "std::vector<int64_t> kept = {nb - 1};\n    for (int s = 0; s < m - 1 && s < int(cand.size()); ++s)"),
    "block ties to the highest id": (BLOCK_SORT, BLOCK_SORT.replace("x.second < y.second", "x.second > y.second")),
    "token ties to the highest index": (TOKEN_SORT, TOKEN_SORT.replace("x.second < y.second", "x.second > y.second")),
    "keys j < t only": ("j < (b + 1) * B && j <= t; ++j)", "j < (b + 1) * B && j < t; ++j)"),
    "query position t = i": ("const int64_t t = Lk - Lq + i;", "const int64_t t = i;"),
    "block sum misses a row": ("for (int64_t j = b * B; j < (b + 1) * B; ++j) s +=",
                               "for (int64_t j = b * B + 1; j < (b + 1) * B; ++j) s +="),
    "no softmax scale": ("x[a] = s * scale;", "x[a] = s;"),
    "no maximum shift": ("std::exp(x[a] - mx)", "std::exp(x[a])"),
    "indices not sorted": ("    std::sort(kept.begin(), kept.end());\n    int32_t* out = indices + r * k;",
                           "    int32_t* out = indices + r * k;"),
    "padding with 0": ("static_cast<int32_t>(kept[s]) : -1;", "static_cast<int32_t>(kept[s]) : 0;"),
    "V replaced by K": ("o[c] += p * bf16_to_float(V[S[a] * d + c]);", "o[c] += p * bf16_to_float(K[S[a] * d + c]);"),
    "block 0 among the scored": ("for (int64_t b = 1; b <= nb - 2; ++b) {", "for (int64_t b = 0; b <= nb - 2; ++b) {"),
    "last complete block never scored": ("for (int64_t b = 1; b <= nb - 2; ++b) {",
                                         "for (int64_t b = 1; b < nb - 2; ++b) {"),
    "a block spills one token into the next": ("j < (b + 1) * B && j <= t; ++j)", "j <= (b + 1) * B && j <= t; ++j)"),
    "no normalisation": ("for (int c = 0; c < d; ++c) o[c] /= l;", ""),
}


def build_and_run_pins(src_text, workdir):
    """Build `src_text` as the oracle library in `workdir` and run tests/test_oracle.py on it;
    returns pytest's exit status."""
    os.makedirs(workdir, exist_ok=True)
    src = os.path.join(workdir, "hsa_oracle.cpp")
    lib = os.path.join(workdir, "libhsa_oracle.so")
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread", src,
                    "-o", lib], check=True)
    env = dict(os.environ, HSA_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    return r.returncode


def test_unmodified_oracle_passes_its_pins(tmp_path):
    with open(SRC) as f:
        assert build_and_run_pins(f.read(), str(tmp_path / "clean")) == 0


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with open(SRC) as f:
        clean = f.read()
    jobs = {}
    for i, (name, (old, new)) in enumerate(MUTATIONS.items()):
        assert clean.count(old) >= 1, f"{name}: anchor not in the oracle source"
        jobs[name] = (clean.replace(old, new), str(tmp_path / f"m{i}"))
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        status = dict(zip(jobs, ex.map(lambda j: build_and_run_pins(*j), jobs.values())))
    # pytest's status 1: some pin failed (not a crash, not a collection error)
    missed = {name: rc for name, rc in status.items() if rc != 1}
    assert not missed, f"mistakes no pin catches (pytest status): {missed}"
