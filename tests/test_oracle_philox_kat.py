"""Word-for-word pins of the oracle's Philox4x32-10, on the CPU.

1. The published known answer (tests/golden/philox4x32_10_kat.txt): the C++26
   standard fixes the 10000th word of a default-constructed philox4x32.
2. Two independent host implementations of the same published generator,
   compiled here from their headers (tests/philox_engines_host.cpp): the
   C++26 standard engine as shipped in libcudacxx, and PyTorch's
   at::Philox4_32.  Every word of every block must agree with the oracle on
   edge and random (counter, key) pairs, including the counters the
   verification rule uses ((d, g, 0, 0) and (x / 4, g, 1, 0)).
The generator's counter and key layout (key = seed, counters keyed by request
and position or token) is this library's convention; the pages name no
generator."""
import importlib.util
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden", "philox4x32_10_kat.txt")
PROBE = os.path.join(ROOT, "tests", "philox_engines_host.cpp")


def read_kat():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(v) for v in line.split()])
    return rows


def test_published_known_answer(svo):
    rows = read_kat()
    assert rows
    for c0, c1, c2, c3, k0, k1, word, value in rows:
        assert svo.philox4x32_10([c0, c1, c2, c3], [k0, k1])[word] == value


def _include_dirs():
    """(libcudacxx include dir or None, torch include dir or None)."""
    std_dir = None
    spec = importlib.util.find_spec("flashinfer")
    if spec and spec.submodule_search_locations:
        for loc in spec.submodule_search_locations:
            d = os.path.join(loc, "data", "cccl", "libcudacxx", "include")
            if os.path.exists(os.path.join(d, "cuda", "std", "__random", "philox_engine.h")):
                std_dir = d
    torch_dir = None
    spec = importlib.util.find_spec("torch")
    if spec and spec.submodule_search_locations:
        for loc in spec.submodule_search_locations:
            d = os.path.join(loc, "include")
            if os.path.exists(os.path.join(d, "ATen", "core", "PhiloxRNGEngine.h")):
                torch_dir = d
    return std_dir, torch_dir


@pytest.fixture(scope="module")
def engines(tmp_path_factory):
    std_dir, torch_dir = _include_dirs()
    if shutil.which("g++") is None or (std_dir is None and torch_dir is None):
        pytest.skip("no host compiler or no engine headers")
    exe = str(tmp_path_factory.mktemp("philox") / "engines")
    cmd = ["g++", "-std=c++17", "-O1", PROBE, "-o", exe]
    kinds = []
    if std_dir:
        cmd[1:1] = ["-DWITH_STD_ENGINE", "-I", std_dir]
        kinds.append("std")
    if torch_dir:
        cmd[1:1] = ["-DWITH_TORCH_ENGINE", "-I", torch_dir]
        kinds.append("torch")
    subprocess.run(cmd, check=True, capture_output=True)
    return exe, kinds


def run_engines(engines, pairs):
    exe, kinds = engines
    text = "".join(" ".join(str(int(v)) for v in c + k) + "\n" for c, k in pairs)
    out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout
    res = {kind: [] for kind in kinds}
    for line in out.splitlines():
        parts = line.split()
        res[parts[0]].append([int(v) for v in parts[1:]])
    for kind in kinds:
        assert len(res[kind]) == len(pairs)
    return res


def pairs_to_check():
    rng = np.random.default_rng(2024)
    M = 2**32 - 1
    pairs = [([0, 0, 0, 0], [0, 0]), ([M, M, M, M], [M, M]), ([2499, 0, 0, 0], [20111115, 0]),
             ([1, 2, 3, 4], [5, 6])]
    # the rule's own counters: accept draws (d, g, 0, 0), race blocks (x / 4, g, 1, 0)
    for seed in (0, 7, 2**40 + 3):
        key = [seed & M, seed >> 32]
        for g in (0, 1, 255, 70000):
            for d in range(8):
                pairs.append(([d, g, 0, 0], key))
            for i in (0, 1, 1023, 32063, 38015):
                pairs.append(([i, g, 1, 0], key))
    for _ in range(1500):
        pairs.append(([int(v) for v in rng.integers(0, 2**32, 4, dtype=np.uint64)],
                      [int(v) for v in rng.integers(0, 2**32, 2, dtype=np.uint64)]))
    return pairs


def test_every_word_matches_independent_implementations(svo, engines):
    pairs = pairs_to_check()
    res = run_engines(engines, pairs)
    for kind, words in res.items():
        for (c, k), w in zip(pairs, words):
            assert svo.philox4x32_10(c, k) == w, (kind, c, k)


def test_the_engines_reproduce_the_published_answer(engines):
    # the outside implementations themselves give the standard's value
    (c0, c1, c2, c3, k0, k1, word, value), = read_kat()
    res = run_engines(engines, [([c0, c1, c2, c3], [k0, k1])])
    for kind, words in res.items():
        assert words[0][word] == value, kind
