"""Pin of the oracle's Philox4x32-10 against NVIDIA cuRAND's Philox4_32_10.

The pages print no known-answer vector for Philox, so the oracle's generator is
checked word for word against an independent implementation of the same
published algorithm (Salmon et al., SC'11): cuRAND, run on the GPU.  With key
(seed mod 2^32, seed >> 32), cuRAND's block at `offset / 4` of subsequence s is
the Philox of the 128-bit counter (offset / 4 as the low 64 bits, s as the high
64 bits)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe(tmp_path_factory, sv):
    lib = str(tmp_path_factory.mktemp("curand") / "libprobe.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                    "-Xcompiler", "-fPIC", os.path.join(HERE, "curand_philox_probe.cu"),
                    "-o", lib], check=True)
    L = ctypes.CDLL(lib)
    L.curand_philox_words.restype = ctypes.c_int
    return L


def test_oracle_philox_equals_curand(probe):
    rng = np.random.default_rng(2024)
    n = 4096
    seeds = rng.integers(0, 2**64, n, dtype=np.uint64)
    seeds[:4] = [0, 1, 2**32, 2**64 - 1]
    subseq = rng.integers(0, 2**64, n, dtype=np.uint64)
    subseq[:8] = 0
    blocks = rng.integers(0, 2**62, n, dtype=np.uint64)
    blocks[:16] = np.arange(16)
    offsets = (blocks * np.uint64(4)).astype(np.uint64)
    words = np.zeros((n, 4), dtype=np.uint32)
    u64p = ctypes.POINTER(ctypes.c_ulonglong)
    rc = probe.curand_philox_words(seeds.ctypes.data_as(u64p), subseq.ctypes.data_as(u64p),
                                   offsets.ctypes.data_as(u64p),
                                   words.ctypes.data_as(ctypes.POINTER(ctypes.c_uint)), n)
    assert rc == 0
    for i in range(n):
        s, q, c = int(seeds[i]), int(subseq[i]), int(blocks[i])
        ctr = [c & 0xFFFFFFFF, c >> 32, q & 0xFFFFFFFF, q >> 32]
        key = [s & 0xFFFFFFFF, s >> 32]
        assert oracle.philox4x32_10(ctr, key) == [int(w) for w in words[i]], i


def test_accept_and_race_streams_match_curand_positions(probe):
    # u_d is word 0 at counter (d, g, 0, 0): cuRAND block d + g*2^32 of subsequence 0
    # (g < 2^30 keeps the byte offset 4 * block below 2^64);
    # the race word of token x is at counter (x/4, g, 1, 0): subsequence 1
    seed = 0x0123456789ABCDEF
    cases = [(d, g, 0) for d in range(8) for g in (0, 1, 77, 2**29)] + \
            [(x // 4, g, 1) for x in range(0, 64, 4) for g in (0, 5)]
    n = len(cases)
    seeds = np.full(n, seed, dtype=np.uint64)
    subseq = np.array([s for (_, _, s) in cases], dtype=np.uint64)
    offsets = np.array([4 * (c + (g << 32)) for (c, g, _) in cases], dtype=np.uint64)
    words = np.zeros((n, 4), dtype=np.uint32)
    u64p = ctypes.POINTER(ctypes.c_ulonglong)
    assert probe.curand_philox_words(seeds.ctypes.data_as(u64p), subseq.ctypes.data_as(u64p),
                                     offsets.ctypes.data_as(u64p),
                                     words.ctypes.data_as(ctypes.POINTER(ctypes.c_uint)), n) == 0
    for i, (c, g, s) in enumerate(cases):
        if s == 0:
            assert oracle.accept_uniform(seed, g, c) == (int(words[i][0]) >> 8) * 2.0**-24
        else:
            for lane in range(4):
                W = (int(words[i][lane]) + 0.5) * 2.0**-32
                e = oracle.race_exponential(seed, g, 4 * c + lane)
                assert abs(e - (-np.log1p(-W))) <= 4e-16 * e  # same word (libm rounding aside)
