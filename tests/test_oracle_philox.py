"""Statistical pins for the oracle's counter-based generator.

The exact words are pinned on the CPU by test_oracle_philox_kat.py (the C++26
standard's known answer for philox4x32 and two independent host
implementations of the same published generator) and on the GPU against
cuRAND's Philox4_32_10 (test_gpu_philox_curand.py).  Here the generator is
also pinned by properties any correct 10-round Philox has and a broken one
loses: uniform words, uniform accept draws, unit-exponential race draws, full
avalanche on every input bit, and independence of neighbouring counters."""
import math

import numpy as np
import pytest
from scipy import stats


def words(svo, n, key=(0x1234ABCD, 0x0BADF00D), lane_stride=1):
    out = np.empty((n, 4), dtype=np.uint64)
    for i in range(n):
        out[i] = svo.philox4x32_10([i * lane_stride, 7, 0, 0], key)
    return out


def test_words_are_uniform_bytes(svo):
    w = words(svo, 20000)
    for lane in range(4):
        for shift in (0, 8, 16, 24):
            counts = np.bincount(((w[:, lane] >> shift) & 0xFF).astype(np.int64), minlength=256)
            assert stats.chisquare(counts).pvalue > 1e-4


def test_accept_uniform_is_uniform_on_24_bits(svo):
    u = np.array([svo.accept_uniform(99, g, d) for g in range(4000) for d in range(8)])
    assert np.all(u >= 0) and np.all(u < 1)
    # exactly representable as k * 2^-24
    assert np.all(np.floor(u * 2**24) == u * 2**24)
    counts = np.histogram(u, bins=64, range=(0, 1))[0]
    assert stats.chisquare(counts).pvalue > 1e-4
    assert stats.kstest(u, "uniform").pvalue > 1e-4


def test_race_draws_are_unit_exponential(svo):
    e = np.array([svo.race_exponential(5, g, x) for g in range(300) for x in range(100)])
    assert np.all(e > 0)
    assert stats.kstest(e, "expon").pvalue > 1e-4
    assert abs(e.mean() - 1.0) < 4 / math.sqrt(len(e))


def _popcount(a):
    return bin(a).count("1")


@pytest.mark.parametrize("which", ["ctr0", "ctr1", "ctr2", "ctr3", "key0", "key1"])
def test_full_avalanche_on_every_input_word(svo, which):
    # flipping one input bit flips each of the 128 output bits with probability
    # 1/2 after ten rounds: mean distance 64, sd 5.66 per trial
    rng = np.random.default_rng(abs(hash(which)) % 2**32)
    dists = []
    for t in range(400):
        ctr = [int(v) for v in rng.integers(0, 2**32, 4, dtype=np.uint64)]
        key = [int(v) for v in rng.integers(0, 2**32, 2, dtype=np.uint64)]
        bit = 1 << int(rng.integers(0, 32))
        a = svo.philox4x32_10(ctr, key)
        if which.startswith("ctr"):
            c2 = list(ctr)
            c2[int(which[-1])] ^= bit
            b = svo.philox4x32_10(c2, key)
        else:
            k2 = list(key)
            k2[int(which[-1])] ^= bit
            b = svo.philox4x32_10(ctr, k2)
        dists.append(sum(_popcount(x ^ y) for x, y in zip(a, b)))
    dists = np.array(dists, dtype=np.float64)
    assert abs(dists.mean() - 64.0) < 4 * 5.66 / math.sqrt(len(dists))
    assert dists.min() > 30


def test_neighbouring_counters_are_uncorrelated(svo):
    w = words(svo, 20000).astype(np.float64) / 2**32
    for lane in range(4):
        x = w[:, lane]
        r = np.corrcoef(x[:-1], x[1:])[0, 1]
        assert abs(r) < 4 / math.sqrt(len(x))
    r01 = np.corrcoef(w[:, 0], w[:, 1])[0, 1]
    assert abs(r01) < 4 / math.sqrt(len(w))


def test_streams_are_distinct_per_request_position_and_tag(svo):
    seen = set()
    for g in range(50):
        for d in range(20):
            seen.add(svo.accept_uniform(1, g, d))
    assert len(seen) > 990
    # the accept stream (tag 0) and the race stream (tag 1) differ for equal (g, .)
    e = svo.race_exponential(1, 3, 0)
    u = svo.accept_uniform(1, 3, 0)
    assert abs((1 - math.exp(-e)) - u) > 1e-6
