"""Small helpers shared by the tests (no verification arithmetic here beyond
the textbook softmax used to state expected laws)."""
import numpy as np


def bf16_bits(x):
    """float32 array -> bf16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    b = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_to_f32(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def softmax(z, T=1.0):
    z = np.asarray(z, dtype=np.float64) / T
    m = np.max(z, axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


def sample_categorical(rng, probs, n):
    """n draws from one categorical distribution (inverse CDF)."""
    c = np.cumsum(probs)
    c[-1] = 1.0
    return np.searchsorted(c, rng.random(n), side="right").astype(np.int32)


def sample_rows(rng, probs):
    """one draw per row of probs[..., V] (inverse CDF)."""
    c = np.cumsum(probs, axis=-1)
    c[..., -1] = 1.0
    u = rng.random(probs.shape[:-1] + (1,))
    return (c < u).sum(axis=-1).astype(np.int32)


def within_sigma(counts, probs, k=3.0):
    """per-cell |count/N - p| <= k * sqrt(p (1 - p) / N)"""
    counts = np.asarray(counts, dtype=np.float64)
    N = counts.sum()
    f = counts / N
    sd = np.sqrt(np.maximum(probs * (1 - probs), 1e-300) / N)
    return np.all(np.abs(f - probs) <= k * sd + 1e-15), np.max(np.abs(f - probs) / sd)


def chi2_pvalue(counts, probs):
    from scipy.stats import chisquare
    counts = np.asarray(counts, dtype=np.float64)
    N = counts.sum()
    exp = np.asarray(probs, dtype=np.float64) * N
    keep = exp > 0
    assert counts[~keep].sum() == 0, "mass on a cell of probability zero"
    return chisquare(counts[keep], exp[keep] * counts[keep].sum() / exp[keep].sum()).pvalue
