"""The race's word filter is safe and sharp.  For a reference key K0, every
token whose exact key reaches K0 - 1e-6 (the near-tie band) must survive the
filter, and every survivor must satisfy the filter's inequality
    log2(o + 1/2) <= L(x) + 2,   L(x) = (z/T - lse_t - K0 + delta) log2(e) + 32,
so that it keeps no more than its documented rounding slack allows.  The
single-precision bound that screens survivors before their exact key must be
at least the exact key (in log2 units) for every candidate, and close to it.  Checked
on real rows for bonus and residual races, plain and saguaro, fp32 and bf16, T
of 1 and 0.7, peaked rows, masked tokens and logits with a large offset, and
for K0 at several depths of the key order."""
import ctypes
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from gpu_util import host_logits

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "speculative_decoding_verification_lse_b200", "csrc")
INC = os.path.join(os.path.dirname(HERE), "include")
LOG2E = 1.4426950408889634
BAND = 1e-5


@pytest.fixture(scope="module")
def probe(tmp_path_factory, sv):
    lib = str(tmp_path_factory.mktemp("filter") / "libfilter.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INC,
                    os.path.join(HERE, "race_filter_probe.cu"), "-o", lib], check=True)
    L = ctypes.CDLL(lib)
    L.race_filter_probe.restype = ctypes.c_int
    L.race_filter_probe.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_float,
        ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
        ctypes.c_double, ctypes.c_double, ctypes.c_ulonglong, ctypes.c_uint, ctypes.c_int,
        ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.POINTER(ctypes.c_float)]
    return L


def _as_f64(h):
    if h.dtype == np.float32:
        return h.astype(np.float64)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _run(probe, zt, zq, T, kind, K0, V):
    ht, hq = host_logits(zt), host_logits(zq)
    lse_t, lse_q = oracle.row_lse(ht, T), oracle.row_lse(hq, T)
    ntop, top, ln_c, ln_Z = 0, (ctypes.c_int * 8)(), math.log(0.5), 0.0
    if kind == "saguaro":
        zqf = _as_f64(hq)
        K = np.lexsort((np.arange(V), -np.nan_to_num(zqf, neginf=-1e300)))[:5]
        ntop = 5
        for i, x in enumerate(K):
            top[i] = int(x)
        ln_Z = math.log1p(-0.5 * float(np.sum(np.exp(zqf[K] / T - lse_q))))
    keep = torch.full((V,), 7, dtype=torch.uint8, device="cuda")
    words = torch.zeros((V,), dtype=torch.int32, device="cuda")
    exact = torch.full((V,), float("nan"), dtype=torch.float64, device="cuda")
    upper = torch.full((V,), float("nan"), dtype=torch.float32, device="cuda")
    cup = ctypes.c_float(0.0)
    rc = probe.race_filter_probe(zt.data_ptr(), zq.data_ptr(), V,
                                 0 if zt.dtype == torch.float32 else 1, T, lse_t, lse_q, ntop, top,
                                 ln_c, ln_Z, 12345, 3, 0 if kind == "bonus" else 1, K0,
                                 keep.data_ptr(), words.data_ptr(), exact.data_ptr(),
                                 upper.data_ptr(), ctypes.byref(cup))
    assert rc == 0
    return (keep.cpu().numpy(), words.cpu().numpy().view(np.uint32).astype(np.float64),
            exact.cpu().numpy(), lse_t, _as_f64(ht), cup.value, upper.cpu().numpy().astype(np.float64))


def _rows(dtype, offset):
    g = torch.Generator(device="cuda").manual_seed(7)
    V = 128256 + 5
    zt = torch.randn(V, generator=g, device="cuda") * 3 + offset
    zt[17] += 14.0                       # a peaked token
    zt[::97] = float("-inf")             # masked tokens
    zq = zt + torch.randn(V, generator=g, device="cuda")
    return zt.to(dtype).contiguous(), zq.to(dtype).contiguous(), V


@pytest.mark.parametrize("offset", [0.0, 3000.0])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T", [1.0, 0.7])
@pytest.mark.parametrize("kind", ["bonus", "residual", "saguaro"])
def test_word_filter_keeps_every_contender(probe, dtype, T, kind, offset):
    zt, zq, V = _rows(dtype, offset)
    T = float(np.float32(T))
    # K0 = -inf: every unmasked token survives, and the exact keys come back
    keep, o, e, lse_t, z, cup, ub = _run(probe, zt, zq, T, kind, float("-inf"), V)
    assert cup == float("inf")
    live = np.isfinite(z)
    assert np.all(keep[live] == 1)
    assert np.all(keep <= 1)
    # the survivor bound: never below the exact key; tight where the word is small
    # (it bounds E by W, and E / W -> 1 as W -> 0: the filter's survivors) and the
    # logits are of moderate size (its slack grows with |z|, and with a large offset
    # and bf16 rounding p and q' nearly coincide, where log2(1 - q'/p) is steep)
    cand = np.isfinite(e)
    slack = ub[cand] - e[cand] * LOG2E
    assert slack.min() >= 0.0, (slack.min(), int(np.flatnonzero(cand)[np.argmin(slack)]))
    if offset == 0.0:
        small = (o[cand] < 2.0 ** 24)
        assert small.sum() > 0
        assert np.median(slack[small]) < 0.01, np.median(slack[small])
    fin = np.sort(e[np.isfinite(e)])[::-1]
    assert fin.size >= 200  # bf16 with a large offset leaves few tokens with p > q
    for depth in (0, 1, 9, 99, fin.size // 2):
        K0 = float(fin[depth])
        keep, o2, e2, _, _, cup, _ = _run(probe, zt, zq, T, kind, K0, V)
        assert np.array_equal(o2, o) and np.array_equal(np.isnan(e2), np.isnan(e))
        assert math.isfinite(cup)
        # safe: every token within the near-tie band of K0 (or above it) is kept
        must = np.isfinite(e) & (e >= K0 - 1e-6)
        assert np.all(keep[must] == 1), np.flatnonzero(must & (keep == 0))[:5]
        # sharp: a kept token passes the inequality up to the filter's slack
        L = (z / T - lse_t - K0 + BAND) * LOG2E + 32.0
        kept = (keep == 1) & live
        assert np.all(np.log2(o[kept] + 0.5) <= L[kept] + 2.0)
        # and at K0 = the best key only a handful survive
        if depth == 0:
            assert kept.sum() <= 64, kept.sum()
