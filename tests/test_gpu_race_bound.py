"""The race's filter is safe: on real rows, every token's single-precision key
bound (log2 units) is at least its exact double-precision key, so no token
that could win or tie is ever skipped.  Checked for bonus and residual races,
plain and saguaro, fp32 and bf16, peaked rows and masked tokens."""
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


@pytest.fixture(scope="module")
def probe(tmp_path_factory, sv):
    lib = str(tmp_path_factory.mktemp("bound") / "libbound.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INC,
                    os.path.join(HERE, "race_bound_probe.cu"), "-o", lib], check=True)
    L = ctypes.CDLL(lib)
    L.race_bound_probe.restype = ctypes.c_int
    L.race_bound_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_float, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                   ctypes.POINTER(ctypes.c_int), ctypes.c_double, ctypes.c_double,
                                   ctypes.c_ulonglong, ctypes.c_uint, ctypes.c_int,
                                   ctypes.c_void_p, ctypes.c_void_p]
    return L


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T", [1.0, 0.7])
@pytest.mark.parametrize("kind", ["bonus", "residual", "saguaro"])
def test_bound_dominates_exact_key(probe, dtype, T, kind):
    g = torch.Generator(device="cuda").manual_seed(7)
    V = 128256 + 5
    zt = torch.randn(V, generator=g, device="cuda") * 3
    zt[17] += 14.0                       # a peaked token
    zt[::97] = float("-inf")             # masked tokens
    zq = zt + torch.randn(V, generator=g, device="cuda")
    zt, zq = zt.to(dtype).contiguous(), zq.to(dtype).contiguous()
    ht, hq = host_logits(zt), host_logits(zq)
    Tf = float(np.float32(T))
    lse_t, lse_q = oracle.row_lse(ht, Tf), oracle.row_lse(hq, Tf)
    ntop, top, ln_c, ln_Z = 0, (ctypes.c_int * 8)(), math.log(0.5), 0.0
    if kind == "saguaro":
        zqf = hq.astype(np.float64) if hq.dtype == np.float32 else \
            (hq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        K = np.lexsort((np.arange(V), -np.nan_to_num(zqf, neginf=-1e300)))[:5]
        ntop = 5
        for i, x in enumerate(K):
            top[i] = int(x)
        mass = float(np.sum(np.exp(zqf[K] / Tf - lse_q)))
        ln_Z = math.log1p(-0.5 * mass)
    bounds = torch.full((V,), float("nan"), device="cuda")
    exact = torch.full((V,), float("nan"), dtype=torch.float64, device="cuda")
    rc = probe.race_bound_probe(zt.data_ptr(), zq.data_ptr(), V, 0 if dtype == torch.float32 else 1,
                                Tf, lse_t, lse_q, ntop, top, ln_c, ln_Z, 12345, 3,
                                0 if kind == "bonus" else 1, bounds.data_ptr(), exact.data_ptr())
    assert rc == 0
    b = bounds.cpu().numpy().astype(np.float64)
    e = exact.cpu().numpy()
    # a masked token gets a NaN or -inf bound (never selected) and no exact key
    masked = np.isneginf(zt.float().cpu().numpy())
    assert np.all(np.isnan(b[masked]) | np.isneginf(b[masked]))
    visited = ~np.isnan(b)
    cand = visited & np.isfinite(e)
    assert cand.sum() > V // 4
    e2 = e[cand] * 1.4426950408889634
    slack = b[cand] - e2
    assert slack.min() >= 0.0, (slack.min(), int(np.argmin(slack)))
    # and the bound is tight enough to filter: small slack for most tokens
    assert np.median(slack) < 1e-3, np.median(slack)
    # a token with no exact key (not a candidate) may have any bound; a candidate
    # never has a -inf bound
    assert np.all(np.isfinite(b[cand]))
