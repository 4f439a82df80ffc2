"""The fused kernel's grid barrier waits a bounded time.  In a cooperative launch
of two CTAs where the second never arrives (a count that nothing completes),
the first gives up after its bounded poll, reports it, and sets the timeout bit
of the status word; the context stays usable, and a launch where both arrive
passes.  No GPU fault is involved: the wait simply runs out."""
import ctypes
import os
import subprocess

import pytest

import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl
from gpu_util import compare, gpu_run, oracle_on

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "speculative_decoding_verification_lse_b200", "csrc")
INC = os.path.join(os.path.dirname(HERE), "include")


@pytest.fixture(scope="module")
def probe(tmp_path_factory, sv):
    lib = str(tmp_path_factory.mktemp("barrier") / "libbarrier.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INC,
                    os.path.join(HERE, "barrier_probe.cu"), "-o", lib], check=True)
    L = ctypes.CDLL(lib)
    L.barrier_probe.restype = ctypes.c_int
    L.barrier_probe.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_uint),
                                ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float)]
    return L


def _run(probe, skip):
    status = ctypes.c_uint(0)
    result = (ctypes.c_int * 2)()
    ms = ctypes.c_float(0.0)
    assert probe.barrier_probe(skip, ctypes.byref(status), result, ctypes.byref(ms)) == 0
    return status.value, list(result), ms.value


def test_barrier_wait_runs_out_and_reports(probe):
    status, result, ms = _run(probe, 1)
    assert result == [0, -1]                  # the first CTA gave up; the second never came
    assert status == sv.SV_STATUS_TIMEOUT
    assert 1.0 < ms < 30000.0                 # bounded: 2^22 polls with a short sleep
    # the context is still usable: a full barrier passes, and so does a verify call
    status, result, _ = _run(probe, 0)
    assert result == [1, 1] and status == 0
    w = wl.make("tiny", "cuda")
    s = compare(w, gpu_run(w, variant=sv.SV_VARIANT_FUSED), oracle_on(w))
    assert s["checked"] + s["exempt"] == 1
