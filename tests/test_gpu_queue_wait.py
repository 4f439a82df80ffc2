"""The fused kernel's waits are bounded.  A claim on a race slot that nothing
ever publishes, and the idle wait of a warp that never gets work, each give up
on their own time bound (about two seconds), report it and set the timeout bit
of the status word; the context stays usable, and a verify call in the fused
variant still matches the oracle afterwards.  No GPU fault is involved: the
waits simply run out."""
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
    lib = str(tmp_path_factory.mktemp("queue") / "libqueue.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INC,
                    os.path.join(HERE, "queue_probe.cu"), "-o", lib], check=True)
    L = ctypes.CDLL(lib)
    L.queue_probe.restype = ctypes.c_int
    L.queue_probe.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_uint),
                              ctypes.POINTER(ctypes.c_uint), ctypes.POINTER(ctypes.c_float)]
    return L


def _run(probe, fill, idle):
    status = ctypes.c_uint(0)
    result = (ctypes.c_uint * 2)()
    ms = ctypes.c_float(0.0)
    assert probe.queue_probe(fill, idle, ctypes.byref(status), result, ctypes.byref(ms)) == 0
    return status.value, list(result), ms.value


def test_waits_run_out_and_report(probe):
    status, result, ms = _run(probe, 0, 1)
    assert result[0] == 0                      # the claim gave up: no request
    assert result[1] > 10                      # the idle warp slept many turns, then gave up
    assert status == sv.SV_STATUS_TIMEOUT
    assert 1500.0 < ms < 30000.0               # bounded: about 2 s each
    # a filled slot returns at once, with no timeout
    status, result, ms = _run(probe, 1, 0)
    assert result[0] == 42 and status == 0 and ms < 1000.0
    # the context is still usable: a fused verify call matches the oracle
    w = wl.make("tiny", "cuda")
    s = compare(w, gpu_run(w, variant=sv.SV_VARIANT_FUSED), oracle_on(w))
    assert s["checked"] + s["exempt"] == 1
