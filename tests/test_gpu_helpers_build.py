"""The CUDA helpers that the GPU tests compile on the fly (the cuRAND Philox
probe, the race word-filter probe and the work-queue wait probe, which include the
library's device headers)
must keep compiling for sm_100a; nvcc works without a GPU, so this runs here."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "speculative_decoding_verification_lse_b200", "csrc")
INC = os.path.join(ROOT, "include")


@pytest.mark.parametrize("src", ["curand_philox_probe.cu", "race_filter_probe.cu",
                                 "queue_probe.cu"])
def test_gpu_test_helper_compiles(tmp_path, src):
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-I", CSRC, "-I", INC,
                    os.path.join(HERE, src), "-o", str(tmp_path / "lib.so")], check=True)
