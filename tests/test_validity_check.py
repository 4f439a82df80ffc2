"""The near-tie validity check of the GPU parity tests (gpu_util.check_valid),
exercised on the CPU: every output the oracle itself produces passes it, and
outputs broken in the ways a wrong kernel could break them fail it."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_lse_b200 import workloads as wl


@pytest.fixture(scope="module")
def util():
    import gpu_util
    return gpu_util


def oracle_as_got(util, w, seed):
    ref = util.oracle_on(w, seed=seed, nthreads=4)
    got = {"tokens": ref["tokens"].copy(), "accept_len": ref["accept_len"].copy(),
           "flags": ref["flags"].astype(np.int64)}
    return ref, got


@pytest.mark.parametrize("name", ["b256", "ragged", "saguaro"])
def test_the_oracle_outputs_are_valid(util, name):
    w = wl.make(name, "cpu", B=12, V=3001)
    for seed in range(3):
        ref, got = oracle_as_got(util, w, seed)
        for b, m in enumerate(w.modes()):
            if m != wl.GREEDY and not (int(ref["flags"][b]) & 0xF00):
                util.check_valid(w, b, got, ref["row_lse"][b], seed)


def test_broken_outputs_are_rejected(util):
    w = wl.make("b256", "cpu", B=12, V=3001)
    ref, got = oracle_as_got(util, w, 0)
    b = 0
    n = int(got["accept_len"][b]) - 1
    broken = []
    # a token outside the vocabulary
    g = {k: v.copy() for k, v in got.items()}
    g["tokens"][b, n] = w.V
    broken.append(g)
    # a padding slot that is not -1
    if n < w.D_max:
        g = {k: v.copy() for k, v in got.items()}
        g["tokens"][b, n + 1] = 0
        broken.append(g)
    # one more accepted draft than the draws allow (the scan must stop at the rejection)
    rejected = [bb for bb in range(w.B) if int(got["accept_len"][bb]) - 1 < w.D_max]
    bb = rejected[0]
    nn = int(got["accept_len"][bb]) - 1
    g = {k: v.copy() for k, v in got.items()}
    g["accept_len"][bb] = nn + 2
    g["tokens"][bb, nn] = int(w.tokens[bb, nn])
    g["tokens"][bb, nn + 1] = 0
    broken.append((bb, g))
    # a residual token with p <= q
    zt = w.target[bb, nn].float().numpy()
    zq = w.draft[bb, nn].float().numpy()
    bad = int(np.argmax(zq - zt))
    g = {k: v.copy() for k, v in got.items()}
    g["tokens"][bb, nn] = bad
    broken.append((bb, g))
    for item in broken:
        bq, gq = item if isinstance(item, tuple) else (b, item)
        with pytest.raises(AssertionError):
            util.check_valid(w, bq, gq, ref["row_lse"][bq], 0)
