"""CUDA path versus the oracle, element by element, on the same seeded inputs.

Bar: accepted lengths and tokens bit-exact outside requests the oracle flags as
near-ties (|u - a| < 1e-5, or top-2 race keys within 1e-6); per-row LSE within
1e-5 relative for fp32 logits and 1e-3 for bf16.  Sizes span several 32 KiB
chunks and a ragged tail; the full-size workloads run in the configuration the
benchmark times, with the oracle on sampled requests."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl
from gpu_util import compare, gpu_run, oracle_on

pytestmark = pytest.mark.gpu

# every launch structure, the split one with each layout of the work after the statistics
VARIANTS = pytest.mark.parametrize(
    "variant",
    [sv.SV_VARIANT_SPLIT | sv.SV_TAIL_PER_REQUEST, sv.SV_VARIANT_SPLIT | sv.SV_TAIL_ITEMS,
     sv.SV_VARIANT_FUSED, sv.SV_VARIANT_CLUSTER],
    ids=["split-per-request", "split-items", "fused", "cluster"])


@VARIANTS
@pytest.mark.parametrize("mode", [0, 1, 2], ids=["stochastic", "greedy", "saguaro"])
def test_tiny_workload(sv, mode, variant):
    w = wl.make("tiny", "cuda", mode=mode)
    for seed in range(20):
        got = gpu_run(w, seed=seed, variant=variant)
        s = compare(w, got, oracle_on(w, seed=seed))
        assert s["checked"] + s["exempt"] == 1


@VARIANTS
@pytest.mark.parametrize("name", sorted(wl.CONFIGS))
# rows whose length in bytes is a multiple of 16 stream through the per-request
# tail's bulk-copy ring, the others through registers; 32776 bf16 ends in a
# segment of one 16-byte vector
@pytest.mark.parametrize("V", [40000 + 13, 16384 * 2 + 7, 40000 + 8, 16384 * 2 + 8])
def test_reduced_workloads(sv, name, V, variant):
    B = {"tiny": 3, "b32": 32, "b256": 24, "ragged": 24, "saguaro": 24}[name]
    w = wl.make(name, "cuda", B=B, V=V)
    s = compare(w, gpu_run(w, variant=variant), oracle_on(w))
    assert s["checked"] >= B - 1


@VARIANTS
@pytest.mark.parametrize("name,sample", [("b32", None), ("b256", 24), ("ragged", None),
                                          ("saguaro", 24)])
def test_full_size_workloads(sv, name, sample, variant):
    w = wl.make(name, "cuda")
    got = gpu_run(w, variant=variant)
    reqs = None
    if sample:
        rng = np.random.default_rng(5)
        reqs = sorted(set([0, w.B - 1] + list(rng.choice(w.B, sample, replace=False))))
    s = compare(w, got, oracle_on(w, reqs))
    n = len(reqs) if reqs else w.B
    assert s["checked"] >= n - 1
    print(name, s)


# (workload, seeds): about 2e5 stochastic requests in all, so that the bound
# 1e-4 allows about 20 of them
NEAR_TIE_POOL = [("b256", 400), ("saguaro", 400), ("b32", 800), ("ragged", 800)]
_POOL_CACHE = {}


@VARIANTS
def test_near_tie_rate_below_1e4(sv, variant):
    """Near-tie flags, counted per request against the stochastic requests
    verified (the strictest unit: a flagged request holds at least one near-tie
    row, so flagged rows / verified rows is lower still), pooled over four
    full-size workloads and many seeds; the bound is 0.01%."""
    flagged = total = 0
    for name, nseeds in NEAR_TIE_POOL:
        if name not in _POOL_CACHE:
            _POOL_CACHE.clear()
            _POOL_CACHE[name] = wl.make(name, "cuda")
        w = _POOL_CACHE[name]
        stoch = torch.tensor([m != sv.SV_GREEDY for m in w.modes()], device="cuda")
        acc = torch.zeros((), dtype=torch.int64, device="cuda")
        errs = torch.zeros((), dtype=torch.int64, device="cuda")
        out = None
        for seed in range(nseeds):
            out = sv.verify_workload(w, seed=seed, variant=variant, out=out)
            acc += (((out["flags"] & sv.SV_FLAG_NEAR_TIE) != 0) & stoch).sum()
            errs += ((out["flags"] & sv.SV_FLAG_ERRORS) != 0).sum()
        torch.cuda.synchronize()
        assert int(errs) == 0, name
        flagged += int(acc)
        total += int(stoch.sum()) * nseeds
    print(f"near-tie requests: {flagged} of {total} stochastic requests")
    assert total >= 200_000
    assert flagged <= 1e-4 * total, (flagged, total)


def test_full_size_is_deterministic_and_variants_agree(sv):
    # every launch structure and tail layout gives bit-identical outputs, run after run
    w = wl.make("b256", "cuda")
    runs = [gpu_run(w, seed=3, variant=v)
            for v in (sv.SV_VARIANT_SPLIT, sv.SV_VARIANT_SPLIT, sv.SV_VARIANT_FUSED,
                      sv.SV_VARIANT_FUSED, sv.SV_VARIANT_SPLIT | sv.SV_TAIL_ITEMS,
                      sv.SV_VARIANT_CLUSTER, sv.SV_VARIANT_CLUSTER, sv.SV_VARIANT_AUTO)]
    for r in runs[1:]:
        for k in runs[0]:
            assert np.array_equal(runs[0][k], r[k], equal_nan=True), k


def test_accept_length_mean_is_plausible(sv):
    # not a parity test: the draft noise sets acceptance; AL stays in range and
    # the bonus/residual slot is always a valid token
    w = wl.make("b256", "cuda")
    got = gpu_run(w)
    AL = got["accept_len"]
    assert AL.min() >= 1 and AL.max() <= 8
    n = AL - 1
    assert np.all(got["tokens"][np.arange(w.B), n] >= 0)
    assert np.all(got["tokens"][np.arange(w.B), n] < w.V)
