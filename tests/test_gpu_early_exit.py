"""The early-exit schedule (SV_VARIANT_EARLY_EXIT): the rows read position by
position, in rounds, only for the requests that accepted every earlier draft.
Against the oracle element by element (rows past a request's outcome may be
unread, so they may have no LSE), against the split path bit for bit on
tokens, accepted lengths and flags, and the rows it reads checked against the
round rule."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl
from gpu_util import compare, gpu_run, oracle_on

pytestmark = pytest.mark.gpu

EE = sv.SV_VARIANT_EARLY_EXIT


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["stochastic", "greedy", "saguaro"])
def test_tiny(sv, mode):
    w = wl.make("tiny", "cuda", mode=mode)
    for seed in range(20):
        s = compare(w, gpu_run(w, seed=seed, variant=EE), oracle_on(w, seed=seed), early_exit=True)
        assert s["checked"] + s["exempt"] == 1


@pytest.mark.parametrize("name", sorted(wl.CONFIGS))
@pytest.mark.parametrize("V", [40000 + 13, 40000 + 8])
def test_reduced_workloads(sv, name, V):
    B = {"tiny": 3, "b32": 32, "b256": 24, "ragged": 24, "saguaro": 24}[name]
    w = wl.make(name, "cuda", B=B, V=V)
    for seed in (0, 1):
        s = compare(w, gpu_run(w, seed=seed, variant=EE), oracle_on(w, seed=seed), early_exit=True)
        assert s["checked"] >= B - 1


@pytest.mark.parametrize("name,sample", [("b32", None), ("b256", 24), ("ragged", None),
                                          ("saguaro", 24)])
def test_full_size_workloads(sv, name, sample):
    w = wl.make(name, "cuda")
    got = gpu_run(w, variant=EE)
    reqs = None
    if sample:
        rng = np.random.default_rng(5)
        reqs = sorted(set([0, w.B - 1] + list(rng.choice(w.B, sample, replace=False))))
    s = compare(w, got, oracle_on(w, reqs), early_exit=True)
    n = len(reqs) if reqs else w.B
    assert s["checked"] >= n - 1


@pytest.mark.parametrize("name", ["b32", "b256", "ragged", "saguaro", "tiny"])
def test_same_outcomes_as_the_split_path(sv, name):
    # the rounds compute the same statistics and the same decisions: tokens,
    # accepted lengths and flags are identical, call for call
    w = wl.make(name, "cuda")
    for seed in range(3):
        a = gpu_run(w, seed=seed, variant=sv.SV_VARIANT_SPLIT)
        b = gpu_run(w, seed=seed, variant=EE)
        for k in ("tokens", "accept_len", "flags"):
            assert np.array_equal(a[k], b[k]), (name, seed, k)
        # the LSEs it reports are the split path's, for exactly the rows of the
        # positions up to each request's outcome n
        rows_D, modes = w.row_D_list(), w.modes()
        for r in range(w.B):
            n = int(b["accept_len"][r]) - 1
            Db, m = rows_D[r], modes[r]
            for slot in range(2 * w.D_max + 1):
                d = slot if slot <= w.D_max else slot - w.D_max - 1
                draft = slot > w.D_max
                read = m != 1 and d <= n and (d < Db if draft else d <= Db)
                got_lse = b["row_lse"][r, slot]
                if read:
                    assert got_lse == a["row_lse"][r, slot], (name, r, slot)
                else:
                    assert np.isnan(got_lse), (name, r, slot)


@pytest.mark.parametrize("D", [0, 1, 2, 3, 5])
@pytest.mark.parametrize("mode", [0, 1, 2], ids=["stochastic", "greedy", "saguaro"])
def test_every_round_boundary(sv, D, mode):
    # D_max = 0 .. 5 cover one, two and three rounds and the edges between them
    w = wl.make("b256", "cuda", B=40, D=D, V=9001, mode=mode)
    for seed in range(3):
        got = gpu_run(w, seed=seed, variant=EE)
        compare(w, got, oracle_on(w, seed=seed), early_exit=True)
        ref = gpu_run(w, seed=seed, variant=sv.SV_VARIANT_SPLIT)
        for k in ("tokens", "accept_len", "flags"):
            assert np.array_equal(got[k], ref[k]), (D, mode, seed, k)


def test_bad_tokens_and_ragged_lengths(sv):
    sv.sv_get_device_status()
    w = wl.make("ragged", "cuda", B=48, V=7001)
    tok = w.tokens.clone()
    tok[3, 0] = w.V + 5   # out of range at position 0
    tok[7, 2] = -3        # out of range at position 2
    w.tokens = tok
    got = gpu_run(w, variant=EE)
    ref = gpu_run(w, variant=sv.SV_VARIANT_SPLIT)
    for k in ("tokens", "accept_len", "flags"):
        assert np.array_equal(got[k], ref[k]), k
    assert got["accept_len"][3] == -1 and got["accept_len"][7] == -1
    assert (got["flags"][3] & sv.SV_FLAG_BAD_TOKEN) and (got["flags"][7] & sv.SV_FLAG_BAD_TOKEN)
    assert sv.sv_get_device_status() & sv.SV_FLAG_BAD_TOKEN  # reading it clears it
