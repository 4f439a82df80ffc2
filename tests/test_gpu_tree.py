"""Tree (multi-candidate) verification on the device (sv_verify_tree) against
the oracle (svo_verify_tree), element by element: accepted lengths, tokens
and accepted nodes bit-exact outside requests the oracle flags as near-ties;
a chain tree against the library's own linear path bit for bit; greedy trees;
errors; rows of leaves never read."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl
from gpu_util import gpu_run, host_logits

pytestmark = pytest.mark.gpu


def tree_gpu(w, seed=0, **kw):
    out = sv.verify_tree(w.target, w.draft, w.tokens, w.parents, temperature=w.temperature,
                         mode=w.mode, seed=seed, **kw)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def tree_oracle(w, seed=0):
    return oracle.verify_tree(host_logits(w.target), host_logits(w.draft), w.tokens.cpu().numpy(),
                              w.parents.cpu().numpy(), temperature=w.temperature, mode=w.mode,
                              seed=seed, nthreads=8)


def compare_tree(got, ref, min_checked):
    clean = (ref["flags"] & oracle.FLAG_NEAR_TIE) == 0
    assert clean.sum() >= min_checked
    errs = (ref["flags"] & oracle.FLAG_ERRORS).astype(np.int64)
    np.testing.assert_array_equal(got["flags"] & sv.SV_FLAG_ERRORS, errs)
    for k in ("tokens", "accept_len", "nodes"):
        np.testing.assert_array_equal(got[k][clean], ref[k][clean], err_msg=k)
    return int(clean.sum())


@pytest.mark.parametrize("branching", [(3, 2, 2), (4,), (1, 1, 1, 1), (2, 3, 1)])
@pytest.mark.parametrize("mode", [sv.SV_STOCHASTIC, sv.SV_GREEDY], ids=["stochastic", "greedy"])
def test_tree_matches_the_oracle(sv, branching, mode):
    w = wl.make_tree("tree", "cuda", B=24, V=20011, branching=branching, mode=mode)
    for seed in range(4):
        compare_tree(tree_gpu(w, seed), tree_oracle(w, seed), 22)


@pytest.mark.parametrize("B", [30, 100, 160])
def test_tree_every_cluster_size(sv, B):
    # the walk spreads a request over a cluster of 4, 2 or 1 CTAs, as many as
    # fit two CTAs per multiprocessor (on 148 of them: 4 for B=30, 2 for B=100,
    # 1 for B=160); the outputs are the oracle's whatever the size
    w = wl.make_tree("tree", "cuda", B=B, V=5003, branching=(3, 2, 2))
    for seed in range(2):
        compare_tree(tree_gpu(w, seed), tree_oracle(w, seed), B - 2)


def test_chain_tree_is_the_linear_path(sv):
    for name in ("b32", "b256", "tiny"):
        w = wl.make(name, "cuda", B=None if name == "tiny" else 16, V=None if name == "tiny" else 30011)
        chain = torch.arange(w.D_max, dtype=torch.int32, device="cuda").repeat(w.B, 1).contiguous()
        for seed in range(3):
            lin = gpu_run(w, seed=seed)
            tr = sv.verify_tree(w.target, w.draft, w.tokens, chain, temperature=w.temperature,
                                mode=w.mode, seed=seed, row_lse=True)
            torch.cuda.synchronize()
            for k in ("tokens", "accept_len", "flags", "row_lse"):
                np.testing.assert_array_equal(lin[k], tr[k].cpu().numpy(), err_msg=(name, k))


def test_tree_full_size_sample(sv):
    w = wl.make_tree("tree", "cuda")
    got = tree_gpu(w, 5)
    rng = np.random.default_rng(1)
    reqs = sorted(rng.choice(w.B, 12, replace=False))
    sub = wl.TreeWorkload(name=w.name, target=w.target[reqs], draft=w.draft[reqs],
                          tokens=w.tokens[reqs], parents=w.parents[reqs],
                          temperature=w.temperature, mode=w.mode, dtype=w.dtype)
    ref = tree_oracle(sub, 5)
    # request offsets: the oracle ran request j as global index j; rerun on the device alike
    got_sub = tree_gpu(sub, 5)
    compare_tree(got_sub, ref, 11)
    assert np.all(got["accept_len"] >= 1) and np.all(got["accept_len"] <= 4)
    assert sv.sv_get_device_status() & sv.SV_FLAG_ERRORS == 0


def test_tree_errors_and_unread_rows(sv):
    w = wl.make_tree("tree", "cuda", B=6, V=5003, branching=(2, 2))
    tok, par = w.tokens.clone(), w.parents.clone()
    par[0, 3] = 5          # a parent after its node
    tok[1, 0] = w.V        # a token out of range
    draft = w.draft.clone()
    # positions 3..6 (nodes 2..5) are leaves: their draft rows are never read
    draft[2, 3:] = float("nan")
    draft[3, 1] = float("nan")  # position 1 has candidates: read, so an error
    out = sv.verify_tree(w.target, draft, tok, par, seed=3)
    torch.cuda.synchronize()
    f = out["flags"].cpu().numpy()
    al = out["accept_len"].cpu().numpy()
    assert f[0] & sv.SV_FLAG_BAD_PARAM and al[0] == -1
    assert f[1] & sv.SV_FLAG_BAD_TOKEN and al[1] == -1
    assert f[2] & sv.SV_FLAG_ERRORS == 0 and al[2] >= 1
    assert f[3] & sv.SV_FLAG_NONFINITE and al[3] == -1
    status = sv.sv_get_device_status()
    assert status & sv.SV_STATUS_BAD_PARAM and status & sv.SV_STATUS_BAD_TOKEN
