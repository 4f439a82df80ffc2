"""Vocabulary-parallel verification (sv_shard_stats / sv_shard_race /
sv_shard_finish) on one device, every shard in turn with concatenation in
place of the all-gathers: every shard writes the same outputs, and they match
the oracle on the whole rows (bit-exact accepted lengths and tokens outside
flagged near-ties, row LSEs within the tolerance) and the unsharded call."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl
from speculative_decoding_verification_lse_b200.sharding import (
    verify_vocab_parallel_in_one_process, vocab_shard, vocab_shard_width)
from gpu_util import compare, gpu_run, oracle_on

pytestmark = pytest.mark.gpu


def run_sharded(w, n, seed=None, draft_top=False):
    outs = verify_vocab_parallel_in_one_process(
        w.target, w.draft, w.tokens, w.row_D, n_shards=n, temperature=w.temperature, mode=w.mode,
        seed=w.seed if seed is None else seed, temperature_per_req=w.temperature_per_req,
        mode_per_req=w.mode_per_req, saguaro_k=w.saguaro_k, saguaro_c=w.saguaro_c, row_lse=True,
        draft_top=draft_top)
    torch.cuda.synchronize()
    return [{k: v.cpu().numpy() for k, v in o.items()} for o in outs]


def test_shards_cover_the_vocabulary(sv):
    t = torch.randn((2, 3, 1001), device="cuda")
    for n in (1, 2, 3, 7):
        Vl = vocab_shard_width(1001, n)
        assert Vl % 4 == 0 and n * Vl >= 1001
        cat = torch.cat([vocab_shard(t, r, n) for r in range(n)], dim=-1)
        assert torch.equal(cat[..., :1001], t)
        assert torch.isinf(cat[..., 1001:]).all()


@pytest.mark.parametrize("n", [2, 3, 5])
@pytest.mark.parametrize("name", ["tiny", "b32", "ragged", "saguaro"])
def test_sharded_matches_the_oracle(sv, name, n):
    B = {"tiny": 1, "b32": 16, "ragged": 16, "saguaro": 16}[name]
    V = None if name == "tiny" else 40013
    w = wl.make(name, "cuda", B=B, V=V)
    for seed in (0, 1, 2):
        outs = run_sharded(w, n, seed=seed)
        for o in outs[1:]:
            for k in outs[0]:
                assert np.array_equal(outs[0][k], o[k], equal_nan=True), k
        ref = oracle_on(w, seed=seed)
        s = compare(w, outs[0], ref)
        assert s["checked"] >= B - 1
        # the unsharded call agrees on every request the oracle does not flag
        flat = gpu_run(w, seed=seed)
        clean = (ref["flags"] & oracle.FLAG_NEAR_TIE) == 0
        np.testing.assert_array_equal(outs[0]["tokens"][clean], flat["tokens"][clean])
        np.testing.assert_array_equal(outs[0]["accept_len"][clean], flat["accept_len"][clean])


def test_sharded_draft_top_lists(sv):
    w = wl.make("saguaro", "cuda", B=12, V=40013)
    outs = run_sharded(w, 4, draft_top=True)
    flat = sv.verify_workload(w, draft_top=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(outs[0]["draft_top"], flat["draft_top"].cpu().numpy())


def test_full_size_eight_shards(sv):
    w = wl.make("b256", "cuda")
    outs = run_sharded(w, 8)
    rng = np.random.default_rng(3)
    reqs = sorted(set([0, w.B - 1] + list(rng.choice(w.B, 16, replace=False))))
    ref = oracle_on(w, reqs)
    s = compare(w, outs[7], ref)
    assert s["checked"] >= len(reqs) - 1
    flat = gpu_run(w)
    same = np.mean(np.all(outs[0]["tokens"] == flat["tokens"], axis=1))
    assert same >= 0.99
    assert sv.sv_get_device_status() & sv.SV_FLAG_ERRORS == 0


def test_sharded_seed_read_from_device_memory(sv):
    # the seed in device memory (sv_params.seed_device) reaches every stage
    w = wl.make("b32", "cuda", B=8, V=20011)
    sdev = torch.tensor([77], dtype=torch.int64, device="cuda")
    got = verify_vocab_parallel_in_one_process(
        w.target, w.draft, w.tokens, w.row_D, n_shards=3, temperature=w.temperature,
        mode=w.mode, seed=5, seed_device=sdev)
    ref = verify_vocab_parallel_in_one_process(
        w.target, w.draft, w.tokens, w.row_D, n_shards=3, temperature=w.temperature,
        mode=w.mode, seed=77)
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        for k in ("tokens", "accept_len", "flags"):
            assert torch.equal(g[k], r[k]), k
