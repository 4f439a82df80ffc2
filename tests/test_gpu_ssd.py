"""Speculative speculative decoding on the device against the oracle: the
outcome lookup (sv_ssd_lookup) element by element, the draft top lists the
verification returns for saguaro requests (sv_params.out_draft_top, the keys
of the speculation cache) index by index, and the whole cache round trip --
keys from the top lists, lookup of the verified outcome -- on the saguaro
workload."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl
from gpu_util import host_logits, oracle_on

pytestmark = pytest.mark.gpu

VARIANTS = pytest.mark.parametrize(
    "variant", [sv.SV_VARIANT_SPLIT | sv.SV_TAIL_PER_REQUEST, sv.SV_VARIANT_SPLIT | sv.SV_TAIL_ITEMS,
                sv.SV_VARIANT_FUSED, sv.SV_VARIANT_CLUSTER],
    ids=["split-per-request", "split-items", "fused", "cluster"])


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("B,D,K,S", [(1, 0, 0, 0), (50, 4, 20, 4), (300, 7, 45, 8), (40, 32, 100, 33)])
def test_lookup_matches_the_oracle(sv, B, D, K, S):
    rng = np.random.default_rng(B + K)
    out = rng.integers(0, 30, (B, D + 1)).astype(np.int32)
    AL = rng.integers(-1, D + 3, B).astype(np.int32)
    keys_al = rng.integers(1, D + 2, (B, K)).astype(np.int32)
    keys_tok = rng.integers(0, 30, (B, K)).astype(np.int32)
    spec = rng.integers(0, 1000, (B, K, S)).astype(np.int32)
    ref = oracle.ssd_lookup(out, AL, keys_al, keys_tok, spec)
    hit = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    osp = torch.full((B, S), -7, dtype=torch.int32, device="cuda")
    rc = sv.sv_ssd_lookup(dev(out), dev(AL), B, D, dev(keys_al), dev(keys_tok), K, dev(spec), S, hit,
                          osp if S else None)
    assert rc == sv.SV_OK, sv.sv_last_error()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(hit.cpu().numpy(), ref["hit"])
    if S:
        np.testing.assert_array_equal(osp.cpu().numpy(), ref["spec"])


@VARIANTS
def test_draft_top_lists_match_the_oracle(sv, variant):
    w = wl.make("saguaro", "cuda", B=24, V=40013)
    got = sv.verify_workload(w, variant=variant, draft_top=True)
    torch.cuda.synchronize()
    top = got["draft_top"].cpu().numpy()
    draft = host_logits(w.draft)
    k = min(w.saguaro_k, w.V)
    for b in range(w.B):
        for d in range(w.D_max):
            np.testing.assert_array_equal(top[b, d], oracle.row_topk(draft[b, d], k))
    # non-saguaro requests and rows beyond D_b get -1
    r = wl.make("ragged", "cuda", B=16, V=20011)
    got = sv.verify_workload(r, variant=variant, draft_top=True)
    torch.cuda.synchronize()
    assert np.all(got["draft_top"].cpu().numpy() == -1)


def test_speculation_cache_round_trip(sv):
    """Keys (d + 1, each of the draft's top-5 at position d) for every d < D,
    looked up with the verified outcome: the hits equal the oracle's lookup on
    the oracle's own outputs (requests the oracle flags as near-ties aside)."""
    w = wl.make("saguaro", "cuda")
    B, D = w.B, w.D_max
    got = sv.verify_workload(w, draft_top=True)
    k = got["draft_top"].shape[2]
    keys_tok = got["draft_top"].reshape(B, D * k).contiguous()
    keys_al = (torch.arange(D, device="cuda", dtype=torch.int32) + 1).repeat_interleave(k)
    keys_al = keys_al[None].repeat(B, 1).contiguous()
    hit = torch.empty(B, dtype=torch.int32, device="cuda")
    assert sv.sv_ssd_lookup(got["tokens"], got["accept_len"], B, D, keys_al, keys_tok, D * k,
                            None, 0, hit) == sv.SV_OK
    torch.cuda.synchronize()
    ref = oracle_on(w)
    draft = host_logits(w.draft)
    ref_keys = np.stack([np.concatenate([oracle.row_topk(draft[b, d], k) for d in range(D)])
                         for b in range(B)]).astype(np.int32)
    ref_hit = oracle.ssd_lookup(ref["tokens"], ref["accept_len"], keys_al.cpu().numpy(), ref_keys)["hit"]
    clean = (ref["flags"] & oracle.FLAG_NEAR_TIE) == 0
    np.testing.assert_array_equal(hit.cpu().numpy()[clean], ref_hit[clean])
    rate = float(np.mean(hit.cpu().numpy() >= 0))
    print(f"speculation cache hit rate (saguaro, top-{k} keys): {rate:.3f}")
    assert 0.0 < rate < 1.0
