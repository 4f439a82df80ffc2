"""CUDA path versus the oracle on edge cases: tiny and ragged V, unaligned rows,
D_max 0 and 32, D_b = 0, masked tokens, identical target and draft, invalid
device inputs (reported through flags and the status word, no trap), request
offsets, explicit workspaces and streams (the statistical law of the output over
10^6 requests: test_zz_marginals_1e6.py)."""

import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_lse_b200 as sv
from gpu_util import compare, gpu_run, host_logits, oracle_on
from speculative_decoding_verification_lse_b200 import workloads as wl

pytestmark = pytest.mark.gpu

# every launch structure, the split one with each layout of the work after the statistics
VARIANTS = pytest.mark.parametrize(
    "variant",
    [sv.SV_VARIANT_SPLIT | sv.SV_TAIL_PER_REQUEST, sv.SV_VARIANT_SPLIT | sv.SV_TAIL_ITEMS,
     sv.SV_VARIANT_FUSED, sv.SV_VARIANT_CLUSTER],
    ids=["split-per-request", "split-items", "fused", "cluster"])


def make_random(B, D, V, dtype=sv.SV_BF16, seed=0, draft_sd=1.0, T=1.0, mode=0):
    w = wl.make("tiny", "cuda", B=B, D=D, V=V, seed=seed, dtype=dtype, T=T, mode=mode,
                draft_sd=draft_sd)
    return w


@VARIANTS
@pytest.mark.parametrize("V", [1, 2, 5, 7, 8, 9, 100, 1023, 4096, 4096 * 8 + 1, 4096 * 8 + 9])
@pytest.mark.parametrize("dtype", [sv.SV_F32, sv.SV_BF16])
def test_vocab_sizes_and_alignment(sv, V, dtype, variant):
    # odd V makes every row after the first start off a 16-byte boundary
    w = make_random(5, 3, V, dtype=dtype, seed=V)
    for mode in (0, 1, 2):
        w.mode = mode
        compare(w, gpu_run(w, seed=mode, variant=variant), oracle_on(w, seed=mode))


@VARIANTS
@pytest.mark.parametrize("D", [0, 1, 32])
def test_draft_lengths(sv, D, variant):
    w = make_random(6, D, 3000, seed=D)
    for mode in (0, 1, 2):
        w.mode = mode
        compare(w, gpu_run(w, variant=variant), oracle_on(w))


@VARIANTS
def test_draft_lengths_long_short_long(sv, variant):
    # each draft length gets its own launch shape (the fused kernel's shared
    # memory grows with it): a long draft, a short one, then a new long one
    # must each launch and match the oracle, whatever was launched before
    for D, seed in ((12, 41), (1, 42), (11, 43), (12, 44)):
        w = make_random(5, D, 2500, seed=seed)
        compare(w, gpu_run(w, variant=variant), oracle_on(w))


@VARIANTS
def test_row_D_with_zero_and_nan_padding(sv, variant):
    w = make_random(8, 5, 5000, seed=3)
    row_D = torch.tensor([0, 5, 1, 0, 3, 5, 2, 4], dtype=torch.int32, device="cuda")
    for b, d in enumerate(row_D.tolist()):
        w.target[b, d + 1:] = float("nan")
        w.draft[b, d:] = float("nan")
        w.tokens[b, d:] = -5
    w.row_D = row_D
    for mode in (0, 1, 2):
        w.mode = mode
        got = gpu_run(w, variant=variant)
        assert np.all((got["flags"] & sv.SV_FLAG_ERRORS) == 0)
        compare(w, got, oracle_on(w))
    assert sv.sv_get_device_status() == 0


@VARIANTS
def test_saguaro_top_k_with_many_ties(sv, variant):
    # draft logits on a coarse grid (many equal values in and across lanes and
    # segments), plus copies of each row's maximum at spread-out positions, so
    # the top-k selection must break ties by the lowest index exactly as the oracle
    w = make_random(8, 4, 20000 + 37, seed=11, mode=2)
    q = torch.round(w.draft.float() * 2.0) / 2.0
    for b in range(w.B):
        for d in range(w.D_max):
            m = q[b, d].max()
            for x in (5, 4096 + 31, 8191, 12000 + d, 19999):
                q[b, d, x] = m
    w.draft.copy_(q.to(w.draft.dtype))
    got = gpu_run(w, variant=variant)
    assert np.all((got["flags"] & sv.SV_FLAG_ERRORS) == 0)
    compare(w, got, oracle_on(w))


def test_identical_target_and_draft_accept_everything(sv):
    w = make_random(16, 6, 20000, seed=4)
    w.draft.copy_(w.target[:, :6])
    for T in (1.0, 0.7):
        w.temperature = T
        got = gpu_run(w)
        assert np.all(got["accept_len"] == 7)
        compare(w, got, oracle_on(w))


def test_masked_tokens(sv):
    w = make_random(8, 3, 4000, seed=5)
    w.target[:, :, ::3] = float("-inf")
    w.draft[:, :, 1::3] = float("-inf")
    got = gpu_run(w)
    compare(w, got, oracle_on(w))
    n = got["accept_len"] - 1
    emitted = got["tokens"][np.arange(8), n]
    assert np.all(emitted % 3 != 0)  # p = 0 tokens are never emitted


@VARIANTS
def test_invalid_device_inputs_set_flags_and_status(sv, variant):
    w = make_random(6, 3, 3000, seed=6)
    assert sv.sv_get_device_status() == 0
    w.tokens[1, 0] = 3000
    w.target[2, 1, 17] = float("nan")
    w.draft[3, 2, 5] = float("inf")
    w.target[4, 0, :] = float("-inf")
    got = gpu_run(w, variant=variant)
    compare(w, got, oracle_on(w))
    assert got["flags"][1] & sv.SV_FLAG_BAD_TOKEN
    assert got["flags"][2] & sv.SV_FLAG_NONFINITE
    assert got["flags"][3] & sv.SV_FLAG_NONFINITE
    assert got["flags"][4] & sv.SV_FLAG_NONFINITE
    for b in (1, 2, 3, 4):
        assert got["accept_len"][b] == -1 and np.all(got["tokens"][b] == -1)
    st = sv.sv_get_device_status()
    assert st & sv.SV_FLAG_BAD_TOKEN and st & sv.SV_FLAG_NONFINITE
    assert sv.sv_get_device_status() == 0  # cleared by the read


@VARIANTS
def test_bad_row_D_and_per_request_parameters(sv, variant):
    w = make_random(6, 3, 3000, seed=7)
    w.row_D = torch.tensor([3, 4, -1, 2, 3, 3], dtype=torch.int32, device="cuda")
    w.temperature_per_req = torch.tensor([1.0, 1.0, 1.0, 0.0, 0.5, 1.0], device="cuda")
    w.mode_per_req = torch.tensor([0, 0, 0, 0, 1, 7], dtype=torch.int8, device="cuda")
    got = gpu_run(w, variant=variant)
    compare(w, got, oracle_on(w))
    assert got["flags"][1] & sv.SV_FLAG_BAD_ROW_D
    assert got["flags"][2] & sv.SV_FLAG_BAD_ROW_D
    assert got["flags"][3] & sv.SV_FLAG_BAD_PARAM
    assert got["flags"][5] & sv.SV_FLAG_BAD_PARAM
    assert not (got["flags"][4] & sv.SV_FLAG_ERRORS)
    sv.sv_get_device_status()


def test_greedy_entry_point_without_draft_logits(sv):
    w = make_random(10, 4, 9000, seed=8)
    out_t = torch.empty((10, 5), dtype=torch.int32, device="cuda")
    out_al = torch.empty((10,), dtype=torch.int32, device="cuda")
    rc = sv.sv_verify_greedy(w.target, w.tokens, None, 10, 4, 9000, sv.SV_BF16, out_t, out_al)
    assert rc == sv.SV_OK
    torch.cuda.synchronize()
    ref = oracle.verify(host_logits(w.target), None, w.tokens.cpu().numpy(), mode=oracle.SVO_GREEDY)
    assert np.array_equal(out_t.cpu().numpy(), ref["tokens"])
    assert np.array_equal(out_al.cpu().numpy(), ref["accept_len"])


def test_plain_entry_point_matches_ex(sv):
    w = make_random(10, 4, 9000, seed=9)
    out_t = torch.empty((10, 5), dtype=torch.int32, device="cuda")
    out_al = torch.empty((10,), dtype=torch.int32, device="cuda")
    rc = sv.sv_verify(w.target, w.draft, w.tokens, None, 10, 4, 9000, sv.SV_BF16, 1.0,
                      sv.SV_STOCHASTIC, 123, out_t, out_al)
    assert rc == sv.SV_OK
    ex = gpu_run(w, seed=123)
    assert np.array_equal(out_t.cpu().numpy(), ex["tokens"])
    assert np.array_equal(out_al.cpu().numpy(), ex["accept_len"])


def test_request_offset_matches_the_whole_batch(sv):
    w = make_random(12, 4, 7000, seed=10)
    full = gpu_run(w, seed=5)
    for b0, b1 in ((0, 5), (5, 12), (7, 8)):
        part = sv.verify(w.target[b0:b1], w.draft[b0:b1], w.tokens[b0:b1], temperature=1.0,
                         seed=5, request_offset=b0)
        torch.cuda.synchronize()
        assert np.array_equal(part["tokens"].cpu().numpy(), full["tokens"][b0:b1])
        assert np.array_equal(part["accept_len"].cpu().numpy(), full["accept_len"][b0:b1])


def test_explicit_workspace_and_stream(sv):
    w = make_random(9, 4, 20000, seed=11)
    ref = gpu_run(w, seed=2)
    need = sv.sv_workspace_bytes(9, 4, 20000, sv.SV_BF16)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = sv.verify_workload(w, seed=2, workspace=ws, stream=s)
    s.synchronize()
    assert np.array_equal(out["tokens"].cpu().numpy(), ref["tokens"])
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(sv.SvError, match="workspace too small"):
        sv.verify_workload(w, workspace=small)
