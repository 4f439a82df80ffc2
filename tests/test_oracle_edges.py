"""Oracle behaviour on invalid and degenerate inputs, and on the seeded
workloads at reduced sizes (the recipe is the same as at full size)."""
import numpy as np
import pytest

from speculative_decoding_verification_lse_b200 import workloads as wl
from svtest_util import sample_rows, softmax


def base(B=6, D=3, V=40, seed=0):
    rng = np.random.default_rng(seed)
    zt = (rng.standard_normal((B, D + 1, V)) * 3).astype(np.float32)
    zq = (zt[:, :D] + rng.standard_normal((B, D, V))).astype(np.float32)
    tok = sample_rows(rng, softmax(zq))
    return zt, zq, tok


def assert_minus_one(out, b):
    assert out["accept_len"][b] == -1
    assert np.all(out["tokens"][b] == -1)


def test_bad_token_is_reported_and_outputs_minus_one(svo):
    zt, zq, tok = base()
    tok[2, 1] = 40
    tok[4, 0] = -3
    out = svo.verify(zt, zq, tok, seed=1)
    for b in (2, 4):
        assert out["flags"][b] & svo.FLAG_BAD_TOKEN
        assert_minus_one(out, b)
    ok = [b for b in range(6) if b not in (2, 4)]
    assert np.all(out["accept_len"][ok] >= 1)


def test_bad_row_D_is_reported(svo):
    zt, zq, tok = base()
    row_D = np.array([3, 4, -1, 0, 2, 3], np.int32)
    out = svo.verify(zt, zq, tok, row_D, seed=1)
    for b in (1, 2):
        assert out["flags"][b] & svo.FLAG_BAD_ROW_D
        assert_minus_one(out, b)
    assert out["accept_len"][3] == 1 and 0 <= out["tokens"][3, 0] < 40


@pytest.mark.parametrize("bad", [np.nan, np.inf])
def test_nonfinite_needed_row_is_reported(svo, bad):
    zt, zq, tok = base()
    zt[1, 2, 7] = bad
    zq[3, 0, 0] = bad
    out = svo.verify(zt, zq, tok, seed=1)
    for b in (1, 3):
        assert out["flags"][b] & svo.FLAG_NONFINITE
        assert_minus_one(out, b)


def test_all_masked_row_is_reported_but_minus_inf_entries_are_fine(svo):
    zt, zq, tok = base()
    zt[0, 1, :] = -np.inf
    zt[2, 1, :5] = -np.inf
    out = svo.verify(zt, zq, tok, seed=1)
    assert out["flags"][0] & svo.FLAG_NONFINITE
    assert not (out["flags"][2] & svo.FLAG_ERRORS)


def test_padding_rows_and_tokens_are_never_read(svo):
    zt, zq, tok = base()
    row_D = np.array([0, 1, 2, 3, 1, 0], np.int32)
    zt2, zq2, tok2 = zt.copy(), zq.copy(), tok.copy()
    for b, d in enumerate(row_D):
        zt2[b, d + 1:] = np.nan
        zq2[b, d:] = np.nan
        tok2[b, d:] = -7
    a = svo.verify(zt, zq, tok, row_D, seed=4)
    b = svo.verify(zt2, zq2, tok2, row_D, seed=4)
    assert np.all((b["flags"] & svo.FLAG_ERRORS) == 0)
    for k in ("tokens", "accept_len", "flags"):
        np.testing.assert_array_equal(a[k], b[k])
    np.testing.assert_array_equal(a["row_lse"], b["row_lse"])


def test_greedy_never_reads_draft_logits(svo):
    zt, zq, tok = base()
    a = svo.verify(zt, np.full_like(zq, np.nan), tok, mode=svo.SVO_GREEDY)
    b = svo.verify(zt, None, tok, mode=svo.SVO_GREEDY)
    assert np.all(a["flags"] == 0)
    np.testing.assert_array_equal(a["tokens"], b["tokens"])
    assert np.all(np.isnan(a["row_lse"]))


def test_temperature_rules(svo):
    zt, zq, tok = base()
    with pytest.raises(ValueError):
        svo.verify(zt, zq, tok, temperature=0.0)
    # greedy ignores T
    g0 = svo.verify(zt, zq, tok, temperature=0.0, mode=svo.SVO_GREEDY)
    g1 = svo.verify(zt, zq, tok, temperature=3.0, mode=svo.SVO_GREEDY)
    np.testing.assert_array_equal(g0["tokens"], g1["tokens"])
    # a per-request T <= 0 on a stochastic request is reported on that request
    tpr = np.array([1.0, 0.0, 0.5, -1.0, 1.0, 1.0], np.float32)
    mpr = np.array([0, 0, 0, 1, 2, 0], np.int8)
    out = svo.verify(zt, zq, tok, temperature_per_req=tpr, mode_per_req=mpr, seed=2)
    assert out["flags"][1] & svo.FLAG_BAD_PARAM
    assert not (out["flags"][3] & svo.FLAG_ERRORS)  # greedy: T unused
    # per-request T equals a global T for the same value
    one = svo.verify(zt[2:3], zq[2:3], tok[2:3], temperature=0.5, seed=2, request_offset=2)
    np.testing.assert_array_equal(one["tokens"][0], out["tokens"][2])
    np.testing.assert_array_equal(one["row_lse"][0], out["row_lse"][2])


def test_row_lse_slots(svo):
    zt, zq, tok = base(B=2, D=2, V=30)
    T = float(np.float32(0.9))  # the call takes T as a single
    out = svo.verify(zt, zq, tok, temperature=T, seed=0)
    for b in range(2):
        for d in range(3):
            assert out["row_lse"][b, d] == svo.row_lse(zt[b, d], T)
        for d in range(2):
            assert out["row_lse"][b, 3 + d] == svo.row_lse(zq[b, d], T)


@pytest.mark.parametrize("name", sorted(wl.CONFIGS))
def test_workloads_run_clean_through_the_oracle(svo, name):
    small = dict(V=1000, B=min(wl.CONFIGS[name]["B"], 16))
    w = wl.make(name, "cpu", **small)
    h = w.host_arrays()
    out = svo.verify(h["target"], h["draft"], h["tokens"], h["row_D"], temperature=w.temperature,
                     mode=w.mode, seed=w.seed, temperature_per_req=h["temperature_per_req"],
                     mode_per_req=h["mode_per_req"], saguaro_k=w.saguaro_k,
                     saguaro_c=w.saguaro_c)
    assert np.all((out["flags"] & svo.FLAG_ERRORS) == 0)
    D = np.array(w.row_D_list())
    assert np.all(out["accept_len"] >= 1) and np.all(out["accept_len"] <= D + 1)
    assert w.algorithmic_bytes() > 0 and w.verified_rows() == int((D + 1).sum())


def test_full_size_byte_counts():
    # the algorithmic bytes of the two fixed full-size workloads, from their shapes
    # (the ragged one depends on its draws)
    s = 2
    assert (256 * (8 + 7 + 1)) * 128256 * s == 1_050_673_152
    assert (128 * (5 + 4 + 1)) * 129280 * s == 330_956_800
    assert (32 * (5 + 4 + 1)) * 128256 * s == 82_083_840
