"""Pins for the oracle's speculative-speculative-decoding pieces: the top-k of a
row (brute force on rows full of ties), the outcome lookup (a worked example and
an independent dictionary lookup on random cases), and the purpose the page
gives saguaro sampling ("Speculative Speculative Decoding – асинхронизируй
это.", saguaro recipe items 1-3: lowering the draft's top-5 makes the residual
concentrate on them), checked statistically: the correction token lands in the
draft's top-5 more often under saguaro than under the plain rule."""
import numpy as np
import pytest

from svtest_util import bf16_bits, sample_rows, softmax


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_topk_brute_force(svo, dtype):
    rng = np.random.default_rng(4)
    for _ in range(200):
        V = int(rng.integers(1, 300))
        k = int(rng.integers(1, min(V, 8) + 1))
        z = np.round(rng.standard_normal(V) * 2).astype(np.float32)  # many ties
        row = z if dtype == "f32" else bf16_bits(z)
        want = np.lexsort((np.arange(V), -z.astype(np.float64)))[:k]
        np.testing.assert_array_equal(svo.row_topk(row, k), want)


def test_lookup_worked_example(svo):
    out = np.array([[3, 9, -1], [4, 4, 4], [7, -1, -1], [-1, -1, -1]], np.int32)
    AL = np.array([2, 3, 1, -1], np.int32)
    keys_al = np.array([[2, 2, 1], [3, 1, 3], [2, 1, 1], [1, 1, 1]], np.int32)
    keys_tok = np.array([[8, 9, 9], [4, 4, 4], [7, 7, 6], [-1, -1, -1]], np.int32)
    spec = np.arange(4 * 3 * 2, dtype=np.int32).reshape(4, 3, 2)
    r = svo.ssd_lookup(out, AL, keys_al, keys_tok, spec)
    # request 0: (2, 9) is key 1; request 1: (3, 4) is key 0 (the first of two);
    # request 2: (1, 7) is key 1 (key 0 has the token but AL 2); request 3: flagged
    np.testing.assert_array_equal(r["hit"], [1, 0, 1, -1])
    np.testing.assert_array_equal(r["spec"], [[2, 3], [6, 7], [14, 15], [-1, -1]])


def test_lookup_against_a_dictionary(svo):
    rng = np.random.default_rng(8)
    B, D, K, S = 300, 5, 12, 4
    out = rng.integers(0, 20, (B, D + 1)).astype(np.int32)
    AL = rng.integers(-1, D + 3, B).astype(np.int32)
    keys_al = rng.integers(1, D + 2, (B, K)).astype(np.int32)
    keys_tok = rng.integers(0, 20, (B, K)).astype(np.int32)
    spec = rng.integers(0, 1000, (B, K, S)).astype(np.int32)
    r = svo.ssd_lookup(out, AL, keys_al, keys_tok, spec)
    for b in range(B):
        table = {}
        for k in range(K - 1, -1, -1):  # later keys first, so the lowest index stays
            table[(int(keys_al[b, k]), int(keys_tok[b, k]))] = k
        a = int(AL[b])
        want = table.get((a, int(out[b, a - 1])), -1) if 1 <= a <= D + 1 else -1
        assert r["hit"][b] == want
        np.testing.assert_array_equal(r["spec"][b], spec[b, want] if want >= 0 else [-1] * S)


def test_saguaro_concentrates_the_correction_on_the_draft_top5(svo):
    rng = np.random.default_rng(12)
    B, D, V = 3000, 1, 60
    zt = (rng.standard_normal((B, D + 1, V)) * 2.0).astype(np.float32)
    zq = (zt[:, :D] + rng.standard_normal((B, D, V)) * 1.0).astype(np.float32)
    rates = {}
    for mode in (svo.SVO_STOCHASTIC, svo.SVO_SAGUARO):
        q = softmax(zq)
        if mode == svo.SVO_SAGUARO:  # drafts come from q'
            for b in range(B):
                top = svo.row_topk(zq[b, 0], 5)
                q[b, 0, top] *= 0.5
                q[b, 0] /= q[b, 0].sum()
        tok = sample_rows(rng, q)
        out = svo.verify(zt, zq, tok, mode=mode, seed=5, nthreads=8)
        rej = out["accept_len"] == 1
        hits = [out["tokens"][b, 0] in set(svo.row_topk(zq[b, 0], 5).tolist())
                for b in np.nonzero(rej)[0]]
        rates[mode] = float(np.mean(hits))
    assert rates[svo.SVO_SAGUARO] > rates[svo.SVO_STOCHASTIC] + 0.03, rates
