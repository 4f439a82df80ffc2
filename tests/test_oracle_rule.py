"""Pins for the oracle's verification rule: invariants the pages fix, closed-form
laws, brute-force statistical checks and a toy autoregressive chain.

  * AL lies in [1, 1 + D]                        (NVIDIA guidelines page, definitions)
  * p = q accepts every draft                    (SSD post, rule item 1)
  * the residual never emits a token with p <= q (SSD post, rule item 3)
  * output ~ p exactly                           (SSD post, closing remark of the rule)
  * greedy verification = argmax decoding        (NVIDIA guidelines page, "Mit csinál...")
The expected laws are computed here from the textbook softmax, never by the
oracle.  Per-cell bounds are 4 sigma next to a chi^2 test (many cells are
checked, so 3 sigma would fail a correct sampler by chance); the 10^6-draw
marginal test keeps the 3 sigma bound it is specified with."""
import math
import os

import numpy as np
import pytest

from svtest_util import (bf16_bits, chi2_pvalue, sample_categorical, sample_rows, softmax,
                         within_sigma)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

NT = 8  # host threads for the large statistical runs (same code path as 1)


def tile(row_block, B):
    return np.ascontiguousarray(np.broadcast_to(row_block, (B,) + row_block.shape))


def test_openmp_split_is_identical_to_single_thread(svo):
    rng = np.random.default_rng(0)
    B, D, V = 64, 4, 257
    zt = (rng.standard_normal((B, D + 1, V)) * 3).astype(np.float32)
    zq = (zt[:, :D] + rng.standard_normal((B, D, V))).astype(np.float32)
    tok = rng.integers(0, V, (B, D)).astype(np.int32)
    a = svo.verify(zt, zq, tok, seed=5, nthreads=1)
    b = svo.verify(zt, zq, tok, seed=5, nthreads=NT)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1.0, 0.6])
def test_p_equals_q_accepts_everything(svo, dtype, T):
    rng = np.random.default_rng(1)
    B, D, V = 400, 5, 300
    z = (rng.standard_normal((B, D + 1, V)) * 3).astype(np.float32)
    tok = rng.integers(0, V, (B, D)).astype(np.int32)
    zt = z if dtype == "f32" else bf16_bits(z)
    out = svo.verify(zt, np.ascontiguousarray(zt[:, :D]), tok, temperature=T, seed=3)
    assert np.all(out["accept_len"] == D + 1)
    np.testing.assert_array_equal(out["tokens"][:, :D], tok)
    assert np.all((out["flags"] & svo.FLAG_ERRORS) == 0)


def test_accept_length_bounds_and_output_layout(svo):
    rng = np.random.default_rng(2)
    B, D, V = 2000, 6, 64
    zt = (rng.standard_normal((B, D + 1, V)) * 3).astype(np.float32)
    zq = (zt[:, :D] + rng.standard_normal((B, D, V)) * 2).astype(np.float32)
    tok = sample_rows(rng, softmax(zq))
    out = svo.verify(zt, zq, tok, seed=11, nthreads=NT)
    AL = out["accept_len"]
    assert AL.min() >= 1 and AL.max() <= D + 1
    assert len(np.unique(AL)) == D + 1  # every length occurs
    for b in range(B):
        n = AL[b] - 1
        np.testing.assert_array_equal(out["tokens"][b, :n], tok[b, :n])
        assert 0 <= out["tokens"][b, n] < V
        assert np.all(out["tokens"][b, n + 1:] == -1)


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_accept_length_law_closed_form(svo, T):
    # fixed rows and drafts: P(AL = k+1) = prod_{d<k} a_d (1 - a_k), a_D = 0
    rng = np.random.default_rng(4)
    V, D, N = 8, 3, 200_000
    zt = (rng.standard_normal((D + 1, V)) * 1.5).astype(np.float32)
    zq = (zt[:D] + rng.standard_normal((D, V))).astype(np.float32)
    p, q = softmax(zt, T), softmax(zq, T)
    tok = np.array([int(np.argmax(q[d] / p[d][:])) if d % 2 == 0 else int(np.argmax(p[d]))
                    for d in range(D)], dtype=np.int32)
    a = np.minimum(1.0, p[np.arange(D), tok] / q[np.arange(D), tok])
    assert a.min() < 0.9
    law = np.array([np.prod(a[:k]) * (1 - a[k]) for k in range(D)] + [np.prod(a)])
    out = svo.verify(tile(zt, N), tile(zq, N), tile(tok, N), temperature=T, seed=17,
                     nthreads=NT)
    counts = np.bincount(out["accept_len"] - 1, minlength=D + 1)
    ok, worst = within_sigma(counts, law, 4.0)
    assert ok, (counts / N, law, worst)
    assert chi2_pvalue(counts, law) > 1e-4


@pytest.mark.parametrize("T", [1.0, 0.8])
def test_residual_law_and_support(svo, T):
    # after a rejection the emitted token ~ norm(max(0, p - q)) and never has p <= q
    rng = np.random.default_rng(5)
    V, D, N = 8, 1, 200_000
    zt = (rng.standard_normal((D + 1, V)) * 1.5).astype(np.float32)
    zq = (zt[:D] + rng.standard_normal((D, V)) * 1.5).astype(np.float32)
    p, q = softmax(zt, T)[0], softmax(zq, T)[0]
    x0 = int(np.argmax(q / p))
    r = np.maximum(0.0, p - q)
    r /= r.sum()
    out = svo.verify(tile(zt, N), tile(zq, N), np.full((N, 1), x0, np.int32), temperature=T,
                     seed=23, nthreads=NT)
    rej = out["accept_len"] == 1
    assert 0.05 < rej.mean() < 0.95
    emitted = out["tokens"][rej, 0]
    assert np.all(p[emitted] > q[emitted])
    counts = np.bincount(emitted, minlength=V)
    ok, worst = within_sigma(counts, r, 4.0)
    assert ok, worst
    assert chi2_pvalue(counts, r) > 1e-4


@pytest.mark.parametrize("T", [1.0, 0.5])
def test_bonus_law_without_drafts(svo, T):
    # D = 0: no draft, AL = 1 and the token ~ p
    rng = np.random.default_rng(6)
    V, N = 8, 200_000
    zt = (rng.standard_normal((1, V)) * 1.5).astype(np.float32)
    zt[0, 3] = -np.inf  # a masked token is never emitted
    p = softmax(zt, T)[0]
    out = svo.verify(tile(zt, N), np.zeros((N, 0, V), np.float32), np.zeros((N, 0), np.int32),
                     temperature=T, seed=29, nthreads=NT)
    assert np.all(out["accept_len"] == 1)
    counts = np.bincount(out["tokens"][:, 0], minlength=V)
    assert counts[3] == 0
    ok, worst = within_sigma(counts, p, 4.0)
    assert ok, worst
    assert chi2_pvalue(counts, p) > 1e-4


def _marginal_run(svo, mode, seed):
    rng = np.random.default_rng(100 + mode)
    V, D, N = 8, 2, 1_000_000
    zt = (rng.standard_normal((D + 1, V)) * 1.5).astype(np.float32)
    zq = (zt[:D] + rng.standard_normal((D, V)) * 1.2).astype(np.float32)
    p, q = softmax(zt), softmax(zq)
    if mode == svo.SVO_SAGUARO:
        # the draft samples from q' = q c^[x in top5] / Z
        c = 0.5
        qd = q.copy()
        for d in range(D):
            top = np.lexsort((np.arange(V), -zq[d].astype(np.float64)))[:5]
            qd[d, top] *= c
            qd[d] /= qd[d].sum()
    else:
        qd = q
    tok = np.stack([sample_categorical(rng, qd[d], N) for d in range(D)], axis=1)
    out = svo.verify(tile(zt, N), tile(zq, N), tok, mode=mode, seed=seed, nthreads=NT)
    return p, out


@pytest.mark.slow
@pytest.mark.parametrize("mode", [0, 2], ids=["plain", "saguaro"])
def test_emitted_marginals_equal_target_v8_d2_1e6(svo, mode):
    """V=8, D=2, 10^6 draws: the first emitted token ~ p_0, the second (when
    the first draft was accepted) ~ p_1, the third (both accepted) ~ p_2."""
    p, out = _marginal_run(svo, mode, seed=31)
    AL, toks = out["accept_len"], out["tokens"]
    for slot, sel in ((0, np.ones_like(AL, bool)), (1, AL >= 2), (2, AL == 3)):
        counts = np.bincount(toks[sel, slot], minlength=p.shape[1])
        ok, worst = within_sigma(counts, p[slot], 3.0)
        assert ok, (slot, worst)


def _bigram_tables(rng, V, noise):
    Tt = (rng.standard_normal((V, V)) * 1.5).astype(np.float32)
    Qt = (Tt + rng.standard_normal((V, V)) * noise).astype(np.float32)
    return Tt, Qt


@pytest.mark.slow
def test_speculative_chain_reproduces_the_target_chain(svo):
    """Toy bigram 'models': the target's logits for the next token are Tt[prev],
    the draft's Qt[prev].  Repeated speculative steps (draft D tokens, verify,
    append AL tokens) must generate sequences distributed exactly like sampling
    the target chain one token at a time: chi^2 on the first three tokens."""
    rng = np.random.default_rng(8)
    V, D, L, N = 6, 3, 3, 120_000
    Tt, Qt = _bigram_tables(rng, V, 1.0)
    P, Q = softmax(Tt), softmax(Qt)
    seqs = np.full((N, L + D + 1), -1, np.int32)
    lens = np.zeros(N, np.int64)
    c0 = 0
    step = 0
    while np.any(lens < L):
        act = np.nonzero(lens < L)[0]
        last = np.where(lens[act] > 0, seqs[act, np.maximum(lens[act] - 1, 0)], c0)
        prev = np.empty((len(act), D + 1), np.int32)
        prev[:, 0] = last
        tok = np.empty((len(act), D), np.int32)
        for d in range(D):
            tok[:, d] = sample_rows(rng, Q[prev[:, d]])
            prev[:, d + 1] = tok[:, d]
        zt = Tt[prev]              # [n, D+1, V]: target row d scores draft token d
        zq = Qt[prev[:, :D]]       # [n, D, V]
        out = svo.verify(zt, zq, tok, seed=1000 + step, nthreads=NT)
        for i, b in enumerate(act):
            k = int(out["accept_len"][i])
            seqs[b, lens[b]:lens[b] + k] = out["tokens"][i, :k]
            lens[b] += k
        step += 1
    y = seqs[:, :L].astype(np.int64)
    cells = y[:, 0] * V * V + y[:, 1] * V + y[:, 2]
    counts = np.bincount(cells, minlength=V ** 3)
    law = (P[c0][:, None, None] * P[:, :, None] * P[None, :, :]).reshape(-1)
    assert chi2_pvalue(counts, law) > 1e-4


def test_greedy_speculation_equals_argmax_decoding(svo):
    rng = np.random.default_rng(9)
    V, D, L = 40, 4, 60
    Tt, Qt = _bigram_tables(rng, V, 0.8)
    ref = [0]
    for _ in range(L):
        ref.append(int(np.argmax(Tt[ref[-1]])))
    ref = ref[1:]
    seq = []
    last = 0
    while len(seq) < L:
        prev = [last]
        tok = []
        for d in range(D):
            tok.append(int(np.argmax(Qt[prev[-1]])))
            prev.append(tok[-1])
        zt = Tt[np.array(prev)][None]
        zq = np.full((1, D, V), np.nan, np.float32)  # greedy never reads the draft
        out = svo.verify(zt, zq, np.array([tok], np.int32), mode=svo.SVO_GREEDY)
        k = int(out["accept_len"][0])
        assert out["flags"][0] == 0
        seq.extend(int(t) for t in out["tokens"][0, :k])
        last = seq[-1]
    assert seq[:L] == ref
    # a draft that proposes the target's own argmax chain is accepted in full
    for start in range(0, L - D, 7):
        prev = [ref[start - 1] if start else 0] + ref[start:start + D]
        out = svo.verify(Tt[np.array(prev)][None], None, np.array([ref[start:start + D]], np.int32),
                         mode=svo.SVO_GREEDY)
        assert int(out["accept_len"][0]) == D + 1
        assert list(out["tokens"][0]) == ref[start:start + D + 1]


def test_greedy_mismatch_emits_target_argmax(svo):
    V = 10
    zt = np.zeros((1, 3, V), np.float32)
    zt[0, 0, 4] = 2.0
    zt[0, 1, 7] = 2.0
    zt[0, 2, 1] = 2.0
    out = svo.verify(zt, None, np.array([[4, 5]], np.int32), mode=svo.SVO_GREEDY)
    assert out["accept_len"][0] == 2
    np.testing.assert_array_equal(out["tokens"][0], [4, 7, -1])
    out = svo.verify(zt, None, np.array([[4, 7]], np.int32), mode=svo.SVO_GREEDY)
    np.testing.assert_array_equal(out["tokens"][0], [4, 7, 1])


def test_saguaro_topk_and_downweighting(svo):
    """With c = 1 saguaro is the plain rule; with ties the top-k set is the
    lowest indices.  A draft token outside the top-k has q' = q / Z > q."""
    rng = np.random.default_rng(10)
    B, D, V = 300, 3, 50
    zt = (rng.standard_normal((B, D + 1, V)) * 2).astype(np.float32)
    zq = (zt[:, :D] + rng.standard_normal((B, D, V))).astype(np.float32)
    tok = sample_rows(rng, softmax(zq))
    plain = svo.verify(zt, zq, tok, seed=41)
    same = svo.verify(zt, zq, tok, seed=41, mode=svo.SVO_SAGUARO, saguaro_c=1.0)
    for k in ("tokens", "accept_len"):
        np.testing.assert_array_equal(plain[k], same[k])


def read_saguaro_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "saguaro_tied_draft.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, *v = line.split()
                vals[k] = [float(x) for x in v]
    return int(vals["V"][0]), vals["c"][0], vals["Z"][0], np.array(vals["qprime"])


def test_saguaro_tied_draft_matches_the_hand_computed_case(svo):
    """tests/golden/saguaro_tied_draft.txt: every draft logit 0 at V=6, so K is
    tokens 0..4 (lowest indices on ties) and q' is known by hand.  The oracle
    must accept token x with probability min(1, p(x)/q'(x)): always when p(x)
    is just above q'(x), with probability 1/2 when p(x) = q'(x)/2, never when
    p(x) = 0."""
    V, c, Z, qp = read_saguaro_golden()
    zq = np.zeros((1, 1, V), np.float32)
    N = 4000
    for x in (0, 5):
        for scale, rate in ((1.0 + 1e-5, 1.0), (0.5, 0.5), (0.0, 0.0)):
            px = qp[x] * scale
            p = np.full(V, (1.0 - px) / (V - 1))
            p[x] = px
            zt = np.zeros((1, 2, V), np.float32)
            with np.errstate(divide="ignore"):
                zt[0, 0] = np.log(p).astype(np.float32)  # p(x) = 0 -> -inf, a masked token
            out = svo.verify(np.repeat(zt, N, 0), np.repeat(zq, N, 0), np.full((N, 1), x, np.int32),
                             mode=svo.SVO_SAGUARO, saguaro_c=c, seed=3)
            acc = float(np.mean(out["accept_len"] == 2))
            if rate in (0.0, 1.0):
                assert acc == rate, (x, scale, acc)
            else:
                assert abs(acc - rate) < 4 * math.sqrt(rate * (1 - rate) / N), (x, scale, acc)
            # an emitted correction is never the rejected draft when p(x) <= q'(x)
            rej = out["accept_len"] == 1
            assert np.all(out["tokens"][rej, 0] != x)
    assert abs(Z - (1 - (1 - c) * 5 / V)) < 1e-15 and abs(qp.sum() - 1) < 1e-12


def test_accept_near_tie_is_flagged(svo):
    seed = 77
    u = svo.accept_uniform(seed, 0, 0)
    zq = np.zeros((1, 1, 2), np.float32)                  # q(0) = 1/2
    for eps, flagged in ((3e-6, True), (-3e-6, True), (2e-3, False)):
        p0 = 0.5 * (u + eps)
        zt = np.zeros((1, 2, 2), np.float32)
        zt[0, 0] = [math.log(p0), math.log(1 - p0)]
        out = svo.verify(zt, zq, np.array([[0]], np.int32), seed=seed)
        assert bool(out["flags"][0] & svo.FLAG_ACCEPT_NEAR_TIE) == flagged, eps
        if not flagged:
            assert out["accept_len"][0] == 2


def test_race_near_tie_is_flagged(svo):
    seed, V = 5, 2
    e0, e1 = svo.race_exponential(seed, 0, 0), svo.race_exponential(seed, 0, 1)
    for extra, flagged, winner in ((0.0, True, None), (0.05, False, 1), (-0.05, False, 0)):
        zt = np.array([[[0.0, math.log(e1 / e0) + extra]]], np.float32)
        out = svo.verify(zt, np.zeros((1, 0, V), np.float32), np.zeros((1, 0), np.int32),
                         seed=seed)
        assert bool(out["flags"][0] & svo.FLAG_RACE_NEAR_TIE) == flagged
        if winner is not None:
            assert out["tokens"][0, 0] == winner


def test_request_offset_gives_the_same_slice(svo):
    rng = np.random.default_rng(12)
    B, D, V = 12, 3, 100
    zt = (rng.standard_normal((B, D + 1, V)) * 3).astype(np.float32)
    zq = (zt[:, :D] + rng.standard_normal((B, D, V))).astype(np.float32)
    tok = sample_rows(rng, softmax(zq))
    full = svo.verify(zt, zq, tok, seed=9)
    part = svo.verify(zt[4:9], zq[4:9], tok[4:9], seed=9, request_offset=4)
    for k in full:
        np.testing.assert_array_equal(full[k][4:9], part[k])


def test_seed_changes_outcomes(svo):
    rng = np.random.default_rng(13)
    B, D, V = 200, 3, 100
    zt = (rng.standard_normal((B, D + 1, V)) * 3).astype(np.float32)
    zq = (zt[:, :D] + rng.standard_normal((B, D, V))).astype(np.float32)
    tok = sample_rows(rng, softmax(zq))
    a = svo.verify(zt, zq, tok, seed=1)
    b = svo.verify(zt, zq, tok, seed=2**40 + 1)  # differs only in the key's high word
    assert np.mean(a["tokens"] != b["tokens"]) > 0.05
