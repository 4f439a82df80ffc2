"""The pins must reject a broken oracle.

Each case plants one plausible mistake (a dropped term, a wrong sign, a wrong
index, a transposed operand) in a temporary copy of oracle/svo.c, builds it,
and checks that at least one of the pin checks below fails on it.  The
committed oracle itself is never modified.  The checks are smaller versions
of the pins in test_oracle_lse.py, test_oracle_philox.py and
test_oracle_rule.py."""
import math
import os
import subprocess
import tempfile

import numpy as np
import pytest

from svtest_util import bf16_bits, chi2_pvalue, sample_categorical, sample_rows, softmax, within_sigma

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "svo.c")

MUTANTS = {
    "lse_drops_temperature": ("s += exp(z / T - mT);", "s += exp(z - mT);"),
    "lse_wrong_offset": ("return mT + log(s);", "return m + log(s);"),
    "ratio_transposed": ("acc = fmin(1.0, exp(lp - lq));", "acc = fmin(1.0, exp(lq - lp));"),
    "accept_compare_flipped": ("if (!(u < acc)) {", "if (!(u > acc)) {"),
    "accept_scan_no_stop": ("        n = d;\n        break;\n      }\n    }\n\n    double gap",
                            "        n = d;\n      }\n    }\n\n    double gap"),
    "uniform_wrong_scale": ("return ldexp((double)(out[0] >> 8), -24);",
                            "return ldexp((double)(out[0] >> 9), -24);"),
    "residual_drops_q": ("lr = lp + log(-expm1(lq - lp));", "lr = lp;"),
    "residual_wrong_support": ("if (!(lp > lq)) continue;", "if (!(lp < lq)) continue;"),
    "race_noise_sign": ("double key = lr - log(svo_race_exponential",
                        "double key = lr + log(svo_race_exponential"),
    "race_noise_shared_lane": ("ldexp((double)out[x & 3u] + 0.5, -32)",
                               "ldexp((double)out[0] + 0.5, -32)"),
    "race_wrong_row": ("const void* trow_n = row_ptr(a->target, trow0 + n, V, dt);",
                       "const void* trow_n = row_ptr(a->target, trow0 + Db, V, dt);"),
    "philox_drops_key": ("uint32_t n0 = hi1 ^ c1 ^ k0;", "uint32_t n0 = hi1 ^ c1;"),
    "philox_two_rounds": ("for (int round = 0; round < 10; ++round)",
                          "for (int round = 0; round < 2; ++round)"),
    "philox_multipliers_swapped": (
        "    uint64_t prod0 = (uint64_t)0xD2511F53u * (uint64_t)c0;\n"
        "    uint64_t prod1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;",
        "    uint64_t prod0 = (uint64_t)0xCD9E8D57u * (uint64_t)c0;\n"
        "    uint64_t prod1 = (uint64_t)0xD2511F53u * (uint64_t)c2;"),
    "philox_words_permuted": ("  out[0] = c0;\n  out[1] = c1;\n  out[2] = c2;\n  out[3] = c3;",
                              "  out[0] = c2;\n  out[1] = c1;\n  out[2] = c0;\n  out[3] = c3;"),
    "philox_weyl_swapped": ("    k0 += 0x9E3779B9u;\n    k1 += 0xBB67AE85u;",
                            "    k0 += 0xBB67AE85u;\n    k1 += 0x9E3779B9u;"),
    "greedy_wrong_row": ("int am = svo_row_argmax(row_ptr(a->target, trow0 + d, V, dt), V, dt);",
                         "int am = svo_row_argmax(row_ptr(a->target, trow0 + d + 1, V, dt), V, dt);"),
    "argmax_last_tie": ("    if (z > bz) {\n      bz = z;\n      best = x;",
                        "    if (z >= bz) {\n      bz = z;\n      best = x;"),
    "saguaro_no_renormalise": ("return lq + (in_k ? q->ln_c : 0.0) - q->ln_Z;",
                               "return lq + (in_k ? q->ln_c : 0.0);"),
    "saguaro_topk_last_tie": ("if (best < 0 || z > bz) {", "if (best < 0 || z >= bz) {"),
    "epilogue_insert_one_late": ("row[AL - 1] = ot[AL - 1];", "if (AL < (int32_t)W) row[AL] = ot[AL - 1];"),
    "epilogue_no_shift": ("row[j] = window[(size_t)b * W + j + 1];", "row[j] = window[(size_t)b * W + j];"),
    "ssd_ignores_accept_len": ("if (keys_al[(size_t)b * K + k] == AL && keys_token[(size_t)b * K + k] == tok) hit = k;",
                               "if (keys_token[(size_t)b * K + k] == tok) hit = k;"),
    "ssd_last_match_wins": ("for (int k = 0; k < K && hit < 0; ++k)", "for (int k = 0; k < K; ++k)"),
    "tree_no_renormalise": ("for (int y = 0; y < V; ++y) P[y] = fmax(0.0, P[y] - q[y]) / Z;",
                            "for (int y = 0; y < V; ++y) P[y] = fmax(0.0, P[y] - q[y]);"),
    "tree_uniform_per_position": ("const double u = svo_accept_uniform(a->seed, g, (uint32_t)i);",
                                  "const double u = svo_accept_uniform(a->seed, g, (uint32_t)pos);"),
    "tree_greedy_last_child": ("for (int i = 0; i < n && found < 0; ++i)", "for (int i = 0; i < n; ++i)"),
    "epilogue_append_drops_last": ("for (int j = 0; j < AL; ++j) seq", "for (int j = 0; j + 1 < AL; ++j) seq"),
}


def tile(a, B):
    return np.ascontiguousarray(np.broadcast_to(a, (B,) + a.shape))


# ------------------------------------------------------------ pin checks


def check_lse(svo, L):
    for V, T in ((7, 0.7), (1024, 1.0), (300, 2.5)):
        if abs(svo.row_lse(np.full(V, 1.375, np.float32), T, L=L) - (1.375 / T + math.log(V))) > 1e-9:
            return False
    vals = np.array([-2.5] * 3 + [4.0] * 5, np.float32)
    expect = -2.5 / 0.7 + math.log(3 + 5 * math.exp(6.5 / 0.7))
    return abs(svo.row_lse(vals, 0.7, L=L) - expect) < 1e-9


def check_argmax(svo, L):
    rng = np.random.default_rng(11)
    for _ in range(30):
        z = np.round(rng.standard_normal(200) * 2).astype(np.float32)
        if svo.row_argmax(z, L=L) != int(np.argmax(z)):
            return False
    return True


def check_avalanche(svo, L):
    rng = np.random.default_rng(1)
    d = []
    for _ in range(100):
        ctr = [int(v) for v in rng.integers(0, 2**32, 4, dtype=np.uint64)]
        key = [int(v) for v in rng.integers(0, 2**32, 2, dtype=np.uint64)]
        for w in range(6):
            c2, k2 = list(ctr), list(key)
            if w < 4:
                c2[w] ^= 1 << int(rng.integers(0, 32))
            else:
                k2[w - 4] ^= 1 << int(rng.integers(0, 32))
            a = svo.philox4x32_10(ctr, key, L=L)
            b = svo.philox4x32_10(c2, k2, L=L)
            d.append(sum(bin(x ^ y).count("1") for x, y in zip(a, b)))
    d = np.array(d, float)
    return abs(d.mean() - 64) < 4 * 5.66 / math.sqrt(len(d)) and d.min() > 30


def check_kat(svo, L):
    # the published known answer (C++26 philox4x32, tests/golden/philox4x32_10_kat.txt)
    from test_oracle_philox_kat import read_kat
    return all(svo.philox4x32_10([c0, c1, c2, c3], [k0, k1], L=L)[w] == v
               for c0, c1, c2, c3, k0, k1, w, v in read_kat())


_ENGINE_WORDS = {}


def check_engines(svo, L):
    # every word against the independent host implementations (when they build here)
    if not _ENGINE_WORDS:
        import test_oracle_philox_kat as kat
        std_dir, torch_dir = kat._include_dirs()
        if torch_dir is None and std_dir is None:
            _ENGINE_WORDS["none"] = None
        else:
            with tempfile.TemporaryDirectory() as tmp:
                exe = os.path.join(tmp, "engines")
                cmd = ["g++", "-std=c++17", "-O1", kat.PROBE, "-o", exe]
                kinds = []
                if std_dir:
                    cmd[1:1] = ["-DWITH_STD_ENGINE", "-I", std_dir]
                    kinds.append("std")
                if torch_dir:
                    cmd[1:1] = ["-DWITH_TORCH_ENGINE", "-I", torch_dir]
                    kinds.append("torch")
                subprocess.run(cmd, check=True, capture_output=True)
                pairs = kat.pairs_to_check()[:300]
                _ENGINE_WORDS["pairs"] = pairs
                _ENGINE_WORDS["words"] = kat.run_engines((exe, kinds), pairs)
    if "none" in _ENGINE_WORDS:
        return True
    for words in _ENGINE_WORDS["words"].values():
        for (c, k), w in zip(_ENGINE_WORDS["pairs"], words):
            if svo.philox4x32_10(c, k, L=L) != w:
                return False
    return True


def check_uniform(svo, L):
    from scipy import stats
    u = np.array([svo.accept_uniform(9, g, dd, L=L) for g in range(1500) for dd in range(4)])
    return stats.kstest(u, "uniform").pvalue > 1e-4


def check_p_eq_q(svo, L):
    rng = np.random.default_rng(1)
    z = (rng.standard_normal((100, 4, 50)) * 3).astype(np.float32)
    tok = rng.integers(0, 50, (100, 3)).astype(np.int32)
    out = svo.verify(z, np.ascontiguousarray(z[:, :3]), tok, seed=3, L=L)
    return bool(np.all(out["accept_len"] == 4))


def check_al_law(svo, L):
    rng = np.random.default_rng(4)
    V, D, N = 8, 3, 60_000
    zt = (rng.standard_normal((D + 1, V)) * 1.5).astype(np.float32)
    zq = (zt[:D] + rng.standard_normal((D, V))).astype(np.float32)
    p, q = softmax(zt, 0.7), softmax(zq, 0.7)
    tok = np.array([int(np.argmax(q[d] / p[d])) if d % 2 == 0 else int(np.argmax(p[d]))
                    for d in range(D)], np.int32)
    a = np.minimum(1.0, p[np.arange(D), tok] / q[np.arange(D), tok])
    law = np.array([np.prod(a[:k]) * (1 - a[k]) for k in range(D)] + [np.prod(a)])
    out = svo.verify(tile(zt, N), tile(zq, N), tile(tok, N), temperature=0.7, seed=17, nthreads=8, L=L)
    counts = np.bincount(out["accept_len"] - 1, minlength=D + 1)
    return within_sigma(counts, law, 4.0)[0]


def check_residual_law(svo, L):
    rng = np.random.default_rng(5)
    V, N = 8, 60_000
    zt = (rng.standard_normal((2, V)) * 1.5).astype(np.float32)
    zq = (zt[:1] + rng.standard_normal((1, V)) * 1.5).astype(np.float32)
    p, q = softmax(zt)[0], softmax(zq)[0]
    x0 = int(np.argmax(q / p))
    r = np.maximum(0.0, p - q)
    r /= r.sum()
    out = svo.verify(tile(zt, N), tile(zq, N), np.full((N, 1), x0, np.int32), seed=23, nthreads=8, L=L)
    rej = out["accept_len"] == 1
    if not rej.any():
        return False
    emitted = out["tokens"][rej, 0]
    if np.any(emitted < 0) or np.any(p[emitted] <= q[emitted]):
        return False
    return within_sigma(np.bincount(emitted, minlength=V), r, 4.0)[0]


def check_bonus_law(svo, L):
    rng = np.random.default_rng(6)
    V, N = 8, 60_000
    zt = (rng.standard_normal((3, V)) * 1.5).astype(np.float32)
    p = softmax(zt, 0.5)[2]
    out = svo.verify(tile(zt, N), tile(zt[:2], N), np.zeros((N, 2), np.int32), temperature=0.5,
                     seed=29, nthreads=8, L=L)
    if not np.all(out["accept_len"] == 3):
        return False
    return within_sigma(np.bincount(out["tokens"][:, 2], minlength=V), p, 4.0)[0]


def check_marginal(svo, L, mode):
    rng = np.random.default_rng(100 + mode)
    V, D, N = 8, 2, 200_000
    zt = (rng.standard_normal((D + 1, V)) * 1.5).astype(np.float32)
    zq = (zt[:D] + rng.standard_normal((D, V)) * 1.2).astype(np.float32)
    p, q = softmax(zt), softmax(zq)
    qd = q.copy()
    if mode == 2:
        for d in range(D):
            top = np.lexsort((np.arange(V), -zq[d].astype(np.float64)))[:5]
            qd[d, top] *= 0.5
            qd[d] /= qd[d].sum()
    tok = np.stack([sample_categorical(rng, qd[d], N) for d in range(D)], axis=1)
    out = svo.verify(tile(zt, N), tile(zq, N), tok, mode=mode, seed=31, nthreads=8, L=L)
    AL, toks = out["accept_len"], out["tokens"]
    for slot, sel in ((0, np.ones_like(AL, bool)), (1, AL >= 2), (2, AL == 3)):
        if not within_sigma(np.bincount(toks[sel, slot], minlength=V), p[slot], 4.0)[0]:
            return False
    return True


def check_saguaro_ties(svo, L):
    # tied draft logits: K = tokens 0..4, q'(0..4) = 1/7, q'(5) = 2/7
    zq1 = np.zeros((1, 1, 6), np.float32)
    zt1 = np.zeros((1, 2, 6), np.float32)
    zt1[0, 0, :] = math.log(1 / 7) + 1e-6
    zt1[0, 0, 5] = math.log(2 / 7)
    for s in range(40):
        for x in (0, 5):
            out = svo.verify(zt1, zq1, np.array([[x]], np.int32), mode=2, seed=s, L=L)
            if x == 0 and out["accept_len"][0] != 2:
                return False
    return True


def check_greedy(svo, L):
    rng = np.random.default_rng(9)
    V, D = 40, 4
    Tt = (rng.standard_normal((V, V)) * 1.5).astype(np.float32)
    Qt = (Tt + rng.standard_normal((V, V)) * 0.8).astype(np.float32)
    ref, last = [], 0
    for _ in range(30):
        last = int(np.argmax(Tt[last]))
        ref.append(last)
    seq, last = [], 0
    while len(seq) < 30:
        prev, tok = [last], []
        for _ in range(D):
            tok.append(int(np.argmax(Qt[prev[-1]])))
            prev.append(tok[-1])
        out = svo.verify(Tt[np.array(prev)][None], None, np.array([tok], np.int32), mode=1, L=L)
        k = int(out["accept_len"][0])
        if k < 1:
            return False
        seq.extend(int(t) for t in out["tokens"][0, :k])
        last = seq[-1]
    if seq[:30] != ref:
        return False
    # a draft that proposes the target's own argmax chain is accepted in full
    prev = [0] + ref[:D]
    out = svo.verify(Tt[np.array(prev)][None], None, np.array([ref[:D]], np.int32), mode=1, L=L)
    return int(out["accept_len"][0]) == D + 1 and list(out["tokens"][0]) == ref[:D + 1]


def check_epilogue(svo, L):
    # the hand-written example and the greedy chain of test_oracle_epilogue.py
    import test_oracle_epilogue as te

    class Shim:
        SVO_GREEDY = svo.SVO_GREEDY

        @staticmethod
        def epilogue(*a, **k):
            return svo.epilogue(*a, L=L, **k)

        @staticmethod
        def verify(*a, **k):
            return svo.verify(*a, L=L, **k)
    try:
        te.test_worked_example(Shim)
        te.test_greedy_chain_with_epilogue_reproduces_argmax_decoding(Shim)
    except AssertionError:
        return False
    return True


def check_ssd(svo, L):
    import test_oracle_ssd as ts

    class Shim:
        @staticmethod
        def ssd_lookup(*a, **k):
            return svo.ssd_lookup(*a, L=L, **k)
    try:
        ts.test_lookup_worked_example(Shim)
        ts.test_lookup_against_a_dictionary(Shim)
    except AssertionError:
        return False
    return True


def check_tree(svo, L):
    import test_oracle_tree as tt

    class Shim:
        SVO_STOCHASTIC, SVO_GREEDY = svo.SVO_STOCHASTIC, svo.SVO_GREEDY
        FLAG_NEAR_TIE, FLAG_BAD_TOKEN = svo.FLAG_NEAR_TIE, svo.FLAG_BAD_TOKEN

        @staticmethod
        def verify(*a, **k):
            return svo.verify(*a, L=L, **k)

        @staticmethod
        def verify_tree(*a, **k):
            return svo.verify_tree(*a, L=L, **k)
    try:
        tt.test_chain_tree_is_the_linear_rule(Shim)
        tt.test_greedy_tree_reproduces_argmax_decoding(Shim)
        tt.test_emitted_tokens_follow_the_target(Shim)
        tt.test_the_first_matching_candidate_is_taken(Shim)
    except AssertionError:
        return False
    return True


CHECKS = [check_lse, check_argmax, check_kat, check_engines, check_avalanche, check_uniform, check_p_eq_q, check_al_law,
          check_residual_law, check_bonus_law, lambda s, L: check_marginal(s, L, 0),
          lambda s, L: check_marginal(s, L, 2), check_saguaro_ties, check_greedy, check_epilogue, check_ssd, check_tree]


def _build_variant(tmp, text):
    import oracle.build as ob
    src = os.path.join(tmp, "svo.c")
    with open(src, "w") as f:
        f.write(text)
    hdr = os.path.join(ROOT, "oracle", "svo.h")
    os.symlink(hdr, os.path.join(tmp, "svo.h"))
    lib = os.path.join(tmp, "libsvo_variant.so")
    subprocess.run(["gcc", *ob.CFLAGS, src, "-o", lib, "-lm"], check=True,
                   stderr=subprocess.DEVNULL)
    return lib


def test_unmodified_oracle_passes_every_check(svo):
    L = svo.lib()
    for chk in CHECKS:
        assert chk(svo, L), chk


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(svo, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    with tempfile.TemporaryDirectory() as tmp:
        L = svo.load_variant(_build_variant(tmp, text.replace(old, new)))
        failed = []
        for chk in CHECKS:
            try:
                ok = chk(svo, L)
            except Exception:  # a crash or a rejected call also counts as caught
                ok = False
            if not ok:
                failed.append(chk)
                break
        assert failed, f"no pin caught the planted mistake {name}"
