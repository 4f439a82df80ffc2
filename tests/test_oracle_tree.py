"""Pins for the oracle's tree (multi-candidate) verification (svo_verify_tree):
a chain tree is the linear rule, token for token; greedy tree verification
reproduces plain argmax decoding of a toy model; and the output is
distributed like the target at every position (the emitted first token's law
is p at the root, and the next token after an accepted node follows p at that
node's position), checked by per-cell bounds over many requests whose
candidates are independent draws from q."""
import numpy as np
import pytest

from svtest_util import bf16_bits, sample_categorical, softmax, within_sigma


def test_chain_tree_is_the_linear_rule(svo):
    rng = np.random.default_rng(2)
    B, D, V = 200, 5, 300
    for dtype in ("f32", "bf16"):
        zt = (rng.standard_normal((B, D + 1, V)) * 2.5).astype(np.float32)
        zq = (zt[:, :D] + rng.standard_normal((B, D, V))).astype(np.float32)
        p = softmax(zq, 0.8)
        tok = np.stack([sample_categorical(rng, p[b, d], 1)[0] for b in range(B) for d in range(D)]
                       ).reshape(B, D).astype(np.int32)
        if dtype == "bf16":
            zt, zq = bf16_bits(zt), bf16_bits(zq)
        chain = np.tile(np.arange(D, dtype=np.int32), (B, 1))
        for mode in (svo.SVO_STOCHASTIC, svo.SVO_GREEDY):
            lin = svo.verify(zt, zq, tok, temperature=0.8, mode=mode, seed=9, nthreads=8)
            tree = svo.verify_tree(zt, zq, tok, chain, temperature=0.8, mode=mode, seed=9, nthreads=8)
            ok = ((lin["flags"] | tree["flags"]) & svo.FLAG_NEAR_TIE) == 0
            assert ok.sum() >= B - 2
            np.testing.assert_array_equal(lin["tokens"][ok], tree["tokens"][ok])
            np.testing.assert_array_equal(lin["accept_len"][ok], tree["accept_len"][ok])
            al = tree["accept_len"]
            for b in range(B):
                np.testing.assert_array_equal(tree["nodes"][b, :al[b] - 1], np.arange(al[b] - 1))


def test_greedy_tree_reproduces_argmax_decoding(svo):
    """Toy bigram target Tt and draft Qt; each step drafts a tree (the draft's
    top-3 at the root, the draft's top-2 under each of those) and verifies it
    greedily; the accepted path plus the emitted token continue the sequence,
    which equals argmax decoding of Tt."""
    rng = np.random.default_rng(7)
    V = 40
    Tt = (rng.standard_normal((V, V)) * 1.5).astype(np.float32)
    Qt = (Tt + rng.standard_normal((V, V)) * 1.0).astype(np.float32)
    ref, last = [], 0
    for _ in range(60):
        last = int(np.argmax(Tt[last]))
        ref.append(last)
    seq, last = [], 0
    while len(seq) < 60:
        top = lambda t, k: list(np.argsort(-Qt[t], kind="stable")[:k])  # noqa: E731
        tokens, parents, ctx = [], [], [last]
        for x in top(last, 3):
            tokens.append(x)
            parents.append(0)
        for i in range(3):
            for x in top(tokens[i], 2):
                tokens.append(x)
                parents.append(i + 1)
        # target row p: the distribution after position p (root = last, node i = tokens[i])
        rows = [Tt[last]] + [Tt[t] for t in tokens]
        out = svo.verify_tree(np.array(rows, np.float32)[None], None, np.array([tokens], np.int32),
                              np.array([parents], np.int32), mode=svo.SVO_GREEDY)
        k = int(out["accept_len"][0])
        seq.extend(int(t) for t in out["tokens"][0, :k])
        last = seq[-1]
    assert seq[:60] == ref


def test_emitted_tokens_follow_the_target(svo):
    """V = 6; the root has three candidates drawn independently from q_root,
    each with two candidates drawn from q at its position.  Over 2e5 requests
    (independent draws: one request per draw), the first emitted token has law
    p_root, and the token after an accepted node c has law p_(c+1)."""
    rng = np.random.default_rng(31)
    V, N, R = 6, 9, 200_000
    zt = (rng.standard_normal((N + 1, V)) * 1.3).astype(np.float32)
    zq = (zt[:N] + rng.standard_normal((N, V)) * 1.1).astype(np.float32)
    p, q = softmax(zt), softmax(zq)
    parents = np.array([0, 0, 0, 1, 1, 2, 2, 3, 3], np.int32)
    tokens = np.stack([sample_categorical(rng, q[parents[i]], R) for i in range(N)], axis=1)
    out = svo.verify_tree(np.broadcast_to(zt, (R, N + 1, V)), np.broadcast_to(zq, (R, N, V)),
                          tokens, np.broadcast_to(parents, (R, N)), seed=11, nthreads=8)
    first = out["tokens"][:, 0]
    assert within_sigma(np.bincount(first, minlength=V), p[0], 4.0)[0]
    al, nodes = out["accept_len"], out["nodes"]
    for c in range(3):  # an accepted root candidate c: the next token ~ p at position c + 1
        sel = (al >= 2) & (nodes[:, 0] == c)
        assert sel.sum() > 5000
        assert within_sigma(np.bincount(out["tokens"][sel, 1], minlength=V), p[c + 1], 4.0)[0], c
    assert al.max() == 3  # depth-two tree: at most two accepted, then one drawn


def test_tree_errors(svo):
    zt = np.zeros((3, 3, 8), np.float32)
    zq = np.zeros((3, 2, 8), np.float32)
    tok = np.array([[1, 2], [1, 9], [1, 2]], np.int32)
    par = np.array([[0, 2], [0, 0], [0, 1]], np.int32)  # request 0: parent 2 > node index 1
    out = svo.verify_tree(zt, zq, tok, par, seed=1)
    assert out["flags"][0] == 1 << 11 and out["accept_len"][0] == -1
    assert out["flags"][1] & svo.FLAG_BAD_TOKEN and out["accept_len"][1] == -1
    assert out["accept_len"][2] >= 1
    # rows of leaves are never read: NaN there is fine
    zq2 = zq.copy()
    zq2[2, 1] = np.nan  # position 1 (node 0) has a child, position 2 (node 1) has none
    nt = np.array([2, 2, 1], np.int32)
    out2 = svo.verify_tree(zt, zq2, tok, par, n_nodes=nt, seed=1)
    assert out2["flags"][2] == 0


def test_the_first_matching_candidate_is_taken(svo):
    # three root candidates all holding the target's top token: greedy takes node 0
    zt = np.zeros((1, 4, 5), np.float32)
    zt[0, :, 3] = 2.0
    tok = np.array([[3, 3, 3]], np.int32)
    par = np.array([[0, 0, 0]], np.int32)
    out = svo.verify_tree(zt, None, tok, par, mode=svo.SVO_GREEDY)
    assert out["nodes"][0, 0] == 0 and out["accept_len"][0] == 2
    np.testing.assert_array_equal(out["tokens"][0], [3, 3, -1, -1])
