"""Pins for the oracle's epilogue (svo_epilogue): the step after verification
that builds the next run's shifted input window and appends the emitted tokens
to each request's sequence ("Accélérer Sonar par la Spéculation", section
"Calendrier MTP pour un jeton unique").  Pinned by a worked example written out
by hand, by the properties the section fixes (the emitted tokens occupy the
first AL slots of the shifted window; the sequence grows by AL), and by a toy
autoregressive chain in which repeated verify + epilogue steps reproduce plain
argmax decoding token for token."""
import numpy as np
import pytest


def test_worked_example(svo):
    # request 0: window [7 | 10 11 12], two accepted drafts would be AL=3;
    #   here AL=2: draft 10 accepted, 55 emitted at slot 1
    # request 1: all three drafts accepted (AL=4), bonus 99 at slot 3
    # request 2: first draft rejected (AL=1), correction 40 at slot 0
    # request 3: flagged by the verification (AL=-1)
    window = np.array([[7, 10, 11, 12], [8, 20, 21, 22], [9, 30, 31, 32], [6, 1, 2, 3]], np.int32)
    out = np.array([[10, 55, -1, -1], [20, 21, 22, 99], [40, -1, -1, -1], [-1, -1, -1, -1]],
                   np.int32)
    AL = np.array([2, 4, 1, -1], np.int32)
    seq = np.full((4, 6), -5, np.int32)
    seq_len = np.array([1, 2, 6, 0], np.int32)
    r = svo.epilogue(window, out, AL, seq, seq_len)
    np.testing.assert_array_equal(r["next_window"], [[10, 55, 12, -1],
                                                      [20, 21, 22, 99],
                                                      [40, 31, 32, -1],
                                                      [-1, -1, -1, -1]])
    np.testing.assert_array_equal(r["seq_len"], [3, 6, 6, 0])
    np.testing.assert_array_equal(r["seq"], [[-5, 10, 55, -5, -5, -5],
                                             [-5, -5, 20, 21, 22, 99],
                                             [-5, -5, -5, -5, -5, -5],  # 6 + 1 > 6: no room
                                             [-5, -5, -5, -5, -5, -5]])
    np.testing.assert_array_equal(r["full"], [False, False, True, False])


def test_properties_on_random_steps(svo):
    rng = np.random.default_rng(3)
    B, D = 40, 6
    W = D + 1
    for _ in range(20):
        window = rng.integers(0, 1000, (B, W)).astype(np.int32)
        AL = rng.integers(1, W + 1, B).astype(np.int32)
        out = np.full((B, W), -1, np.int32)
        for b in range(B):
            n = AL[b] - 1
            out[b, :n] = window[b, 1:n + 1]          # accepted drafts
            out[b, n] = rng.integers(0, 1000)        # the emitted token
        seq_len = rng.integers(0, 30, B).astype(np.int32)
        seq = rng.integers(0, 1000, (B, 40)).astype(np.int32)
        r = svo.epilogue(window, out, AL, seq, seq_len)
        for b in range(B):
            n = AL[b] - 1
            np.testing.assert_array_equal(r["next_window"][b, :n + 1], out[b, :n + 1])
            np.testing.assert_array_equal(r["next_window"][b, n + 1:D], window[b, n + 2:])
            if n < D:
                assert r["next_window"][b, D] == -1
            assert r["seq_len"][b] == seq_len[b] + AL[b]
            np.testing.assert_array_equal(r["seq"][b, seq_len[b]:seq_len[b] + AL[b]], out[b, :AL[b]])
            np.testing.assert_array_equal(r["seq"][b, :seq_len[b]], seq[b, :seq_len[b]])
            np.testing.assert_array_equal(r["seq"][b, seq_len[b] + AL[b]:], seq[b, seq_len[b] + AL[b]:])


def test_out_of_range_lengths_are_errors(svo):
    window = np.arange(8, dtype=np.int32).reshape(2, 4)
    out = np.arange(8, dtype=np.int32).reshape(2, 4)
    for bad in (0, -1, 5):
        r = svo.epilogue(window, out, np.array([bad, 2], np.int32), np.zeros((2, 8), np.int32),
                         np.array([0, 0], np.int32))
        assert np.all(r["next_window"][0] == -1) and r["seq_len"][0] == 0
        assert r["seq_len"][1] == 2


def test_greedy_chain_with_epilogue_reproduces_argmax_decoding(svo):
    """A toy bigram target (row t of Tt = logits after token t) and a bigram
    draft Qt; each step verifies the window [last, drafts], the epilogue appends
    the emitted tokens and shifts the window, and the next window starts with
    the token the epilogue inserted at slot n.  The sequence equals plain argmax
    decoding of Tt."""
    rng = np.random.default_rng(21)
    V, D, steps = 50, 4, 25
    Tt = (rng.standard_normal((V, V)) * 1.5).astype(np.float32)
    Qt = (Tt + rng.standard_normal((V, V)) * 0.9).astype(np.float32)
    start = 3
    ref, last = [start], start
    for _ in range(steps * (D + 1)):
        last = int(np.argmax(Tt[last]))
        ref.append(last)
    seq = np.full((1, 400), -1, np.int32)
    seq[0, 0] = start
    seq_len = np.array([1], np.int32)
    last = start
    for _ in range(steps):
        drafts, p = [], last
        for _ in range(D):
            p = int(np.argmax(Qt[p]))
            drafts.append(p)
        window = np.array([[last] + drafts], np.int32)
        out = svo.verify(Tt[window[0]][None], None, window[:, 1:], mode=svo.SVO_GREEDY)
        r = svo.epilogue(window, out["tokens"], out["accept_len"], seq, seq_len)
        seq, seq_len = r["seq"], r["seq_len"]
        n = int(out["accept_len"][0]) - 1
        last = int(r["next_window"][0, n])
    L = int(seq_len[0])
    assert L > steps  # several tokens per step on average
    assert list(seq[0, :L]) == ref[:L]
