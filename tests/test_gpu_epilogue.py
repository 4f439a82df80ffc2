"""The on-device epilogue (sv_epilogue, and sv_verify_ex with sv_params.epilogue)
against the oracle's host epilogue, element by element: the shifted window
with the emitted target token inserted, the append to each request's sequence,
the capacity flag, rows of requests the verification flagged, in place and not;
and a decoding loop of several steps that never synchronises with the host
(verify, epilogue, next window and drafts all on the device) reproducing the
oracle's loop token for token."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _random_case(rng, B, D, cap):
    W = D + 1
    window = rng.integers(0, 50000, (B, W)).astype(np.int32)
    AL = rng.integers(1, W + 1, B).astype(np.int32)
    out = np.full((B, W), -1, np.int32)
    for b in range(B):
        n = AL[b] - 1
        out[b, :n] = window[b, 1:n + 1]
        out[b, n] = rng.integers(0, 50000)
    # some requests the verification flagged, some lengths out of range
    bad = rng.choice(B, max(1, B // 10), replace=False)
    AL[bad[: len(bad) // 2 + 1]] = -1
    out[bad[: len(bad) // 2 + 1]] = -1
    AL[bad[len(bad) // 2 + 1:]] = W + 3
    seq_len = rng.integers(0, cap, B).astype(np.int32)
    seq_len[rng.choice(B, max(1, B // 8), replace=False)] = cap - 1  # most of these overflow
    seq = rng.integers(0, 50000, (B, cap)).astype(np.int32)
    return window, out, AL, seq, seq_len


@pytest.mark.parametrize("B,D,cap", [(1, 0, 4), (37, 4, 16), (300, 7, 64), (65, 32, 100)])
@pytest.mark.parametrize("in_place", [False, True], ids=["copy", "in-place"])
def test_epilogue_matches_the_oracle(sv, B, D, cap, in_place):
    rng = np.random.default_rng(B * 100 + D)
    window, out, AL, seq, seq_len = _random_case(rng, B, D, cap)
    ref = oracle.epilogue(window, out, AL, seq, seq_len)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    d_win, d_out, d_al, d_seq, d_len = map(dev, (window, out, AL, seq, seq_len))
    d_next = d_win if in_place else torch.full_like(d_win, -7)
    d_flags = torch.zeros(B, dtype=torch.int32, device="cuda")
    rc = sv.sv_epilogue(d_win, d_out, d_al, B, D, d_next, d_seq, cap, d_len, d_flags)
    assert rc == sv.SV_OK, sv.sv_last_error()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(d_next.cpu().numpy(), ref["next_window"])
    np.testing.assert_array_equal(d_seq.cpu().numpy(), ref["seq"])
    np.testing.assert_array_equal(d_len.cpu().numpy(), ref["seq_len"])
    full = (d_flags.cpu().numpy() & sv.SV_FLAG_SEQ_FULL) != 0
    np.testing.assert_array_equal(full, ref["full"])
    status = sv.sv_get_device_status()
    assert bool(status & sv.SV_STATUS_SEQ_FULL) == bool(ref["full"].any())


def test_epilogue_parts_are_optional(sv):
    rng = np.random.default_rng(5)
    window, out, AL, seq, seq_len = _random_case(rng, 20, 5, 32)
    ref = oracle.epilogue(window, out, AL, seq, seq_len)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    # the window only
    d_next = torch.full((20, 6), -7, dtype=torch.int32, device="cuda")
    assert sv.sv_epilogue(dev(window), dev(out), dev(AL), 20, 5, d_next, None, 0, None) == sv.SV_OK
    # the append only
    d_seq, d_len = dev(seq), dev(seq_len)
    assert sv.sv_epilogue(None, dev(out), dev(AL), 20, 5, None, d_seq, 32, d_len) == sv.SV_OK
    torch.cuda.synchronize()
    np.testing.assert_array_equal(d_next.cpu().numpy(), ref["next_window"])
    np.testing.assert_array_equal(d_seq.cpu().numpy(), ref["seq"])
    np.testing.assert_array_equal(d_len.cpu().numpy(), ref["seq_len"])
    sv.sv_get_device_status()


@pytest.mark.parametrize("variant", [sv.SV_VARIANT_SPLIT, sv.SV_VARIANT_FUSED], ids=["split", "fused"])
@pytest.mark.parametrize("name", ["b256", "ragged"])
def test_verify_with_epilogue_matches_the_oracle(sv, name, variant):
    """sv_verify_ex with sv_params.epilogue: the verification's own outputs feed
    the epilogue on the same stream; compared with the oracle's epilogue applied
    to the library's verification outputs (the verification itself is checked
    against the oracle by the parity tests)."""
    w = wl.make(name, "cuda", B=24, V=40013)
    B, D = w.B, w.D_max
    rng = np.random.default_rng(9)
    last = rng.integers(0, w.V, (B, 1)).astype(np.int32)
    window = np.concatenate([last, w.tokens.cpu().numpy()], axis=1).astype(np.int32)
    cap = 64
    seq = rng.integers(0, w.V, (B, cap)).astype(np.int32)
    seq_len = rng.integers(0, cap - D, B).astype(np.int32)
    d_win = torch.from_numpy(window).cuda()
    d_next = torch.full_like(d_win, -7)
    d_seq = torch.from_numpy(seq).cuda()
    d_len = torch.from_numpy(seq_len).cuda()
    got = sv.verify_workload(w, variant=variant,
                             epilogue=dict(window=d_win, next_window=d_next, seq=d_seq, seq_len=d_len))
    torch.cuda.synchronize()
    toks, al = got["tokens"].cpu().numpy(), got["accept_len"].cpu().numpy()
    ref = oracle.epilogue(window, toks, al, seq, seq_len)
    np.testing.assert_array_equal(d_next.cpu().numpy(), ref["next_window"])
    np.testing.assert_array_equal(d_seq.cpu().numpy(), ref["seq"])
    np.testing.assert_array_equal(d_len.cpu().numpy(), ref["seq_len"])
    assert sv.sv_get_device_status() & sv.SV_FLAG_ERRORS == 0


def test_decoding_loop_without_host_sync_matches_the_oracle(sv):
    """A toy bigram target and draft (row t of a table = the logits after token
    t): each step builds the target and draft logits by gathering table rows at
    the window's tokens, drafts greedily from the draft table, verifies
    (stochastic, T = 1) with the epilogue, and takes the next window's first
    token from the slot the epilogue filled -- every step on the device, with no
    synchronisation.  The oracle runs the same loop on the host; the sequences
    agree token for token (the requests the oracle flags as near-ties at any
    step, where several results are correct, are left out of the comparison)."""
    rng = np.random.default_rng(33)
    B, D, V, steps, cap = 64, 4, 3001, 12, 128
    Tt = (rng.standard_normal((V, V)) * 2.5).astype(np.float32)
    Qt = (Tt + rng.standard_normal((V, V)) * 0.8).astype(np.float32)
    start = rng.integers(0, V, B).astype(np.int32)

    # device loop
    dT, dQ = torch.from_numpy(Tt).cuda(), torch.from_numpy(Qt).cuda()
    last = torch.from_numpy(start).cuda()
    seq = torch.full((B, cap), -1, dtype=torch.int32, device="cuda")
    seq[:, 0] = last
    seq_len = torch.ones(B, dtype=torch.int32, device="cuda")
    flags_any = torch.zeros(B, dtype=torch.int32, device="cuda")
    ar = torch.arange(B, device="cuda")
    for step in range(steps):
        drafts, p = [], last.long()
        for _ in range(D):
            p = torch.argmax(dQ[p], dim=-1)
            drafts.append(p)
        dr = torch.stack(drafts, 1).to(torch.int32)
        window = torch.cat([last[:, None], dr], 1).contiguous()
        target = dT[window.long()].contiguous()              # [B, D+1, V]
        draft = dQ[window[:, :D].long()].contiguous()         # [B, D, V]
        nxt = torch.empty_like(window)
        out = sv.verify(target, draft, dr.contiguous(), seed=100 + step,
                        epilogue=dict(window=window, next_window=nxt, seq=seq, seq_len=seq_len))
        flags_any |= out["flags"]
        last = nxt[ar, (out["accept_len"] - 1).long()].contiguous()
    torch.cuda.synchronize()
    g_seq, g_len = seq.cpu().numpy(), seq_len.cpu().numpy()

    # host loop (the oracle)
    h_seq = np.full((B, cap), -1, np.int32)
    h_seq[:, 0] = start
    h_len = np.ones(B, np.int32)
    h_last = start.copy()
    h_flags = np.zeros(B, np.uint32)
    for step in range(steps):
        dr = np.zeros((B, D), np.int32)
        p = h_last.copy()
        for d in range(D):
            p = np.argmax(Qt[p], axis=-1).astype(np.int32)
            dr[:, d] = p
        window = np.concatenate([h_last[:, None], dr], 1).astype(np.int32)
        o = oracle.verify(Tt[window], Qt[window[:, :D]], dr, seed=100 + step, nthreads=8)
        h_flags |= o["flags"]
        r = oracle.epilogue(window, o["tokens"], o["accept_len"], h_seq, h_len)
        h_seq, h_len = r["seq"], r["seq_len"]
        h_last = r["next_window"][np.arange(B), o["accept_len"] - 1]
    clean = (h_flags & oracle.FLAG_NEAR_TIE) == 0
    assert clean.sum() >= B - 2
    assert np.all(g_len >= steps)
    np.testing.assert_array_equal(g_len[clean], h_len[clean])
    np.testing.assert_array_equal(g_seq[clean], h_seq[clean])
    assert (g_seq[:, 0] == start).all()
