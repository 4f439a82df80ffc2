"""The verification step inside CUDA graphs (stream capture): a decode loop
captures its calls once and replays them, which saves each launch's host and
dependency overhead.  Captured calls (split path, every mode, with and without
the on-device epilogue) must reproduce the same calls made directly, call for
call; the workspace is passed explicitly, and one call is made before the
capture (the first call on a device does its one-time queries)."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _out(w):
    B, D = w.B, w.D_max
    return dict(tokens=torch.full((B, D + 1), -9, dtype=torch.int32, device="cuda"),
                accept_len=torch.full((B,), -9, dtype=torch.int32, device="cuda"),
                flags=torch.full((B,), -9, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("name,kw", [("tiny", dict(mode=0)), ("tiny", dict(mode=1)),
                                     ("tiny", dict(mode=2)), ("b32", dict(B=16, V=30011)),
                                     ("saguaro", dict(B=24, V=20008)),
                                     ("b256", dict(B=160, V=9001))])
def test_captured_calls_equal_direct_calls(sv, name, kw):
    w = wl.make(name, "cuda", **kw)
    ws = torch.empty(sv.sv_workspace_bytes(w.B, w.D_max, w.V, w.dtype), dtype=torch.uint8,
                     device="cuda")
    s = torch.cuda.Stream()
    seeds = [11, 12, 13, 14]
    outs = [_out(w) for _ in seeds]
    with torch.cuda.stream(s):
        sv.verify_workload(w, seed=0, out=_out(w), workspace=ws, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for sd, o in zip(seeds, outs):
            sv.verify_workload(w, seed=sd, out=o, workspace=ws, stream=s)
    for o in outs:  # nothing ran during the capture
        assert int(o["accept_len"][0]) == -9
    with torch.cuda.stream(s):
        g.replay()
        g.replay()  # replaying again gives the same results
    torch.cuda.synchronize()
    for sd, o in zip(seeds, outs):
        ref = sv.verify_workload(w, seed=sd)
        torch.cuda.synchronize()
        for k in ("tokens", "accept_len", "flags"):
            assert torch.equal(o[k], ref[k]), (name, sd, k)
    assert sv.sv_get_device_status() == 0


def test_captured_decode_loop_with_the_epilogue(sv):
    # three verification steps and their epilogues captured as one graph: each
    # step's emitted tokens go into the next window and onto the sequences, as
    # in a decode loop that never synchronises with the host
    w = wl.make("b32", "cuda", B=12, V=20011)
    B, D = w.B, w.D_max
    cap = 64
    ws = torch.empty(sv.sv_workspace_bytes(B, D, w.V, w.dtype), dtype=torch.uint8, device="cuda")
    window0 = torch.randint(0, w.V, (B, D + 1), dtype=torch.int32, device="cuda")
    seq0 = torch.full((B, cap), -1, dtype=torch.int32, device="cuda")
    len0 = torch.randint(0, 8, (B,), dtype=torch.int32, device="cuda")

    def run(capture):
        window = window0.clone()
        seq, seq_len = seq0.clone(), len0.clone()
        outs = [_out(w) for _ in range(3)]
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            sv.verify_workload(w, seed=0, out=_out(w), workspace=ws, stream=s)
        torch.cuda.synchronize()

        def steps():
            for i, o in enumerate(outs):
                sv.verify_workload(w, seed=40 + i, out=o, workspace=ws, stream=s,
                                   epilogue=dict(window=window, next_window=window, seq=seq,
                                                 seq_len=seq_len))
        if capture:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                steps()
            with torch.cuda.stream(s):
                g.replay()
        else:
            with torch.cuda.stream(s):
                steps()
        torch.cuda.synchronize()
        return window.cpu(), seq.cpu(), seq_len.cpu(), [o["accept_len"].cpu() for o in outs]

    a, b = run(True), run(False)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    for x, y in zip(a[3], b[3]):
        assert torch.equal(x, y)
    # the sequences grew by the accepted lengths of the three steps
    grown = sum(al.to(torch.int64) for al in b[3])
    assert torch.equal(b[2].to(torch.int64), len0.cpu().to(torch.int64) + grown)


@pytest.mark.parametrize("name,kw", [("tiny", dict(mode=1)), ("tiny", dict(mode=2)),
                                     ("b32", dict(B=16, V=30011)),
                                     ("saguaro", dict(B=24, V=20008))])
@pytest.mark.parametrize("variant", [sv.SV_VARIANT_AUTO,
                                     sv.SV_VARIANT_SPLIT | sv.SV_TAIL_PER_REQUEST,
                                     sv.SV_VARIANT_SPLIT | sv.SV_TAIL_ITEMS,
                                     sv.SV_VARIANT_FUSED, sv.SV_VARIANT_CLUSTER,
                                     sv.SV_VARIANT_EARLY_EXIT],
                         ids=["auto", "per-request", "items", "fused", "cluster", "early-exit"])
def test_seed_read_from_device_memory_equals_seed_argument(sv, name, kw, variant):
    w = wl.make(name, "cuda", **kw)
    for sd in (0, 7, 2**64 - 3):
        sdev = torch.tensor([sd - 2**64 if sd >= 2**63 else sd], dtype=torch.int64, device="cuda")
        got = sv.verify_workload(w, seed=12345, seed_device=sdev, variant=variant)
        ref = sv.verify_workload(w, seed=sd, variant=variant)
        torch.cuda.synchronize()
        for k in ("tokens", "accept_len", "flags"):
            assert torch.equal(got[k], ref[k]), (name, sd, k)


def test_tree_seed_read_from_device_memory(sv):
    w = wl.make_tree("tree", "cuda", B=20, V=12011, branching=(3, 2, 2))
    sdev = torch.tensor([99], dtype=torch.int64, device="cuda")
    args = (w.target, w.draft, w.tokens, w.parents)
    got = sv.verify_tree(*args, temperature=w.temperature, mode=w.mode, seed=5, seed_device=sdev)
    ref = sv.verify_tree(*args, temperature=w.temperature, mode=w.mode, seed=99)
    torch.cuda.synchronize()
    for k in ("tokens", "accept_len", "nodes", "flags"):
        assert torch.equal(got[k], ref[k]), k


def test_graph_replays_draw_new_numbers_with_an_advanced_seed(sv):
    # three steps captured once, each followed by seed += 1 on the device: the
    # first replay draws with seeds S, S+1, S+2, the second with S+3 .. S+5
    w = wl.make("b32", "cuda", B=16, V=30011)
    ws = torch.empty(sv.sv_workspace_bytes(w.B, w.D_max, w.V, w.dtype), dtype=torch.uint8,
                     device="cuda")
    S = 1000
    sdev = torch.tensor([S], dtype=torch.int64, device="cuda")
    s = torch.cuda.Stream()
    outs = [_out(w) for _ in range(3)]
    with torch.cuda.stream(s):
        sv.verify_workload(w, seed=0, out=_out(w), workspace=ws, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for o in outs:
            sv.verify_workload(w, out=o, workspace=ws, stream=s, seed_device=sdev)
            sv.sv_advance_seed(sdev, 1, stream=s)
    assert int(sdev.item()) == S  # nothing ran during the capture
    for rep in range(2):
        with torch.cuda.stream(s):
            g.replay()
        torch.cuda.synchronize()
        assert int(sdev.item()) == S + 3 * (rep + 1)
        for i, o in enumerate(outs):
            ref = sv.verify_workload(w, seed=S + 3 * rep + i)
            torch.cuda.synchronize()
            for k in ("tokens", "accept_len", "flags"):
                assert torch.equal(o[k], ref[k]), (rep, i, k)
    assert sv.sv_get_device_status() == 0
