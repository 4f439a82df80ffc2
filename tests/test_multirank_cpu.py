"""The N > 1 path on the CPU: world size 2 over gloo.

Requests shard by contiguous slices with the slice's first global index as
request offset; every rank verifies its slice (here with the oracle, as no GPU
is present), the slices are gathered, and the result must equal one call over
the whole batch.  The timing reduction (max over ranks) is checked too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_verification_lse_b200.sharding import max_over_ranks, shard_range


def test_shard_ranges_cover_the_batch():
    for B in (0, 1, 5, 256, 257):
        for world in (1, 2, 3, 8):
            spans = [shard_range(B, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    from speculative_decoding_verification_lse_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.make("ragged", "cpu", B=10, V=3001)  # same seed on every rank
        h = w.host_arrays()
        b0, b1 = shard_range(w.B, world, rank)
        sl = slice(b0, b1)
        res = oracle.verify(h["target"][sl], h["draft"][sl], h["tokens"][sl], h["row_D"][sl],
                            temperature=w.temperature, mode=w.mode, seed=77,
                            temperature_per_req=h["temperature_per_req"][sl],
                            mode_per_req=h["mode_per_req"][sl], request_offset=b0)
        mine = torch.from_numpy(np.concatenate(
            [res["tokens"], res["accept_len"][:, None], res["flags"].astype(np.int32)[:, None]],
            axis=1)).to(torch.int64)
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([mine.shape[0]]))
        parts = [torch.zeros((int(s.item()), mine.shape[1]), dtype=torch.int64) for s in sizes]
        dist.all_gather(parts, mine)
        # the step time every rank waits for
        t = max_over_ranks(1.0 + rank)
        if rank == 0:
            full = oracle.verify(h["target"], h["draft"], h["tokens"], h["row_D"],
                                 temperature=w.temperature, mode=w.mode, seed=77,
                                 temperature_per_req=h["temperature_per_req"],
                                 mode_per_req=h["mode_per_req"])
            ref = np.concatenate([full["tokens"], full["accept_len"][:, None],
                                  full["flags"].astype(np.int32)[:, None]], axis=1)
            got = torch.cat(parts).numpy()
            np.save(os.path.join(out_dir, "ok.npy"),
                    np.array([np.array_equal(got, ref), t == float(world)]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_single_batch(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    ok = np.load(tmp_path / "ok.npy")
    assert ok[0], "sharded outputs differ from the single-batch outputs"
    assert ok[1], "max over ranks is wrong"


def _vocab_rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from speculative_decoding_verification_lse_b200.sharding import (all_gather_bytes, vocab_shard,
                                                                    vocab_shard_width)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(5)
        V = 1003
        rows = torch.randn((4, V), generator=g) * 3  # the same on every rank
        mine = vocab_shard(rows, rank, world)
        Vl = vocab_shard_width(V, world)
        # one exchange: this rank's partial (max, sum of exp) per row and its columns
        m = mine.max(dim=-1).values
        s = torch.exp(mine - m[:, None]).sum(dim=-1)
        rec = torch.cat([m[:, None], s[:, None], mine], dim=1).contiguous()
        got = all_gather_bytes(rec.view(torch.uint8).flatten())
        parts = got.view(world, -1).view(torch.float32).view(world, 4, Vl + 2)
        if rank == 0:
            cols = torch.cat([parts[r, :, 2:] for r in range(world)], dim=1)[:, :V]
            # the partials merged in rank order give the whole row's log-sum-exp
            M = parts[:, :, 0].max(dim=0).values
            S = (parts[:, :, 1] * torch.exp(parts[:, :, 0] - M[None])).sum(dim=0)
            lse = (M + torch.log(S)).double()
            want = torch.logsumexp(rows.double(), dim=-1)
            np.save(os.path.join(out_dir, "vocab_ok.npy"),
                    np.array([torch.equal(cols, rows),
                              bool(torch.allclose(lse, want, rtol=1e-6, atol=1e-6))]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_the_vocabulary(tmp_path):
    """The host side of vocabulary-parallel verification over gloo: each rank
    cuts its columns (vocab_shard), the byte exchange (all_gather_bytes)
    returns every rank's buffer in rank order, and partial (max, sum) pairs
    merged in that order give the whole row's log-sum-exp."""
    world = 2
    mp.start_processes(_vocab_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    ok = np.load(tmp_path / "vocab_ok.npy")
    assert ok[0], "gathered columns are out of rank order"
    assert ok[1], "merged partials differ from the row's log-sum-exp"
