"""Request sharding across ranks (one process per GPU).

Requests are independent: the rule reads only a request's own rows, and its
random numbers are keyed by the request's GLOBAL index.  A batch of B requests
therefore splits into contiguous slices, one per rank, each verified with
request_offset = the slice's first global index, and the concatenated outputs
equal those of one call over the whole batch.  There is no exchange on the data
path; the only collective is the timing reduction (max over ranks).
"""


def shard_range(B: int, world: int, rank: int):
    """[start, stop) of rank's contiguous slice of B requests (sizes differ by <= 1)."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks of the default process group (the
    step time every rank waits for); the value itself without one."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---- vocabulary sharding (tensor-parallel logits), sv_shard_* in the C ABI

def vocab_shard_width(V: int, world: int) -> int:
    """Columns per rank when V is split over `world` ranks: the ceiling of
    V / world rounded up to a multiple of 4 (the race's four-token blocks).
    The last rank's columns past V hold -inf (masked tokens)."""
    if world < 1 or V < 1:
        raise ValueError(f"bad split of V={V} over {world}")
    w = -(-V // world)
    return -(-w // 4) * 4


def vocab_shard(t, rank: int, world: int):
    """Rank's columns of logits t [..., V] as a contiguous [..., V_local] tensor,
    padded with -inf past V."""
    import torch
    V = t.shape[-1]
    Vl = vocab_shard_width(V, world)
    v0, v1 = rank * Vl, min(V, (rank + 1) * Vl)
    out = torch.full(t.shape[:-1] + (Vl,), float("-inf"), dtype=t.dtype, device=t.device)
    if v1 > v0:
        out[..., : v1 - v0] = t[..., v0:v1]
    return out.contiguous()


def all_gather_bytes(buf, group=None):
    """All-gather of one byte buffer per rank, in rank order (NCCL for CUDA
    tensors, gloo for CPU ones)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world * buf.numel(),), dtype=buf.dtype, device=buf.device)
    dist.all_gather_into_tensor(out, buf, group=group)
    return out


class VocabShardCall:
    """One rank's part of a vocabulary-sharded verification, stage by stage:
    stage1() -> this rank's exchange 1; stage2(gathered1) -> exchange 2;
    stage3(gathered2) -> the outputs (the same dict as verify()).  The
    gathered buffers are every rank's exchange concatenated in rank order."""

    def __init__(self, target_local, draft_local, tokens, row_D=None, *, n_shards, shard,
                 temperature=1.0, mode=0, seed=0, temperature_per_req=None, mode_per_req=None,
                 saguaro_k=5, saguaro_c=0.5, request_offset=0, stream=None, row_lse=False,
                 draft_top=False, seed_device=None):
        import torch
        from . import (SvParams, _dtype_code, _p, _seed_device_ptr, _stream_ptr,
                       sv_shard_exchange_bytes)
        B, Dp1, Vl = target_local.shape
        D = Dp1 - 1
        dt = _dtype_code(target_local)
        dev = target_local.device
        prm = SvParams()
        prm.stream = _stream_ptr(stream)
        prm.temperature_per_req = _p(temperature_per_req)
        prm.mode_per_req = _p(mode_per_req)
        prm.saguaro_k = int(saguaro_k)
        prm.saguaro_c = float(saguaro_c)
        prm.request_offset = int(request_offset)
        prm.seed_device = _seed_device_ptr(seed_device)
        out = dict(tokens=torch.empty((B, D + 1), dtype=torch.int32, device=dev),
                   accept_len=torch.empty((B,), dtype=torch.int32, device=dev),
                   flags=torch.empty((B,), dtype=torch.int32, device=dev))
        if row_lse:
            out["row_lse"] = torch.empty((B, 2 * D + 1), dtype=torch.float32, device=dev)
        if draft_top:
            k = int(saguaro_k) if int(saguaro_k) > 0 else 5
            out["draft_top"] = torch.empty((B, D, min(k, n_shards * Vl)), dtype=torch.int32,
                                           device=dev)
        prm.out_flags = _p(out["flags"])
        prm.out_row_lse = _p(out.get("row_lse"))
        prm.out_draft_top = _p(out.get("draft_top"))
        self.prm, self.out, self.dev, self.B, self.D, self.n = prm, out, dev, B, D, int(n_shards)
        self.x1 = torch.empty((sv_shard_exchange_bytes(B, D, Vl, dt, 1),), dtype=torch.uint8,
                              device=dev)
        self.x2 = torch.empty((sv_shard_exchange_bytes(B, D, Vl, dt, 2),), dtype=torch.uint8,
                              device=dev)
        self.args = (target_local, draft_local, tokens, row_D, B, D, Vl, dt, float(temperature),
                     int(mode), int(seed), int(n_shards), int(shard), prm)

    def stage1(self):
        import torch
        from . import _check, sv_shard_stats
        with torch.cuda.device(self.dev):
            _check(sv_shard_stats(*self.args, self.x1))
        return self.x1

    def stage2(self, gathered1):
        import torch
        from . import _check, sv_shard_race
        with torch.cuda.device(self.dev):
            _check(sv_shard_race(*self.args, gathered1, self.out["tokens"], self.out["accept_len"],
                                 self.x2))
        return self.x2

    def stage3(self, gathered2):
        import torch
        from . import _check, sv_shard_finish
        with torch.cuda.device(self.dev):
            _check(sv_shard_finish(self.B, self.D, self.n, gathered2, self.out["tokens"], self.prm))
        return self.out


def verify_vocab_parallel(target_local, draft_local, tokens, row_D=None, *, n_shards, shard,
                          gather=all_gather_bytes, **kw):
    """Verification of a batch whose logits are split by vocabulary: this rank
    holds target_local [B, D_max+1, V_local] and draft_local [B, D_max, V_local]
    (columns [shard V_local, (shard + 1) V_local)); tokens are global.
    gather(byte_tensor) returns every rank's buffer concatenated in rank order
    (all_gather_bytes over the default process group by default).  Returns the
    same dict as verify(); every rank gets the same outputs."""
    call = VocabShardCall(target_local, draft_local, tokens, row_D, n_shards=n_shards,
                          shard=shard, **kw)
    g1 = gather(call.stage1())
    g2 = gather(call.stage2(g1))
    return call.stage3(g2)


def verify_vocab_parallel_in_one_process(target, draft, tokens, row_D=None, *, n_shards, **kw):
    """The same computation with every shard in this process (on one device,
    in turn): shard the full logits, run each stage for every shard, and stand
    in for the all-gathers with concatenation.  Returns the outputs of every
    shard (they are equal)."""
    import torch
    calls = [VocabShardCall(vocab_shard(target, r, n_shards),
                            None if draft is None else vocab_shard(draft, r, n_shards),
                            tokens, row_D, n_shards=n_shards, shard=r, **kw)
             for r in range(n_shards)]
    g1 = torch.cat([c.stage1() for c in calls])
    g2 = torch.cat([c.stage2(g1) for c in calls])
    return [c.stage3(g2) for c in calls]
