"""Seeded synthetic inputs for the verification step.

This module holds no verification arithmetic: it only draws logits and draft
tokens with torch, so that the CUDA library and the CPU oracle can be fed the
same arrays.  The shapes and distributions are those of the five benchmark
workloads:

  tiny     B=1,   D=4,  V=1024,   fp32, target N(0,3^2), draft = target + N(0,1^2), T=1
  b32      B=32,  D=4,  V=128256, bf16, 1 of every 64 target rows peaked (+12 on one
           token, applied before the draft is made), draft = target + N(0,1^2), T=0.7
  b256     B=256, D=7,  V=128256, bf16, draft = target + N(0,0.75^2), T=1
  ragged   B=64,  D_b ~ U{1..8} padded to D_max=8, V=152064, bf16,
           draft = target + N(0,1.5^2); even requests greedy, odd stochastic at T=0.8;
           padding rows are NaN and padding tokens -1
  saguaro  B=128, D=4,  V=129280, bf16, draft = target + N(0,1^2), T=1, k=5, c=0.5

Normals are drawn in fp32; the draft is made from the fp32 target before both
are rounded (round-to-nearest-even) to the storage dtype.  Draft tokens are the
draft model's own samples: Gumbel-max over the stored draft logits at the
request's temperature (for saguaro the draft samples from its down-weighted
distribution, i.e. log c is added to its five largest logits first).  Greedy
requests take the draft's top token.  These draws are the draft model's, not
the verifier's; the verifier's random numbers come from its own counter-based
generator.
"""
import math
from dataclasses import dataclass, field
from typing import Optional

import torch

F32, BF16 = 0, 1
STOCHASTIC, GREEDY, SAGUARO = 0, 1, 2

CONFIGS = {
    "tiny": dict(B=1, D=4, V=1024, dtype=F32, target_sd=3.0, draft_sd=1.0, T=1.0,
                 mode=STOCHASTIC, seed=0),
    "b32": dict(B=32, D=4, V=128256, dtype=BF16, target_sd=3.0, draft_sd=1.0, T=0.7,
                mode=STOCHASTIC, seed=1001, peak_every=64, peak_boost=12.0),
    "b256": dict(B=256, D=7, V=128256, dtype=BF16, target_sd=3.0, draft_sd=0.75, T=1.0,
                 mode=STOCHASTIC, seed=1002),
    "ragged": dict(B=64, D=8, V=152064, dtype=BF16, target_sd=3.0, draft_sd=1.5, T=0.8,
                   mode=STOCHASTIC, seed=1003, ragged=True),
    "saguaro": dict(B=128, D=4, V=129280, dtype=BF16, target_sd=3.0, draft_sd=1.0, T=1.0,
                    mode=SAGUARO, seed=1004, saguaro_k=5, saguaro_c=0.5),
}


@dataclass
class Workload:
    name: str
    target: torch.Tensor            # [B, D_max+1, V] float32 or bfloat16
    draft: torch.Tensor             # [B, D_max, V]
    tokens: torch.Tensor            # [B, D_max] int32
    row_D: Optional[torch.Tensor]   # [B] int32 or None (= D_max for all)
    temperature: float
    mode: int
    dtype: int
    temperature_per_req: Optional[torch.Tensor] = None  # [B] float32
    mode_per_req: Optional[torch.Tensor] = None         # [B] int8
    saguaro_k: int = 5
    saguaro_c: float = 0.5
    seed: int = 0                   # the verifier's seed
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.target.shape[0]

    @property
    def D_max(self):
        return self.target.shape[1] - 1

    @property
    def V(self):
        return self.target.shape[2]

    def row_D_list(self):
        if self.row_D is None:
            return [self.D_max] * self.B
        return [int(v) for v in self.row_D.cpu().tolist()]

    def modes(self):
        if self.mode_per_req is None:
            return [self.mode] * self.B
        return [int(v) for v in self.mode_per_req.cpu().tolist()]

    def verified_rows(self):
        """sum over requests of D_b + 1 (the rows the target scored)."""
        return sum(d + 1 for d in self.row_D_list())

    def algorithmic_bytes(self):
        """Every needed logit row read once, plus one row per sampling request:
        sum_b [(D_b + 1) + D_b * stoch_b + stoch_b] * V * sizeof(dtype)."""
        s = 4 if self.dtype == F32 else 2
        rows = 0
        for d, m in zip(self.row_D_list(), self.modes()):
            stoch = 0 if m == GREEDY else 1
            rows += (d + 1) + d * stoch + stoch
        return rows * self.V * s

    def host_arrays(self):
        """numpy views for the oracle: fp32 as float32, bf16 as uint16 bits."""
        def np_logits(t):
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view("uint16")
            return t.numpy()
        out = dict(target=np_logits(self.target), draft=np_logits(self.draft),
                   tokens=self.tokens.cpu().numpy(),
                   row_D=None if self.row_D is None else self.row_D.cpu().numpy())
        out["temperature_per_req"] = (None if self.temperature_per_req is None
                                      else self.temperature_per_req.cpu().numpy())
        out["mode_per_req"] = (None if self.mode_per_req is None
                               else self.mode_per_req.cpu().numpy())
        return out


def _gumbel_argmax(logits: torch.Tensor, T, gen) -> torch.Tensor:
    """Draft sampling: argmax(z / T + Gumbel) along the last axis."""
    u = torch.rand(logits.shape, generator=gen, device=logits.device, dtype=torch.float32)
    u = u.clamp_(min=1e-20, max=1.0 - 1e-7)
    g = -torch.log(-torch.log(u))
    if not torch.is_tensor(T):
        T = torch.tensor(T, device=logits.device)
    return torch.argmax(logits.float() / T + g, dim=-1)


def make(name: str = "tiny", device="cpu", *, B=None, D=None, V=None, seed=None,
         verify_seed=0, dtype=None, T=None, mode=None, draft_sd=None,
         ragged=None, chunk_rows=64) -> Workload:
    """Build one workload.  Keyword overrides shrink a named configuration
    (same recipe, smaller sizes) for tests the oracle finishes in seconds."""
    cfg = dict(CONFIGS[name])
    if B is not None:
        cfg["B"] = B
    if D is not None:
        cfg["D"] = D
    if V is not None:
        cfg["V"] = V
    if seed is not None:
        cfg["seed"] = seed
    if dtype is not None:
        cfg["dtype"] = dtype
    if T is not None:
        cfg["T"] = T
    if mode is not None:
        cfg["mode"] = mode
    if draft_sd is not None:
        cfg["draft_sd"] = draft_sd
    if ragged is not None:
        cfg["ragged"] = ragged
    Bn, Dm, Vn = cfg["B"], cfg["D"], cfg["V"]
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg["seed"])
    store = torch.float32 if cfg["dtype"] == F32 else torch.bfloat16

    target = torch.empty((Bn, Dm + 1, Vn), dtype=store, device=device)
    draft = torch.empty((Bn, max(Dm, 0), Vn), dtype=store, device=device)
    # draw in slabs of requests to bound the fp32 temporaries
    for b0 in range(0, Bn, chunk_rows):
        b1 = min(Bn, b0 + chunk_rows)
        zt = torch.randn((b1 - b0, Dm + 1, Vn), generator=gen, device=device) * cfg["target_sd"]
        if cfg.get("peak_every"):
            # rows whose global index r = b*(D+1) + d is a multiple of peak_every
            # get +boost on one token drawn uniformly
            for b in range(b0, b1):
                for d in range(Dm + 1):
                    r = b * (Dm + 1) + d
                    if r % cfg["peak_every"] == 0:
                        x = int(torch.randint(0, Vn, (1,), generator=gen, device=device).item())
                        zt[b - b0, d, x] += cfg["peak_boost"]
        if Dm > 0:
            zq = zt[:, :Dm, :] + torch.randn((b1 - b0, Dm, Vn), generator=gen,
                                             device=device) * cfg["draft_sd"]
            draft[b0:b1] = zq.to(store)
            del zq
        target[b0:b1] = zt.to(store)
        del zt

    # request modes and temperatures
    mode_per_req = None
    temperature_per_req = None
    row_D = None
    if cfg.get("ragged"):
        row_D = torch.randint(1, Dm + 1, (Bn,), generator=gen, device=device).to(torch.int32)
        mode_per_req = torch.tensor([GREEDY if b % 2 == 0 else STOCHASTIC for b in range(Bn)],
                                    dtype=torch.int8, device=device)
        temperature_per_req = torch.full((Bn,), cfg["T"], dtype=torch.float32, device=device)
    modes = ([int(m) for m in mode_per_req.tolist()] if mode_per_req is not None
             else [cfg["mode"]] * Bn)

    # draft tokens: the draft model's own samples
    tokens = torch.full((Bn, Dm), -1, dtype=torch.int32, device=device)
    if Dm > 0:
        zq = draft.float()
        if cfg["mode"] == SAGUARO or any(m == SAGUARO for m in modes):
            k = min(cfg.get("saguaro_k", 5), Vn)
            c = cfg.get("saguaro_c", 0.5)
            # the k largest draft logits, lowest index first among equal values
            top = torch.sort(zq, dim=-1, descending=True, stable=True).indices[..., :k]
            adj = torch.zeros_like(zq)
            adj.scatter_(-1, top, torch.full(top.shape, math.log(c) * cfg["T"],
                                             dtype=adj.dtype, device=adj.device))
            zq_s = zq + adj      # divided by T inside the sampler: adds log c
        else:
            zq_s = zq
        sampled = _gumbel_argmax(zq_s, cfg["T"], gen).to(torch.int32)
        top1 = torch.argmax(zq, dim=-1).to(torch.int32)
        for b in range(Bn):
            tokens[b] = top1[b] if modes[b] == GREEDY else sampled[b]
        del zq

    # padding rows and tokens beyond each request's draft length
    if row_D is not None:
        for b, d_b in enumerate(row_D.tolist()):
            target[b, d_b + 1:, :] = float("nan")
            draft[b, d_b:, :] = float("nan")
            tokens[b, d_b:] = -1

    return Workload(
        name=name, target=target, draft=draft, tokens=tokens, row_D=row_D,
        temperature=float(cfg["T"]), mode=int(cfg["mode"]), dtype=int(cfg["dtype"]),
        temperature_per_req=temperature_per_req, mode_per_req=mode_per_req,
        saguaro_k=int(cfg.get("saguaro_k", 5)), saguaro_c=float(cfg.get("saguaro_c", 0.5)),
        seed=int(verify_seed), meta=dict(cfg),
    )


# ---- draft trees

TREE_CONFIGS = {
    # B requests, a draft tree with `branching[k]` candidates under every node of
    # depth k (breadth-first node order), V, bf16; target N(0, 3^2) at every
    # position, draft = target + N(0, 1^2); candidates are independent draws
    # from the draft at their parent position (Gumbel-max at T)
    "tree": dict(B=64, branching=(3, 2, 2), V=128256, dtype=BF16, target_sd=3.0, draft_sd=1.0,
                 T=1.0, seed=1005),
}


@dataclass
class TreeWorkload:
    name: str
    target: torch.Tensor     # [B, N+1, V]
    draft: torch.Tensor      # [B, N, V]
    tokens: torch.Tensor     # [B, N] int32
    parents: torch.Tensor    # [B, N] int32, parent position in [0, i]
    temperature: float
    mode: int
    dtype: int
    seed: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.target.shape[0]

    @property
    def N(self):
        return self.target.shape[1] - 1

    @property
    def D_max(self):
        return self.N

    @property
    def V(self):
        return self.target.shape[2]

    def parent_list(self):
        return [int(v) for v in self.parents[0].cpu().tolist()]

    def verified_rows(self):
        """Candidates tested per call: every node of every request, plus the row
        the final token is drawn from."""
        return self.B * (self.N + 1)

    def algorithmic_bytes(self):
        """Every target row and every draft row with candidates read once, plus
        one row pair per request for the residual sums and the race."""
        s = 4 if self.dtype == F32 else 2
        with_child = len(set(self.parent_list()))
        rows = (self.N + 1) + (0 if self.mode == GREEDY else with_child)
        extra = 0 if self.mode == GREEDY else 2
        return self.B * (rows + extra) * self.V * s


def tree_parents(branching):
    """Parent positions of a breadth-first tree: branching[k] children under
    every node of depth k (the root has depth 0)."""
    parents, level = [], [0]
    for k in branching:
        nxt = []
        for pos in level:
            for _ in range(k):
                parents.append(pos)
                nxt.append(len(parents))  # the new node's position
        level = nxt
    return parents


def make_tree(name="tree", device="cpu", *, B=None, V=None, branching=None, seed=None,
              mode=STOCHASTIC, dtype=None, T=None, chunk_rows=16) -> TreeWorkload:
    cfg = dict(TREE_CONFIGS[name])
    for k, v in (("B", B), ("V", V), ("branching", branching), ("seed", seed), ("dtype", dtype),
                 ("T", T)):
        if v is not None:
            cfg[k] = v
    parents = tree_parents(cfg["branching"])
    Bn, N, Vn = cfg["B"], len(parents), cfg["V"]
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg["seed"])
    store = torch.float32 if cfg["dtype"] == F32 else torch.bfloat16
    target = torch.empty((Bn, N + 1, Vn), dtype=store, device=device)
    draft = torch.empty((Bn, N, Vn), dtype=store, device=device)
    tokens = torch.empty((Bn, N), dtype=torch.int32, device=device)
    par = torch.tensor(parents, dtype=torch.long, device=device)
    for b0 in range(0, Bn, chunk_rows):
        b1 = min(Bn, b0 + chunk_rows)
        zt = torch.randn((b1 - b0, N + 1, Vn), generator=gen, device=device) * cfg["target_sd"]
        zq = zt[:, :N] + torch.randn((b1 - b0, N, Vn), generator=gen, device=device) * cfg["draft_sd"]
        target[b0:b1] = zt.to(store)
        draft[b0:b1] = zq.to(store)
        # node i's token: an independent draw from the draft at its parent position
        zp = draft[b0:b1].float()[:, par, :]
        tokens[b0:b1] = _gumbel_argmax(zp, cfg["T"], gen).to(torch.int32)
        del zt, zq, zp
    if mode == GREEDY:
        # greedy drafting: each node's candidates are the draft's top tokens at its parent
        # position, distinct, best first (the i-th child of a position takes the i-th best)
        rank = {}
        for i, p in enumerate(parents):
            rank[i] = sum(1 for j in range(i) if parents[j] == p)
        kmax = max(rank.values()) + 1
        top = torch.topk(draft.float(), kmax, dim=-1).indices  # [B, N, kmax]
        for i, p in enumerate(parents):
            tokens[:, i] = top[:, p, rank[i]].to(torch.int32)
    parents_t = torch.tensor(parents, dtype=torch.int32, device=device).repeat(Bn, 1).contiguous()
    return TreeWorkload(name=name, target=target, draft=draft, tokens=tokens, parents=parents_t,
                        temperature=float(cfg["T"]), mode=int(mode), dtype=int(cfg["dtype"]),
                        seed=0, meta=dict(cfg, N=N))
