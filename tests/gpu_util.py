"""Helpers for the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare them element by element."""
import math

import numpy as np
import torch

import oracle
import speculative_decoding_verification_lse_b200 as sv

LSE_TOL = {sv.SV_F32: 1e-5, sv.SV_BF16: 1e-3}  # relative, as specified


def host_logits(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def gpu_run(w, **kw):
    out = sv.verify_workload(w, row_lse=True, **kw)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def oracle_on(w, reqs=None, seed=None, nthreads=8):
    """Oracle outputs for the requests `reqs` (all when None), each run with its
    global index as request offset, so any subset is checked exactly."""
    B = w.B
    reqs = list(range(B)) if reqs is None else sorted(reqs)
    # contiguous runs of requests -> one oracle call each
    runs, start = [], None
    for i, b in enumerate(reqs):
        if start is None:
            start = b
        if i + 1 == len(reqs) or reqs[i + 1] != b + 1:
            runs.append((start, b + 1))
            start = None
    parts = []
    for b0, b1 in runs:
        sl = slice(b0, b1)
        parts.append(oracle.verify(
            host_logits(w.target[sl]), host_logits(w.draft[sl]), w.tokens[sl].cpu().numpy(),
            None if w.row_D is None else w.row_D[sl].cpu().numpy(),
            temperature=w.temperature, mode=w.mode, seed=w.seed if seed is None else seed,
            temperature_per_req=None if w.temperature_per_req is None
            else w.temperature_per_req[sl].cpu().numpy(),
            mode_per_req=None if w.mode_per_req is None else w.mode_per_req[sl].cpu().numpy(),
            saguaro_k=w.saguaro_k, saguaro_c=float(np.float32(w.saguaro_c)), request_offset=b0,
            nthreads=nthreads))
    out = {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}
    out["reqs"] = np.array(reqs)
    out["seed"] = w.seed if seed is None else seed
    return out


def _row(t, b, r):
    return t[b, r].float().cpu().numpy().astype(np.float64)


def check_valid(w, b, got, ref_lse, seed):
    """Checks of request b's GPU outputs that hold for every correct result when
    several are (a near-tie in the accept test or the race): the accepted
    prefix is the drafts; every accepted draft had u < a and the rejected one
    u >= a, within the 1e-5 near-tie band, with u the oracle's own draws and a
    from the oracle's row LSEs; the token at slot n is in [0, V) with p > 0,
    and after a rejection p > q' there (or the request says the residual was
    empty); the slots after n are -1."""
    D_list, modes = w.row_D_list(), w.modes()
    Db, mode = D_list[b], modes[b]
    T = float(w.temperature_per_req[b]) if w.temperature_per_req is not None else w.temperature
    al = int(got["accept_len"][b])
    assert 1 <= al <= Db + 1, (b, al)
    n = al - 1
    toks = got["tokens"][b]
    drafts = w.tokens[b].cpu().numpy()
    assert np.array_equal(toks[:n], drafts[:n]), b
    assert np.all(toks[n + 1:] == -1), b
    x = int(toks[n])
    assert 0 <= x < w.V, (b, x)
    zt_n = _row(w.target, b, n)
    assert np.isfinite(zt_n[x]), (b, x)
    assert mode != oracle.SVO_GREEDY, "greedy requests have no near-ties"

    def logq(d, tok):
        zq = _row(w.draft, b, d)
        lq = zq[tok] / T - ref_lse[w.D_max + 1 + d]
        if mode == oracle.SVO_SAGUARO and lq != -np.inf:
            k = min(w.saguaro_k, w.V)
            top = np.lexsort((np.arange(w.V), -zq))[:k]
            mass = np.exp(zq[top] / T - ref_lse[w.D_max + 1 + d]).sum()
            c = float(np.float32(w.saguaro_c))
            lq += (math.log(c) if tok in set(top.tolist()) else 0.0) - math.log1p(-(1 - c) * mass)
        return lq

    g = b  # the request's global index (no offset in these runs)
    for d in range(min(n + 1, Db)):
        xd = int(drafts[d])
        lp = _row(w.target, b, d)[xd] / T - ref_lse[d]
        lq = logq(d, xd)
        a = 0.0 if lp == -np.inf else (1.0 if lq == -np.inf else min(1.0, math.exp(lp - lq)))
        u = oracle.accept_uniform(seed, g, d)
        if d < n:
            assert u < a + 1e-5, (b, d, u, a)
        else:
            assert u >= a - 1e-5, (b, d, u, a)
    if n < Db and not (int(got["flags"][b]) & sv.SV_FLAG_RESIDUAL_EMPTY):
        lp = zt_n[x] / T - ref_lse[n]
        assert lp > logq(n, x), (b, x)


def compare(w, got, ref, early_exit=False):
    """Assert parity; return a summary.  Requests the oracle flags as near-ties
    are exempt from bit-exactness; their outputs are checked for validity
    (check_valid) instead.  Offsets are not used: request b is global index b.
    early_exit: rows past the request's outcome may be unread (no LSE); those
    up to it must have one."""
    reqs = ref["reqs"]
    D_list = w.row_D_list()
    lse_tol = LSE_TOL[w.dtype]
    exempt, checked = 0, 0
    worst_lse = 0.0
    for i, b in enumerate(reqs):
        rf, gf = int(ref["flags"][i]), int(got["flags"][b])
        assert (rf & oracle.FLAG_ERRORS) == (gf & sv.SV_FLAG_ERRORS), (b, rf, gf)
        if rf & oracle.FLAG_NEAR_TIE:
            exempt += 1
            check_valid(w, b, got, ref["row_lse"][i], ref["seed"])
            continue
        checked += 1
        assert got["accept_len"][b] == ref["accept_len"][i], (b, got["accept_len"][b], ref["accept_len"][i])
        assert np.array_equal(got["tokens"][b], ref["tokens"][i]), (b, got["tokens"][b], ref["tokens"][i])
        if rf & oracle.FLAG_ERRORS:
            continue
        r = ref["row_lse"][i]
        g = got["row_lse"][b].astype(np.float64)
        used = ~np.isnan(r)
        if early_exit:
            n = int(ref["accept_len"][i]) - 1
            pos = np.array([s if s <= w.D_max else s - w.D_max - 1 for s in range(len(r))])
            needed = used & (pos <= n)
            assert np.all(~np.isnan(g[needed])), (b, g)
            assert np.all(np.isnan(g[~used])), (b, g)
            used = used & ~np.isnan(g)
        else:
            assert np.array_equal(used, ~np.isnan(g)), (b, r, g)
        if used.any():
            # relative to |LSE|, or absolute where |LSE| < 1 (relative error is ill-posed near 0)
            rel = np.abs(g[used] - r[used]) / np.maximum(np.abs(r[used]), 1.0)
            worst_lse = max(worst_lse, float(rel.max()))
            assert rel.max() <= lse_tol, (b, rel.max())
    return dict(checked=checked, exempt=exempt, worst_lse_rel=worst_lse)
