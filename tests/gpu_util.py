"""Helpers for the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare them element by element."""
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
    return out


def compare(w, got, ref):
    """Assert parity; return a summary.  Requests the oracle flags as near-ties
    are exempt from bit-exactness (they are only checked for validity)."""
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
            al = int(got["accept_len"][b])
            assert 1 <= al <= D_list[b] + 1
            assert np.array_equal(got["tokens"][b, :al - 1], w.tokens[b, :al - 1].cpu().numpy())
            continue
        checked += 1
        assert got["accept_len"][b] == ref["accept_len"][i], (b, got["accept_len"][b], ref["accept_len"][i])
        assert np.array_equal(got["tokens"][b], ref["tokens"][i]), (b, got["tokens"][b], ref["tokens"][i])
        if rf & oracle.FLAG_ERRORS:
            continue
        r = ref["row_lse"][i]
        g = got["row_lse"][b].astype(np.float64)
        used = ~np.isnan(r)
        assert np.array_equal(used, ~np.isnan(g)), (b, r, g)
        if used.any():
            # relative to |LSE|, or absolute where |LSE| < 1 (relative error is ill-posed near 0)
            rel = np.abs(g[used] - r[used]) / np.maximum(np.abs(r[used]), 1.0)
            worst_lse = max(worst_lse, float(rel.max()))
            assert rel.max() <= lse_tol, (b, rel.max())
    return dict(checked=checked, exempt=exempt, worst_lse_rel=worst_lse)
