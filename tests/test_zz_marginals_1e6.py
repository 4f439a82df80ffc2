"""The statistical law of the emitted tokens over 10^6 requests in one call
(V=8, D=2), for every launch structure, and the oracle's exact outputs on a
slice of them.  The most expensive cases of the GPU suite, so they run last."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_lse_b200 as sv

pytestmark = pytest.mark.gpu

VARIANTS = pytest.mark.parametrize(
    "variant",
    [sv.SV_VARIANT_SPLIT | sv.SV_TAIL_PER_REQUEST, sv.SV_VARIANT_SPLIT | sv.SV_TAIL_ITEMS,
     sv.SV_VARIANT_FUSED, sv.SV_VARIANT_CLUSTER],
    ids=["split-per-request", "split-items", "fused", "cluster"])


@VARIANTS
@pytest.mark.parametrize("mode", [0, 2], ids=["plain", "saguaro"])
def test_emitted_marginals_equal_target_1e6_requests(sv, mode, variant):
    """V=8, D=2: 10^6 requests in one call (independent Philox streams): the
    emitted tokens follow p within 3 sigma per cell, as the oracle's do."""
    from svtest_util import sample_categorical, softmax
    rng = np.random.default_rng(100 + mode)
    V, D, N = 8, 2, 1_000_000
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
    T = torch.from_numpy(np.ascontiguousarray(np.broadcast_to(zt, (N, D + 1, V)))).cuda()
    Q = torch.from_numpy(np.ascontiguousarray(np.broadcast_to(zq, (N, D, V)))).cuda()
    out = sv.verify(T, Q, torch.from_numpy(tok).cuda(), mode=mode, seed=31, variant=variant)
    torch.cuda.synchronize()
    AL = out["accept_len"].cpu().numpy()
    toks = out["tokens"].cpu().numpy()
    assert sv.sv_get_device_status() == 0
    emitted = toks[np.arange(N), AL - 1]
    assert (emitted >= 0).all(), ("requests without an emitted token", np.nonzero(emitted < 0)[0][:8])
    from svtest_util import within_sigma
    for slot, sel in ((0, np.ones_like(AL, bool)), (1, AL >= 2), (2, AL == 3)):
        ok, worst = within_sigma(np.bincount(toks[sel, slot], minlength=V), p[slot], 3.0)
        assert ok, (slot, worst)
    # and exactly the oracle's outputs on a slice
    ref = oracle.verify(np.broadcast_to(zt, (2000, D + 1, V)), np.broadcast_to(zq, (2000, D, V)),
                        tok[:2000], mode=mode, seed=31)
    keep = (ref["flags"] & oracle.FLAG_NEAR_TIE) == 0
    assert np.array_equal(toks[:2000][keep], ref["tokens"][keep])
