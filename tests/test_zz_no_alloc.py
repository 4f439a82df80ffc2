"""sv_verify_static: the entry point that allocates no device memory.

Some callers cannot call cudaMalloc (their device memory belongs to a caching
allocator the library must not bypass, or an allocation's device-wide
synchronisation would stall their decode loop).  sv_verify_static runs the same
kernels with a fixed scratch array that lives in the library's own device
memory.  Here it is called through the C ABI and checked against the ordinary
entry point, sv_verify_ex with its own workspace, on two calls in a row (the
array keeps the previous call's contents, so the second call shows that every
call clears what it needs), in every launch structure.  This file is collected
last so that a run stopping at its first failure has run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import speculative_decoding_verification_lse_b200 as sv
from speculative_decoding_verification_lse_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LSE_TOL = {sv.SV_F32: 1e-5, sv.SV_BF16: 1e-3}


def _call(fn, w, seed, variant):
    B, D, V = w.B, w.D_max, w.V
    out = dict(tokens=torch.full((B, D + 1), -7, dtype=torch.int32, device="cuda"),
               accept_len=torch.full((B,), -7, dtype=torch.int32, device="cuda"),
               flags=torch.full((B,), -7, dtype=torch.int32, device="cuda"),
               row_lse=torch.full((B, 2 * D + 1), -7.0, dtype=torch.float32, device="cuda"))
    p = sv.SvParams()
    p.temperature_per_req = None if w.temperature_per_req is None else w.temperature_per_req.data_ptr()
    p.mode_per_req = None if w.mode_per_req is None else w.mode_per_req.data_ptr()
    p.saguaro_k, p.saguaro_c, p.variant = w.saguaro_k, w.saguaro_c, variant
    p.out_row_lse = out["row_lse"].data_ptr()
    p.out_flags = out["flags"].data_ptr()
    rc = fn(w.target, w.draft, w.tokens, w.row_D, B, D, V, w.dtype, w.temperature, w.mode, seed,
            out["tokens"], out["accept_len"], p)
    assert rc == sv.SV_OK, sv.sv_last_error()
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.parametrize("variant", [sv.SV_VARIANT_SPLIT, sv.SV_VARIANT_FUSED, sv.SV_VARIANT_CLUSTER,
                                     sv.SV_VARIANT_EARLY_EXIT],
                         ids=["split", "fused", "cluster", "early-exit"])
@pytest.mark.parametrize("name", ["b256", "ragged", "saguaro", "tiny"])
def test_static_entry_point_matches_the_ordinary_one(variant, name):
    sv.load()
    w = wl.make(name, "cuda")
    for seed in (11, 12):  # two calls in a row
        ref = _call(sv.sv_verify_ex, w, seed, variant)
        got = _call(sv.sv_verify_static, w, seed, variant)
        np.testing.assert_array_equal(got["tokens"], ref["tokens"])
        np.testing.assert_array_equal(got["accept_len"], ref["accept_len"])
        np.testing.assert_array_equal(got["flags"], ref["flags"])
        used = ~np.isnan(ref["row_lse"])
        assert np.array_equal(used, ~np.isnan(got["row_lse"]))
        rel = np.abs(got["row_lse"][used] - ref["row_lse"][used]) / np.maximum(
            np.abs(ref["row_lse"][used]), 1.0)
        assert rel.max(initial=0.0) <= LSE_TOL[w.dtype]
    assert sv.sv_get_device_status() == 0


def test_static_entry_point_rejects_sizes_beyond_its_array():
    sv.load()
    B, D, V = 4096, 7, 128256
    need = sv.sv_workspace_bytes(B, D, V, sv.SV_BF16)
    assert need > sv.SV_STATIC_WORKSPACE_BYTES
    fake = 1 << 20  # never dereferenced: the call is rejected before any launch
    rc = sv.sv_verify_static(fake, fake, fake, None, B, D, V, sv.SV_BF16, 1.0, sv.SV_STOCHASTIC,
                             0, fake, fake, None)
    assert rc == sv.SV_ERR_UNSUPPORTED
    msg = sv.sv_last_error()
    assert "sv_verify_static" in msg and str(need) in msg
