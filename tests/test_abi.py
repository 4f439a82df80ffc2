"""The C ABI without a GPU: the library builds, loads, exports every entry point
include/specverify.h declares, and rejects invalid arguments on the host before
any CUDA call (no compute runs here)."""
import ctypes
import os
import re

import pytest

import speculative_decoding_verification_lse_b200 as sv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(sv_\w+)\s*\(", text, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    return sv.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sv_verify", "sv_verify_greedy", "sv_verify_ex", "sv_workspace_bytes",
                     "sv_get_device_status", "sv_last_error", "sv_shutdown", "sv_version"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(sv.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(raw, n)]
    assert not missing, missing


def test_only_the_abi_is_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", sv.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {n for n in exported if n.startswith("sv_")}
    assert ours == set(declared_functions())


def header_constants():
    """Every `SV_NAME = value` of the header's enums, values evaluated (1u << n,
    plain integers, and references to earlier names)."""
    text = open(os.path.join(ROOT, "include", "specverify.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    vals = {}
    for body in re.findall(r"enum\s*\{(.*?)\}", text, flags=re.S):
        for item in body.split(","):
            m = re.match(r"\s*(SV_\w+)\s*=\s*(.+?)\s*$", item, flags=re.S)
            if not m:
                continue
            expr = re.sub(r"(\d+)u\b", r"\1", m.group(2))
            vals[m.group(1)] = eval(expr, {}, dict(vals))
    return vals


def test_binding_constants_equal_the_header():
    vals = header_constants()
    assert len(vals) >= 20
    for name, v in vals.items():
        assert hasattr(sv, name), name
        assert getattr(sv, name) == v, (name, getattr(sv, name), v)


def test_version_and_workspace_sizes(lib):
    assert sv.sv_version() == 10000
    a = sv.sv_workspace_bytes(256, 7, 128256, sv.SV_BF16)
    b = sv.sv_workspace_bytes(1, 4, 1024, sv.SV_F32)
    assert a > b > 0 and a % 256 == 0
    assert sv.sv_workspace_bytes(-1, 4, 10, sv.SV_F32) == 0
    assert sv.sv_workspace_bytes(1, 4, 10, 9) == 0


@pytest.mark.parametrize("kw,needle", [
    (dict(B=-1), "B must"),
    (dict(D_max=33), "D_max"),
    (dict(D_max=-1), "D_max"),
    (dict(V=0), "V must"),
    (dict(dtype=5), "dtype"),
    (dict(mode=7), "mode"),
    (dict(temperature=0.0), "temperature"),
    (dict(temperature=float("nan")), "temperature"),
    (dict(temperature=float("inf")), "temperature"),
])
def test_invalid_arguments_are_rejected_on_the_host(lib, kw, needle):
    args = dict(B=2, D_max=3, V=100, dtype=sv.SV_BF16, temperature=1.0, mode=sv.SV_STOCHASTIC)
    args.update(kw)
    rc = sv.sv_verify(None, None, None, None, args["B"], args["D_max"], args["V"], args["dtype"],
                      args["temperature"], args["mode"], 0, None, None)
    assert rc == sv.SV_ERR_INVALID_ARG
    assert needle in sv.sv_last_error()


@pytest.mark.parametrize("field,value,needle", [
    ("saguaro_k", 9, "saguaro_k"),
    ("saguaro_c", 1.5, "saguaro_c"),
    ("variant", 5, "variant"),
])
def test_invalid_params_are_rejected_on_the_host(lib, field, value, needle):
    p = sv.SvParams()
    setattr(p, field, value)
    rc = sv.sv_verify_ex(None, None, None, None, 2, 3, 100, sv.SV_BF16, 1.0, sv.SV_SAGUARO, 0,
                         None, None, p)
    assert rc == sv.SV_ERR_INVALID_ARG and needle in sv.sv_last_error()


def test_null_pointers_are_rejected_on_the_host(lib):
    rc = sv.sv_verify(None, None, None, None, 2, 3, 100, sv.SV_BF16, 1.0, sv.SV_STOCHASTIC, 0,
                      None, None)
    assert rc == sv.SV_ERR_INVALID_ARG and "non-NULL" in sv.sv_last_error()
    # greedy needs no draft logits, stochastic does
    fake = 1 << 20  # never dereferenced: the call is rejected first
    rc = sv.sv_verify(fake, None, fake, None, 2, 3, 100, sv.SV_BF16, 1.0, sv.SV_STOCHASTIC, 0,
                      fake, fake)
    assert rc == sv.SV_ERR_INVALID_ARG and "draft_logits" in sv.sv_last_error()
    rc = sv.sv_verify(fake + 1, fake, fake, None, 2, 3, 100, sv.SV_BF16, 1.0, sv.SV_STOCHASTIC,
                      0, fake, fake)
    assert rc == sv.SV_ERR_INVALID_ARG and "aligned" in sv.sv_last_error()


def test_seed_advance_rejects_bad_pointers_on_the_host(lib):
    L = sv.load()
    assert L.sv_advance_seed(None, 1, None) == sv.SV_ERR_INVALID_ARG
    assert "seed_device" in sv.sv_last_error()
    assert L.sv_advance_seed((1 << 20) + 4, 1, None) == sv.SV_ERR_INVALID_ARG
    with pytest.raises(sv.SvError):
        sv.sv_advance_seed(None)


def test_empty_batch_is_a_no_op(lib):
    assert sv.sv_verify(None, None, None, None, 0, 3, 100, sv.SV_BF16, 1.0, sv.SV_STOCHASTIC, 0,
                        None, None) == sv.SV_OK


def test_no_cpu_path_in_the_binding():
    import torch
    t = torch.zeros((1, 2, 8), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        sv.verify(t, t[:, :1], torch.zeros((1, 1), dtype=torch.int32))


def test_device_seed_must_be_a_64_bit_integer_cuda_tensor():
    import torch
    from speculative_decoding_verification_lse_b200 import _seed_device_ptr
    assert _seed_device_ptr(None) is None
    assert _seed_device_ptr(1 << 20) == 1 << 20  # a raw device address passes through
    # host tensors (this test needs no GPU), of the right and of wrong shapes and types
    for bad in (torch.zeros(1, dtype=torch.int64), torch.zeros(2, dtype=torch.int64),
                torch.zeros(1, dtype=torch.float64), torch.zeros(1, dtype=torch.int32)):
        with pytest.raises(ValueError, match="seed_device"):
            _seed_device_ptr(bad)


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "speculative_decoding_verification_lse_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "svo_" not in text and "svo.h" not in text, f


def test_static_entry_point_checks_arguments_before_its_size(lib):
    # the ordinary argument checks come first, so an invalid call of any size
    # gets sv_verify_ex's code, and a valid call too large for the fixed array
    # gets SV_ERR_UNSUPPORTED; neither reaches a CUDA call
    fake = 1 << 20
    rc = sv.sv_verify_static(fake, fake, fake, None, 4096, 33, 128256, sv.SV_BF16, 1.0,
                             sv.SV_STOCHASTIC, 0, fake, fake, None)
    assert rc == sv.SV_ERR_INVALID_ARG and "D_max" in sv.sv_last_error()
    rc = sv.sv_verify_static(fake, fake, fake, None, 4096, 7, 128256, sv.SV_BF16, 0.0,
                             sv.SV_STOCHASTIC, 0, fake, fake, None)
    assert rc == sv.SV_ERR_INVALID_ARG and "temperature" in sv.sv_last_error()
    rc = sv.sv_verify_static(fake, fake, fake, None, 4096, 7, 128256, sv.SV_BF16, 1.0,
                             sv.SV_STOCHASTIC, 0, fake, fake, None)
    assert rc == sv.SV_ERR_UNSUPPORTED and "sv_verify_static" in sv.sv_last_error()


def test_epilogue_rejects_invalid_arguments_on_the_host(lib):
    fake = 1 << 20  # never dereferenced: each call is rejected before any launch
    cases = [
        (dict(B=-1), "B must"),
        (dict(D_max=33), "D_max"),
        (dict(out_tokens=None), "non-NULL"),
        (dict(window=None), "next_window needs window"),
        (dict(seq_len=None), "seq needs seq_len"),
        (dict(seq_cap=-1), "seq needs seq_len"),
    ]
    for kw, needle in cases:
        a = dict(window=fake, out_tokens=fake, al=fake, B=4, D_max=3, next_window=fake, seq=fake,
                 seq_cap=16, seq_len=fake)
        a.update(kw)
        rc = sv.sv_epilogue(a["window"], a["out_tokens"], a["al"], a["B"], a["D_max"],
                            a["next_window"], a["seq"], a["seq_cap"], a["seq_len"])
        assert rc == sv.SV_ERR_INVALID_ARG and needle in sv.sv_last_error(), kw
    assert sv.sv_epilogue(None, None, None, 0, 3, None, None, 0, None) == sv.SV_OK
    # the verification's own epilogue option is checked the same way, before any launch
    p = sv.SvParams()
    ep = sv.SvEpilogueArgs()
    ep.next_window = fake
    p.epilogue = ctypes.pointer(ep)
    rc = sv.sv_verify_ex(fake, fake, fake, None, 2, 3, 100, sv.SV_BF16, 1.0, sv.SV_STOCHASTIC, 0,
                         fake, fake, p)
    assert rc in (sv.SV_ERR_INVALID_ARG, sv.SV_ERR_CUDA)


def test_shard_calls_reject_invalid_arguments_on_the_host(lib):
    fake = 1 << 20  # never dereferenced
    base = (fake, fake, fake, None, 4, 3, 1000, sv.SV_BF16, 1.0, sv.SV_STOCHASTIC, 0)
    for n, r, Vl, needle in ((2, 2, 1000, "out of range"), (0, 0, 1000, "out of range"),
                             (2, 0, 1002, "multiple of 4")):
        args = base[:6] + (Vl,) + base[7:]
        rc = sv.sv_shard_stats(*args, n, r, None, fake)
        assert rc == sv.SV_ERR_INVALID_ARG and needle in sv.sv_last_error(), (n, r, Vl)
        rc = sv.sv_shard_race(*args, n, r, None, fake, fake, fake, fake)
        assert rc == sv.SV_ERR_INVALID_ARG and needle in sv.sv_last_error(), (n, r, Vl)
    rc = sv.sv_shard_stats(*base, 2, 0, None, None)
    assert rc == sv.SV_ERR_INVALID_ARG and "exchange1" in sv.sv_last_error()
    assert sv.sv_shard_finish(4, 3, 0, fake, fake) == sv.SV_ERR_INVALID_ARG
    assert sv.sv_shard_exchange_bytes(4, 3, 1000, sv.SV_BF16, 1) > 0
    assert sv.sv_shard_exchange_bytes(4, 3, 1000, sv.SV_BF16, 3) == 0
