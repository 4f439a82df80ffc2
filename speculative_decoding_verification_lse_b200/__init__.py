"""Python binding of libspecverify (the C ABI in include/specverify.h).

Argument marshalling only: tensors are turned into device pointers and sizes,
and every step of the verification runs in the library's CUDA kernels.  There
is no CPU path: without the built library or a CUDA device the calls raise.

    import speculative_decoding_verification_lse_b200 as sv
    out = sv.verify(target, draft, tokens, temperature=1.0, seed=0)   # torch CUDA tensors
    out["tokens"], out["accept_len"], out["flags"]
"""
import ctypes
import os

SV_F32, SV_BF16 = 0, 1
SV_STOCHASTIC, SV_GREEDY, SV_SAGUARO = 0, 1, 2
SV_OK, SV_ERR_INVALID_ARG, SV_ERR_UNSUPPORTED, SV_ERR_CUDA = 0, -1, -2, -3
SV_VARIANT_AUTO, SV_VARIANT_SPLIT, SV_VARIANT_FUSED, SV_VARIANT_CLUSTER = 0, 1, 2, 3
SV_VARIANT_EARLY_EXIT = 4
SV_TAIL_PER_REQUEST, SV_TAIL_ITEMS = 1 << 4, 1 << 5

SV_FLAG_ACCEPT_NEAR_TIE = 1 << 0
SV_FLAG_RACE_NEAR_TIE = 1 << 1
SV_FLAG_RESIDUAL_EMPTY = 1 << 2
SV_FLAG_BAD_TOKEN = 1 << 8
SV_FLAG_BAD_ROW_D = 1 << 9
SV_FLAG_NONFINITE = 1 << 10
SV_FLAG_BAD_PARAM = 1 << 11
SV_FLAG_SEQ_FULL = 1 << 13
SV_FLAG_NEAR_TIE = SV_FLAG_ACCEPT_NEAR_TIE | SV_FLAG_RACE_NEAR_TIE
SV_STATUS_BAD_TOKEN = SV_FLAG_BAD_TOKEN
SV_STATUS_BAD_ROW_D = SV_FLAG_BAD_ROW_D
SV_STATUS_NONFINITE = SV_FLAG_NONFINITE
SV_STATUS_BAD_PARAM = SV_FLAG_BAD_PARAM
SV_STATUS_RESIDUAL_EMPTY = SV_FLAG_RESIDUAL_EMPTY
SV_STATUS_TIMEOUT = 1 << 12
SV_STATUS_SEQ_FULL = SV_FLAG_SEQ_FULL
SV_FLAG_ERRORS = (SV_FLAG_BAD_TOKEN | SV_FLAG_BAD_ROW_D | SV_FLAG_NONFINITE | SV_FLAG_BAD_PARAM
                  | SV_STATUS_TIMEOUT)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspecverify.so")


class SvEpilogueArgs(ctypes.Structure):
    """Mirror of sv_epilogue_args."""
    _fields_ = [
        ("window", ctypes.c_void_p),
        ("next_window", ctypes.c_void_p),
        ("seq", ctypes.c_void_p),
        ("seq_cap", ctypes.c_int),
        ("seq_len", ctypes.c_void_p),
    ]


class SvParams(ctypes.Structure):
    """Mirror of sv_params."""
    _fields_ = [
        ("stream", ctypes.c_void_p),
        ("temperature_per_req", ctypes.c_void_p),
        ("mode_per_req", ctypes.c_void_p),
        ("saguaro_k", ctypes.c_int),
        ("saguaro_c", ctypes.c_float),
        ("variant", ctypes.c_int),
        ("request_offset", ctypes.c_uint32),
        ("out_row_lse", ctypes.c_void_p),
        ("out_flags", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("timing_events", ctypes.c_void_p),
        ("out_draft_top", ctypes.c_void_p),
        ("epilogue", ctypes.POINTER(SvEpilogueArgs)),
        ("seed_device", ctypes.c_void_p),
    ]


class SvError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"libspecverify error {code}: {msg}")
        self.code = code


_lib = None

_VERIFY_ARGS = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_float, ctypes.c_int, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]


def load(build_if_needed=True):
    """Load libspecverify.so (compiling it first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_needed:
        from . import build as _build
        _build.build()
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run __graft_entry__.build()")
    L = ctypes.CDLL(LIB_PATH)
    L.sv_verify.argtypes = _VERIFY_ARGS
    L.sv_verify.restype = ctypes.c_int
    L.sv_verify_ex.argtypes = _VERIFY_ARGS + [ctypes.POINTER(SvParams)]
    L.sv_verify_ex.restype = ctypes.c_int
    L.sv_verify_static.argtypes = _VERIFY_ARGS + [ctypes.POINTER(SvParams)]
    L.sv_verify_static.restype = ctypes.c_int
    L.sv_verify_greedy.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_void_p, ctypes.c_void_p]
    L.sv_verify_greedy.restype = ctypes.c_int
    L.sv_epilogue.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                              ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    L.sv_epilogue.restype = ctypes.c_int
    L.sv_ssd_lookup.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    L.sv_ssd_lookup.restype = ctypes.c_int
    L.sv_shard_exchange_bytes.argtypes = [ctypes.c_int] * 5
    L.sv_shard_exchange_bytes.restype = ctypes.c_size_t
    L.sv_shard_stats.argtypes = _VERIFY_ARGS[:11] + [ctypes.c_int, ctypes.c_int,
                                                     ctypes.POINTER(SvParams), ctypes.c_void_p]
    L.sv_shard_stats.restype = ctypes.c_int
    L.sv_shard_race.argtypes = _VERIFY_ARGS[:11] + [ctypes.c_int, ctypes.c_int,
                                                    ctypes.POINTER(SvParams), ctypes.c_void_p,
                                                    ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_void_p]
    L.sv_shard_race.restype = ctypes.c_int
    L.sv_shard_finish.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.POINTER(SvParams)]
    L.sv_shard_finish.restype = ctypes.c_int
    L.sv_verify_tree.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 4 + [
        ctypes.c_float, ctypes.c_int, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.POINTER(SvParams)]
    L.sv_verify_tree.restype = ctypes.c_int
    L.sv_advance_seed.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p]
    L.sv_advance_seed.restype = ctypes.c_int
    L.sv_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    L.sv_workspace_bytes.restype = ctypes.c_size_t
    L.sv_get_device_status.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]
    L.sv_get_device_status.restype = ctypes.c_int
    L.sv_last_error.argtypes = []
    L.sv_last_error.restype = ctypes.c_char_p
    L.sv_shutdown.argtypes = []
    L.sv_shutdown.restype = None
    L.sv_version.argtypes = []
    L.sv_version.restype = ctypes.c_int
    _lib = L
    return L


def _p(x):
    """A device pointer from a tensor, an int or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _check(rc):
    if rc != SV_OK:
        raise SvError(rc, load().sv_last_error().decode())
    return rc


# ---- the C ABI, same names (pointers may be tensors or ints)

def sv_verify(target_logits, draft_logits, draft_tokens, row_D, B, D_max, V, dtype,
              temperature, mode, seed, out_tokens, out_accept_len):
    return load().sv_verify(_p(target_logits), _p(draft_logits), _p(draft_tokens), _p(row_D),
                            B, D_max, V, dtype, temperature, mode, seed & (2**64 - 1),
                            _p(out_tokens), _p(out_accept_len))


def sv_verify_greedy(target_logits, draft_tokens, row_D, B, D_max, V, dtype, out_tokens,
                     out_accept_len):
    return load().sv_verify_greedy(_p(target_logits), _p(draft_tokens), _p(row_D), B, D_max, V,
                                   dtype, _p(out_tokens), _p(out_accept_len))


def sv_verify_ex(target_logits, draft_logits, draft_tokens, row_D, B, D_max, V, dtype,
                 temperature, mode, seed, out_tokens, out_accept_len, params=None):
    return load().sv_verify_ex(_p(target_logits), _p(draft_logits), _p(draft_tokens), _p(row_D),
                               B, D_max, V, dtype, temperature, mode, seed & (2**64 - 1),
                               _p(out_tokens), _p(out_accept_len),
                               ctypes.byref(params) if params is not None else None)


def sv_verify_static(target_logits, draft_logits, draft_tokens, row_D, B, D_max, V, dtype,
                     temperature, mode, seed, out_tokens, out_accept_len, params=None):
    """sv_verify_ex without any device allocation (fixed in-library scratch)."""
    return load().sv_verify_static(_p(target_logits), _p(draft_logits), _p(draft_tokens),
                                   _p(row_D), B, D_max, V, dtype, temperature, mode,
                                   seed & (2**64 - 1), _p(out_tokens), _p(out_accept_len),
                                   ctypes.byref(params) if params is not None else None)


SV_STATIC_WORKSPACE_BYTES = 8 << 20


def sv_epilogue(window, out_tokens, out_accept_len, B, D_max, next_window, seq, seq_cap, seq_len,
                flags=None, stream=None):
    return load().sv_epilogue(_p(window), _p(out_tokens), _p(out_accept_len), B, D_max,
                              _p(next_window), _p(seq), int(seq_cap), _p(seq_len), _p(flags),
                              _stream_ptr(stream))


def sv_ssd_lookup(out_tokens, out_accept_len, B, D_max, keys_al, keys_token, K, spec, S, out_hit,
                  out_spec=None, stream=None):
    return load().sv_ssd_lookup(_p(out_tokens), _p(out_accept_len), B, D_max, _p(keys_al),
                                _p(keys_token), int(K), _p(spec), int(S), _p(out_hit),
                                _p(out_spec), _stream_ptr(stream))


def sv_shard_exchange_bytes(B, D_max, V_local, dtype, stage):
    return load().sv_shard_exchange_bytes(B, D_max, V_local, dtype, stage)


def sv_shard_stats(target_local, draft_local, draft_tokens, row_D, B, D_max, V_local, dtype,
                   temperature, mode, seed, n_shards, shard, params, exchange1):
    return load().sv_shard_stats(_p(target_local), _p(draft_local), _p(draft_tokens), _p(row_D),
                                 B, D_max, V_local, dtype, temperature, mode, seed & (2**64 - 1),
                                 n_shards, shard,
                                 ctypes.byref(params) if params is not None else None,
                                 _p(exchange1))


def sv_shard_race(target_local, draft_local, draft_tokens, row_D, B, D_max, V_local, dtype,
                  temperature, mode, seed, n_shards, shard, params, gathered1, out_tokens,
                  out_accept_len, exchange2):
    return load().sv_shard_race(_p(target_local), _p(draft_local), _p(draft_tokens), _p(row_D),
                                B, D_max, V_local, dtype, temperature, mode, seed & (2**64 - 1),
                                n_shards, shard,
                                ctypes.byref(params) if params is not None else None,
                                _p(gathered1), _p(out_tokens), _p(out_accept_len), _p(exchange2))


def sv_shard_finish(B, D_max, n_shards, gathered2, out_tokens, params=None):
    return load().sv_shard_finish(B, D_max, n_shards, _p(gathered2), _p(out_tokens),
                                  ctypes.byref(params) if params is not None else None)


def sv_verify_tree(target_logits, draft_logits, node_tokens, parents, n_nodes, B, N_max, V, dtype,
                   temperature, mode, seed, out_tokens, out_accept_len, out_nodes, params=None):
    return load().sv_verify_tree(_p(target_logits), _p(draft_logits), _p(node_tokens), _p(parents),
                                 _p(n_nodes), B, N_max, V, dtype, temperature, mode,
                                 seed & (2**64 - 1), _p(out_tokens), _p(out_accept_len),
                                 _p(out_nodes), ctypes.byref(params) if params is not None else None)


def verify_tree(target, draft, tokens, parents, n_nodes=None, *, temperature=1.0,
                mode=SV_STOCHASTIC, seed=0, temperature_per_req=None, mode_per_req=None,
                request_offset=0, stream=None, row_lse=False, timing_events=None,
                seed_device=None):
    """Tree verification of a batch held in CUDA tensors (sv_verify_tree):
    target [B, N+1, V], draft [B, N, V] (or None when greedy), tokens and parents
    [B, N] int32, n_nodes [B] int32 or None.  Returns dict(tokens, accept_len,
    nodes, flags [, row_lse]) as CUDA tensors (not synchronised)."""
    import torch
    if not target.is_cuda:
        raise ValueError("target logits must be a CUDA tensor (there is no CPU path)")
    dt = _dtype_code(target)
    B, Np1, V = target.shape
    N = Np1 - 1
    for name, t in (("tokens", tokens), ("parents", parents)):
        if t.dtype != torch.int32 or tuple(t.shape) != (B, N) or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous int32 [B, N]")
    dev = target.device
    out = dict(tokens=torch.empty((B, N + 1), dtype=torch.int32, device=dev),
               accept_len=torch.empty((B,), dtype=torch.int32, device=dev),
               nodes=torch.empty((B, N), dtype=torch.int32, device=dev),
               flags=torch.empty((B,), dtype=torch.int32, device=dev))
    if row_lse:
        out["row_lse"] = torch.empty((B, 2 * N + 1), dtype=torch.float32, device=dev)
    prm = SvParams()
    prm.stream = _stream_ptr(stream)
    prm.temperature_per_req = _p(temperature_per_req)
    prm.mode_per_req = _p(mode_per_req)
    prm.request_offset = int(request_offset)
    prm.out_flags = _p(out["flags"])
    prm.out_row_lse = _p(out.get("row_lse"))
    prm.seed_device = _seed_device_ptr(seed_device)
    if timing_events is not None:
        arr = (ctypes.c_void_p * 2)(timing_events[0].cuda_event, timing_events[1].cuda_event)
        prm.timing_events = ctypes.cast(arr, ctypes.c_void_p)
    with torch.cuda.device(dev):
        _check(sv_verify_tree(target, draft, tokens, parents, n_nodes, B, N, V, dt,
                              float(temperature), int(mode), int(seed), out["tokens"],
                              out["accept_len"], out["nodes"], prm))
    return out


def sv_advance_seed(seed_device, by=1, stream=None):
    """Enqueue seed_device += by (a CUDA uint64/int64 tensor of one element, or
    a device pointer) on `stream`: between the captured calls of a graph whose
    calls read their seed from it (verify(..., seed_device=...))."""
    _check(load().sv_advance_seed(_p(seed_device), int(by) & (2**64 - 1), _stream_ptr(stream)))


def sv_workspace_bytes(B, D_max, V, dtype):
    return load().sv_workspace_bytes(B, D_max, V, dtype)


def sv_get_device_status(stream=None):
    bits = ctypes.c_uint32(0)
    _check(load().sv_get_device_status(_stream_ptr(stream), ctypes.byref(bits)))
    return bits.value


def sv_last_error():
    return load().sv_last_error().decode()


def sv_shutdown():
    load().sv_shutdown()


def sv_version():
    return load().sv_version()


# ---- convenience wrapper over torch tensors

def _stream_ptr(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _seed_device_ptr(t):
    import torch
    if t is None or isinstance(t, int):
        return t
    if not t.is_cuda or t.numel() != 1 or t.element_size() != 8 or t.dtype.is_floating_point:
        raise ValueError("seed_device must be a one-element 64-bit integer CUDA tensor")
    return t.data_ptr()


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return SV_F32
    if t.dtype == torch.bfloat16:
        return SV_BF16
    raise TypeError(f"logits must be float32 or bfloat16 CUDA tensors, got {t.dtype}")


def verify(target, draft, tokens, row_D=None, *, temperature=1.0, mode=SV_STOCHASTIC, seed=0,
           temperature_per_req=None, mode_per_req=None, saguaro_k=5, saguaro_c=0.5,
           request_offset=0, variant=SV_VARIANT_AUTO, stream=None, row_lse=False,
           out=None, workspace=None, timing_events=None, epilogue=None, draft_top=False,
           seed_device=None):
    """Verify a batch held in CUDA tensors; returns dict(tokens, accept_len, flags
    [, row_lse]) as CUDA tensors, enqueued on `stream` (not synchronised).
    epilogue: optional dict(window, next_window, seq, seq_len) of int32 CUDA
    tensors (any may be None) for the on-device step after verification
    (sv_epilogue), run on the same stream.  draft_top: also return the k
    largest logits of each saguaro draft row (sv_params.out_draft_top).
    seed_device: optional CUDA int64/uint64 tensor of one element whose value
    the kernels read as the seed (sv_params.seed_device; `seed` is then
    unused), for CUDA graphs that advance it between replays."""
    import torch
    if not target.is_cuda:
        raise ValueError("target logits must be a CUDA tensor (there is no CPU path)")
    dt = _dtype_code(target)
    if not target.is_contiguous():
        raise ValueError("target logits must be contiguous")
    B, Dp1, V = target.shape
    D = Dp1 - 1
    if draft is not None:
        if draft.dtype != target.dtype or tuple(draft.shape) != (B, D, V) or not draft.is_contiguous():
            raise ValueError("draft logits must be contiguous [B, D_max, V] of the target's dtype")
    if tokens.dtype != torch.int32 or tuple(tokens.shape) != (B, D) or not tokens.is_contiguous():
        raise ValueError("draft tokens must be contiguous int32 [B, D_max]")
    for name, t, dtp in (("row_D", row_D, torch.int32),
                         ("temperature_per_req", temperature_per_req, torch.float32),
                         ("mode_per_req", mode_per_req, torch.int8)):
        if t is not None and (t.dtype != dtp or t.numel() != B or not t.is_cuda):
            raise ValueError(f"{name} must be a CUDA {dtp} tensor of {B} elements")
    dev = target.device
    if out is None:
        out = dict(tokens=torch.empty((B, D + 1), dtype=torch.int32, device=dev),
                   accept_len=torch.empty((B,), dtype=torch.int32, device=dev),
                   flags=torch.empty((B,), dtype=torch.int32, device=dev))
        if row_lse:
            out["row_lse"] = torch.empty((B, 2 * D + 1), dtype=torch.float32, device=dev)
        if draft_top:
            k = int(saguaro_k) if int(saguaro_k) > 0 else 5
            out["draft_top"] = torch.empty((B, D, min(k, V)), dtype=torch.int32, device=dev)
    prm = SvParams()
    prm.stream = _stream_ptr(stream)
    prm.temperature_per_req = _p(temperature_per_req)
    prm.mode_per_req = _p(mode_per_req)
    prm.saguaro_k = int(saguaro_k)
    prm.saguaro_c = float(saguaro_c)
    prm.variant = int(variant)
    prm.request_offset = int(request_offset)
    prm.out_row_lse = _p(out.get("row_lse"))
    prm.out_flags = _p(out.get("flags"))
    prm.out_draft_top = _p(out.get("draft_top"))
    prm.seed_device = _seed_device_ptr(seed_device)
    if workspace is not None:
        prm.workspace = _p(workspace)
        prm.workspace_bytes = workspace.numel() * workspace.element_size()
    if timing_events is not None:
        # torch creates an event's CUDA handle on its first record()
        if not timing_events[0].cuda_event or not timing_events[1].cuda_event:
            raise ValueError("timing events must have been recorded once before use")
        arr = (ctypes.c_void_p * 2)(timing_events[0].cuda_event, timing_events[1].cuda_event)
        prm.timing_events = ctypes.cast(arr, ctypes.c_void_p)
    ep = None
    if epilogue is not None:
        ep = SvEpilogueArgs()
        ep.window = _p(epilogue.get("window"))
        ep.next_window = _p(epilogue.get("next_window"))
        sq = epilogue.get("seq")
        ep.seq = _p(sq)
        ep.seq_cap = 0 if sq is None else int(sq.shape[-1])
        ep.seq_len = _p(epilogue.get("seq_len"))
        prm.epilogue = ctypes.pointer(ep)
    with torch.cuda.device(dev):
        _check(sv_verify_ex(target, draft, tokens, row_D, B, D, V, dt, float(temperature),
                            int(mode), int(seed), out["tokens"], out["accept_len"], prm))
    return out


def verify_workload(w, **kw):
    """verify() on a workloads.Workload."""
    return verify(w.target, w.draft, w.tokens, w.row_D, temperature=w.temperature, mode=w.mode,
                  seed=kw.pop("seed", w.seed), temperature_per_req=w.temperature_per_req,
                  mode_per_req=w.mode_per_req, saguaro_k=w.saguaro_k, saguaro_c=w.saguaro_c, **kw)
