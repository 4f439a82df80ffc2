"""ctypes binding of the C oracle (oracle/svo.c).

TEST INFRASTRUCTURE ONLY.  The oracle is a plain double-precision CPU
restatement of the speculative-decoding verification rule.  Only the tests,
the smoke check and the benchmark's CPU-baseline leg may import this package;
the product library never does, and it shares no code with it.

Arrays are numpy: fp32 logits as ``float32``, bf16 logits as their raw
``uint16`` bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

SVO_F32, SVO_BF16 = 0, 1
SVO_STOCHASTIC, SVO_GREEDY, SVO_SAGUARO = 0, 1, 2

FLAG_ACCEPT_NEAR_TIE = 1 << 0
FLAG_RACE_NEAR_TIE = 1 << 1
FLAG_RESIDUAL_EMPTY = 1 << 2
FLAG_BAD_TOKEN = 1 << 8
FLAG_BAD_ROW_D = 1 << 9
FLAG_NONFINITE = 1 << 10
FLAG_BAD_PARAM = 1 << 11
FLAG_NEAR_TIE = FLAG_ACCEPT_NEAR_TIE | FLAG_RACE_NEAR_TIE
FLAG_ERRORS = FLAG_BAD_TOKEN | FLAG_BAD_ROW_D | FLAG_NONFINITE | FLAG_BAD_PARAM


class _Params(ctypes.Structure):
    _fields_ = [
        ("temperature_per_req", ctypes.c_void_p),
        ("mode_per_req", ctypes.c_void_p),
        ("saguaro_k", ctypes.c_int),
        ("saguaro_c", ctypes.c_double),
        ("request_offset", ctypes.c_uint32),
    ]


_lib = None


def _declare(L):
    u32p = ctypes.POINTER(ctypes.c_uint32)
    L.svo_philox4x32_10.argtypes = [u32p, u32p, u32p]
    L.svo_philox4x32_10.restype = None
    L.svo_accept_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32]
    L.svo_accept_uniform.restype = ctypes.c_double
    L.svo_race_exponential.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32]
    L.svo_race_exponential.restype = ctypes.c_double
    L.svo_row_lse.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_double]
    L.svo_row_lse.restype = ctypes.c_double
    L.svo_row_argmax.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
    L.svo_row_argmax.restype = ctypes.c_int
    L.svo_verify.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_float, ctypes.c_int, ctypes.c_uint64, ctypes.POINTER(_Params),
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int,
    ]
    L.svo_verify.restype = ctypes.c_int
    L.svo_epilogue.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                               ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                               ctypes.c_void_p, ctypes.c_void_p]
    L.svo_epilogue.restype = ctypes.c_int
    L.svo_row_topk.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_void_p]
    L.svo_row_topk.restype = None
    L.svo_ssd_lookup.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                 ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    L.svo_ssd_lookup.restype = ctypes.c_int
    L.svo_verify_tree.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
        ctypes.c_uint64, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_int]
    L.svo_verify_tree.restype = ctypes.c_int
    L.svo_has_openmp.argtypes = []
    L.svo_has_openmp.restype = ctypes.c_int
    return L


def lib():
    """The oracle library (built from oracle/svo.c on first use)."""
    global _lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(_build.build()))
    return _lib


def load_variant(path):
    """Load another build of the same source (the tests use this to check that
    their pins reject deliberately broken copies of the oracle)."""
    return _declare(ctypes.CDLL(path))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a):
    if a.dtype == np.float32:
        return SVO_F32
    if a.dtype == np.uint16:
        return SVO_BF16
    raise TypeError(f"logits must be float32 or uint16 (bf16 bits), got {a.dtype}")


def philox4x32_10(ctr, key, L=None):
    c = (ctypes.c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in ctr])
    k = (ctypes.c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    o = (ctypes.c_uint32 * 4)()
    (L or lib()).svo_philox4x32_10(c, k, o)
    return [int(v) for v in o]


def accept_uniform(seed, g, d, L=None):
    return (L or lib()).svo_accept_uniform(int(seed), int(g), int(d))


def race_exponential(seed, g, x, L=None):
    return (L or lib()).svo_race_exponential(int(seed), int(g), int(x))


def row_lse(row, T, L=None):
    row = np.ascontiguousarray(row)
    return (L or lib()).svo_row_lse(_ptr(row), row.shape[-1], _dtype_code(row), float(T))


def row_argmax(row, L=None):
    row = np.ascontiguousarray(row)
    return (L or lib()).svo_row_argmax(_ptr(row), row.shape[-1], _dtype_code(row))


def has_openmp():
    return bool(lib().svo_has_openmp())


def verify(target, draft, tokens, row_D=None, *, temperature=1.0, mode=SVO_STOCHASTIC,
           seed=0, temperature_per_req=None, mode_per_req=None, saguaro_k=5,
           saguaro_c=0.5, request_offset=0, nthreads=1, L=None):
    """Run the oracle on host arrays.

    target [B, D_max+1, V], draft [B, D_max, V] (or None when all greedy),
    tokens [B, D_max] int32, row_D [B] int32 or None.
    Returns dict(tokens [B, D_max+1] int32, accept_len [B] int32,
    flags [B] uint32, row_lse [B, 2*D_max+1] float64).
    """
    target = np.ascontiguousarray(target)
    B, Dp1, V = target.shape
    D_max = Dp1 - 1
    dt = _dtype_code(target)
    if draft is not None:
        draft = np.ascontiguousarray(draft)
        assert draft.dtype == target.dtype and draft.shape == (B, D_max, V)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, D_max)
    if row_D is not None:
        row_D = np.ascontiguousarray(row_D, dtype=np.int32).reshape(B)
    tpr = None if temperature_per_req is None else np.ascontiguousarray(
        temperature_per_req, dtype=np.float32).reshape(B)
    mpr = None if mode_per_req is None else np.ascontiguousarray(
        mode_per_req, dtype=np.int8).reshape(B)
    p = _Params(
        temperature_per_req=None if tpr is None else tpr.ctypes.data,
        mode_per_req=None if mpr is None else mpr.ctypes.data,
        saguaro_k=int(saguaro_k), saguaro_c=float(saguaro_c),
        request_offset=int(request_offset),
    )
    out_tokens = np.empty((B, D_max + 1), dtype=np.int32)
    out_al = np.empty((B,), dtype=np.int32)
    out_flags = np.empty((B,), dtype=np.uint32)
    out_lse = np.empty((B, 2 * D_max + 1), dtype=np.float64)
    rc = (L or lib()).svo_verify(
        _ptr(target), _ptr(draft), _ptr(tokens), _ptr(row_D), B, D_max, V, dt,
        float(temperature), int(mode), int(seed) & (2**64 - 1), ctypes.byref(p),
        _ptr(out_tokens), _ptr(out_al), _ptr(out_flags), _ptr(out_lse), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    return dict(tokens=out_tokens, accept_len=out_al, flags=out_flags, row_lse=out_lse)


def epilogue(window, out_tokens, accept_len, seq=None, seq_len=None, *, next_window=True,
             L=None):
    """The host epilogue (svo_epilogue).  window, out_tokens [B, D_max+1] int32,
    accept_len [B]; seq [B, cap] and seq_len [B] are updated in copies.
    Returns dict(next_window or None, seq, seq_len, full [B] bool)."""
    out_tokens = np.ascontiguousarray(out_tokens, dtype=np.int32)
    B, W = out_tokens.shape
    accept_len = np.ascontiguousarray(accept_len, dtype=np.int32).reshape(B)
    win = None if window is None else np.ascontiguousarray(window, dtype=np.int32).reshape(B, W)
    nw = np.empty((B, W), np.int32) if next_window else None
    sq = None if seq is None else np.array(seq, dtype=np.int32, copy=True, order="C")
    sl = None if seq_len is None else np.array(seq_len, dtype=np.int32, copy=True).reshape(B)
    full = np.zeros(((B + 31) // 32,), np.uint32)
    cap = 0 if sq is None else sq.shape[1]
    rc = (L or lib()).svo_epilogue(_ptr(win), _ptr(out_tokens), _ptr(accept_len), B, W - 1,
                                   _ptr(nw), _ptr(sq), cap, _ptr(sl), _ptr(full))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    bits = np.array([(full[b // 32] >> (b % 32)) & 1 for b in range(B)], bool)
    return dict(next_window=nw, seq=sq, seq_len=sl, full=bits)


def row_topk(row, k, L=None):
    """Indices of the k largest logits of a row (logit desc, index asc)."""
    row = np.ascontiguousarray(row)
    idx = np.empty(k, np.int32)
    (L or lib()).svo_row_topk(_ptr(row), row.shape[-1], _dtype_code(row), int(k), _ptr(idx))
    return idx


def ssd_lookup(out_tokens, accept_len, keys_al, keys_token, spec=None, L=None):
    """The outcome lookup (svo_ssd_lookup).  out_tokens [B, D_max+1], accept_len [B],
    keys_al / keys_token [B, K], spec [B, K, S] or None.
    Returns dict(hit [B], spec [B, S] or None)."""
    out_tokens = np.ascontiguousarray(out_tokens, dtype=np.int32)
    B, W = out_tokens.shape
    accept_len = np.ascontiguousarray(accept_len, dtype=np.int32).reshape(B)
    keys_al = np.ascontiguousarray(keys_al, dtype=np.int32)
    keys_token = np.ascontiguousarray(keys_token, dtype=np.int32)
    assert keys_al.shape == keys_token.shape and keys_al.shape[0] == B
    K = keys_al.shape[1]
    S = 0
    if spec is not None:
        spec = np.ascontiguousarray(spec, dtype=np.int32)
        assert spec.ndim == 3 and spec.shape[:2] == (B, K)
        S = spec.shape[2]
    hit = np.empty(B, np.int32)
    osp = np.empty((B, S), np.int32) if spec is not None else None
    rc = (L or lib()).svo_ssd_lookup(_ptr(out_tokens), _ptr(accept_len), B, W - 1, _ptr(keys_al),
                                     _ptr(keys_token), K, _ptr(spec), S, _ptr(hit), _ptr(osp))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    return dict(hit=hit, spec=osp)


def verify_tree(target, draft, tokens, parents, n_nodes=None, *, temperature=1.0, mode=SVO_STOCHASTIC,
                seed=0, request_offset=0, nthreads=1, L=None):
    """Tree verification on host arrays (svo_verify_tree): target [B, N+1, V],
    draft [B, N, V] (or None when greedy), tokens and parents [B, N] int32,
    n_nodes [B] or None.  Returns dict(tokens [B, N+1], accept_len [B],
    nodes [B, N], flags [B])."""
    target = np.ascontiguousarray(target)
    B, Np1, V = target.shape
    N = Np1 - 1
    dt = _dtype_code(target)
    if draft is not None:
        draft = np.ascontiguousarray(draft)
        assert draft.dtype == target.dtype and draft.shape == (B, N, V)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, N)
    parents = np.ascontiguousarray(parents, dtype=np.int32).reshape(B, N)
    if n_nodes is not None:
        n_nodes = np.ascontiguousarray(n_nodes, dtype=np.int32).reshape(B)
    out_tokens = np.empty((B, N + 1), np.int32)
    out_al = np.empty((B,), np.int32)
    out_nodes = np.empty((B, N), np.int32)
    out_flags = np.empty((B,), np.uint32)
    rc = (L or lib()).svo_verify_tree(
        _ptr(target), _ptr(draft), _ptr(tokens), _ptr(parents), _ptr(n_nodes), B, N, V, dt,
        float(temperature), int(mode), int(seed) & (2**64 - 1), int(request_offset),
        _ptr(out_tokens), _ptr(out_al), _ptr(out_nodes), _ptr(out_flags), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    return dict(tokens=out_tokens, accept_len=out_al, nodes=out_nodes, flags=out_flags)
