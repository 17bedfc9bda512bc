"""Python binding of libsa.so: argument marshalling only.

Every function here passes raw device pointers, sizes and the current CUDA
stream to the C ABI declared in ``include/sa.h``; every step of the path runs
in the library's CUDA kernels.  torch is used for device memory (outputs and
workspaces) and streams.  If ``libsa.so`` is missing the import of a compute
function fails loudly; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsa.so")
LIB_DEBUG_PATH = os.path.join(_HERE, "libsa_debug.so")

SA_OK = 0
SA_ERR_INVALID_ARG = 1
SA_ERR_UNSUPPORTED = 2
SA_ERR_WORKSPACE = 3
SA_ERR_CUDA = 4
SA_ERR_TIMEOUT = 5
SA_ERR_STALE_INDEX = 6
SA_MAX_K = 4096
SA_WS_ALIGN = 256

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/sa.h
SIGNATURES = {
    "sa_status_string": (ctypes.c_char_p, [_I]),
    "sa_last_error": (ctypes.c_char_p, []),
    "sa_version": (_I, []),
    "sa_index_score_topk_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "sa_index_score_topk": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "sa_index_score_topk_mh_workspace": (_Z, [_I, _I, _I, _I, _I, _I]),
    "sa_index_score_topk_mh": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "sa_index_score_topk_fp8_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "sa_workspace_status": (_I, [_P, _P]),
    "sa_index_score_topk_fp8": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "sa_sparse_attn_prefill": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P]),
    "sa_sparse_attn_decode_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "sa_sparse_attn_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _Z, _P]),
    "sa_sparse_attn_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P]),
    "sa_gather_rows": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "sa_sparse_attn_decode_rows": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P, _P, _Z, _P]),
    "sa_self_test_bounded_wait": (_I, [_P, ctypes.c_uint32, _P]),
    "sa_gist_route_unfold_workspace": (_Z, [_I, _I, _I, _I]),
    "sa_gist_route_unfold": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "sa_hier_gist_route_unfold": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "sa_index_overlap": (_I, [_P, _P, _P, _P, _I, _I, _P, _P]),
    "sa_index_pattern_greedy": (_I, [_P, _I, _I, ctypes.c_char_p]),
    "sa_debug_enabled": (_I, []),
    "sa_debug_read": (_I, [_P, _I]),
    "sa_debug_check_canary": (_I, [_P, _Z, _I, _P]),
    "sa_index_cache_create": (_I, [_I, ctypes.c_char_p, _I, _I, _I, _I, _P, _P, ctypes.POINTER(_P)]),
    "sa_index_cache_destroy": (None, [_P]),
    "sa_index_cache_is_full": (_I, [_P, _I]),
    "sa_index_cache_owner": (_I, [_P, _I]),
    "sa_index_cache_begin_step": (_I, [_P]),
    "sa_index_cache_update": (_I, [_P, _I, _P, _P, _I, _I, _I, _I, _P, _P, _Z, _P]),
    "sa_index_cache_mark_written": (_I, [_P, _I]),
    "sa_index_cache_get": (_I, [_P, _I, ctypes.POINTER(_P), ctypes.POINTER(_P),
                                ctypes.POINTER(ctypes.c_uint64)]),
}

_lib = None
_lock = threading.Lock()


class SAError(RuntimeError):
    def __init__(self, status: int, func: str, detail: str):
        super().__init__(f"{func} -> {status_string(status)}: {detail}")
        self.status = status


def lib():
    """The loaded libsa.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"libsa.so not found at {LIB_PATH}; build it with "
                        "`python -m shared_top_routing_b200.build` (no fallback exists)")
                L = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    f = getattr(L, name)
                    f.restype = res
                    f.argtypes = args
                _lib = L
    return _lib


_lib_debug = None


def lib_debug():
    """The debug build libsa_debug.so (same ABI; see sa.h), loaded on its own."""
    global _lib_debug
    if _lib_debug is None:
        with _lock:
            if _lib_debug is None:
                if not os.path.exists(LIB_DEBUG_PATH):
                    raise RuntimeError(f"libsa_debug.so not found at {LIB_DEBUG_PATH}; build it with "
                                       "`python -m shared_top_routing_b200.build --debug`")
                L = ctypes.CDLL(LIB_DEBUG_PATH)
                for name, (res, args) in SIGNATURES.items():
                    f = getattr(L, name)
                    f.restype = res
                    f.argtypes = args
                _lib_debug = L
    return _lib_debug


def debug_read(L=None, reset: bool = True):
    """The debug record {code, detail, detail, count} of a library (see sa.h)."""
    rec = (ctypes.c_int32 * 4)()
    st = (L or lib_debug()).sa_debug_read(ctypes.cast(rec, ctypes.c_void_p), 1 if reset else 0)
    if st != SA_OK:
        raise SAError(st, "sa_debug_read", last_error())
    return list(rec)


def status_string(s: int) -> str:
    return lib().sa_status_string(s).decode()


def last_error() -> str:
    return lib().sa_last_error().decode()


def _check(status: int, func: str):
    if status != SA_OK:
        raise SAError(status, func, last_error())


# ------------------------------------------------------------ torch plumbing

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype_size, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.element_size() != dtype_size:
        raise ValueError(f"{name} must have {dtype_size}-byte elements")


_ws_cache: dict = {}


def workspace(nbytes: int, device, key: str = "", stream=None):
    """A cached, zero-filled device workspace of at least ``nbytes`` (256-byte
    aligned).  The decode-attention workspace must start zero-filled; the
    library returns its ticket region to zero after each call, so the cache
    can hand the same buffer to later calls of any shape."""
    torch = _torch()
    if nbytes <= 0:
        return None
    s = stream if stream is not None else torch.cuda.current_stream(device)
    k = (str(device), s.cuda_stream, key)
    buf = _ws_cache.get(k)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[k] = buf
    return buf


# --------------------------------------------------------------- the calls

def sa_index_score_topk(q_idx, k_idx, k: int, Tk: int | None = None, q_pos0: int | None = None,
                        kv_len=None, idx_out=None, count_out=None, with_scores: bool = False,
                        ws=None, stream=None):
    """Indexer scores + per-query top-k (see sa.h).

    q_idx [B, Tq, d] or [B, d] (decode) bf16; k_idx [B, Tk_max, d] bf16.
    Tk defaults to Tk_max; q_pos0 defaults to Tk - Tq (prefill whose queries
    are the last Tq cached tokens; for decode Tk - 1).
    Returns (idx [B, Tq, k] int32, count [B, Tq] int32[, score [B, Tq, k] fp32]).
    """
    torch = _torch()
    decode_shape = q_idx.dim() == 2
    q3 = q_idx.unsqueeze(1) if decode_shape else q_idx
    B, Tq, d = q3.shape
    Tk_max = k_idx.shape[1]
    Tk = Tk_max if Tk is None else Tk
    q_pos0 = Tk - Tq if q_pos0 is None else q_pos0
    _need(q3, "q_idx", 2)
    _need(k_idx, "k_idx", 2)
    dev = q3.device
    if idx_out is None:
        idx_out = torch.empty((B, Tq, k), dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty((B, Tq), dtype=torch.int32, device=dev)
    score = torch.empty((B, Tq, k), dtype=torch.float32, device=dev) if with_scores else None
    need = lib().sa_index_score_topk_workspace(B, Tq, Tk_max, d, k)
    if ws is None:
        ws = workspace(need, dev, "index", stream)
    st = lib().sa_index_score_topk(_ptr(q3), _ptr(k_idx), B, Tq, Tk, Tk_max, d, k, q_pos0,
                                   _ptr(kv_len), _ptr(idx_out), _ptr(count_out), _ptr(score),
                                   _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "sa_index_score_topk")
    if decode_shape:
        idx_v, cnt_v = idx_out.view(B, k), count_out.view(B)
        return (idx_v, cnt_v, score.view(B, k)) if with_scores else (idx_v, cnt_v)
    return (idx_out, count_out, score) if with_scores else (idx_out, count_out)


def sa_index_score_topk_mh(q_idx, w, k_idx, k: int, Tk: int | None = None, q_pos0: int | None = None,
                           kv_len=None, idx_out=None, count_out=None, with_scores: bool = False,
                           ws=None, stream=None):
    """Multi-head weighted indexer scores + per-query top-k (see sa.h).

    q_idx [B, Tq, H, d] or [B, H, d] (decode) bf16; w [B, Tq, H] or [B, H]
    fp32; k_idx [B, Tk_max, d] bf16.  Defaults and results as for
    sa_index_score_topk.
    """
    torch = _torch()
    decode_shape = q_idx.dim() == 3
    q4 = q_idx.unsqueeze(1) if decode_shape else q_idx
    w3 = w.unsqueeze(1) if decode_shape else w
    B, Tq, H, d = q4.shape
    Tk_max = k_idx.shape[1]
    Tk = Tk_max if Tk is None else Tk
    q_pos0 = Tk - Tq if q_pos0 is None else q_pos0
    _need(q4, "q_idx", 2)
    _need(w3, "w", 4)
    _need(k_idx, "k_idx", 2)
    dev = q4.device
    if idx_out is None:
        idx_out = torch.empty((B, Tq, k), dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty((B, Tq), dtype=torch.int32, device=dev)
    score = torch.empty((B, Tq, k), dtype=torch.float32, device=dev) if with_scores else None
    need = lib().sa_index_score_topk_mh_workspace(B, Tq, Tk_max, H, d, k)
    if ws is None:
        ws = workspace(need, dev, "index_mh", stream)
    st = lib().sa_index_score_topk_mh(_ptr(q4), _ptr(w3), _ptr(k_idx), B, Tq, H, Tk, Tk_max, d, k, q_pos0,
                                      _ptr(kv_len), _ptr(idx_out), _ptr(count_out), _ptr(score),
                                      _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "sa_index_score_topk_mh")
    if decode_shape:
        idx_v, cnt_v = idx_out.view(B, k), count_out.view(B)
        return (idx_v, cnt_v, score.view(B, k)) if with_scores else (idx_v, cnt_v)
    return (idx_out, count_out, score) if with_scores else (idx_out, count_out)


def sa_index_score_topk_fp8(q_idx, k_idx, k: int, w=None, Tk: int | None = None, q_pos0: int | None = None,
                            kv_len=None, idx_out=None, count_out=None, with_scores: bool = False,
                            ws=None, stream=None):
    """fp8 (E4M3) indexer scores + top-k of one decode query per sequence
    (see sa.h).

    q_idx [B, d] (one head) or [B, H, d]; k_idx [B, Tk_max, d]: E4M3 codes as
    uint8 (or torch.float8_e4m3fn) tensors.  w [B, H] fp32 selects the
    multi-head score; without it H must be 1.  Tk defaults to Tk_max, q_pos0
    to Tk - 1.  Returns (idx [B, k] int32, count [B] int32[, score [B, k]]).
    """
    torch = _torch()
    as_bytes = lambda t: t.view(torch.uint8) if t.dtype != torch.uint8 else t
    q3 = as_bytes(q_idx)
    q3 = q3.unsqueeze(1) if q3.dim() == 2 else q3
    kb = as_bytes(k_idx)
    B, H, d = q3.shape
    Tk_max = kb.shape[1]
    Tk = Tk_max if Tk is None else Tk
    q_pos0 = Tk - 1 if q_pos0 is None else q_pos0
    _need(q3, "q_idx", 1)
    _need(kb, "k_idx", 1)
    if w is not None:
        _need(w, "w", 4)
    dev = q3.device
    if idx_out is None:
        idx_out = torch.empty((B, k), dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty((B,), dtype=torch.int32, device=dev)
    score = torch.empty((B, k), dtype=torch.float32, device=dev) if with_scores else None
    need = lib().sa_index_score_topk_fp8_workspace(B, Tk_max, H, d, k)
    if ws is None:
        ws = workspace(need, dev, "index", stream)
    st = lib().sa_index_score_topk_fp8(_ptr(q3), _ptr(w), _ptr(kb), B, H, Tk, Tk_max, d, k, q_pos0, _ptr(kv_len),
                                       _ptr(idx_out), _ptr(count_out), _ptr(score), _ptr(ws),
                                       0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "sa_index_score_topk_fp8")
    return (idx_out, count_out, score) if with_scores else (idx_out, count_out)


def sa_workspace_status(ws, stream=None) -> int:
    """The status the error word at the start of a workspace reports (see
    sa.h): SA_OK, or SA_ERR_TIMEOUT when a kernel wait of a call that used it
    gave up.  Synchronizes `stream`."""
    return lib().sa_workspace_status(_ptr(ws), _stream(stream))


def sa_sparse_attn_prefill(q, k_cache, v_cache, idx, count, scale: float = 0.0, out=None,
                           with_lse: bool = False, stream=None):
    """q [B, T, Hq, D]; k_cache/v_cache [B, Tk_max, Hkv, D]; idx [B, T, k]; count [B, T]."""
    torch = _torch()
    B, T, Hq, D = q.shape
    _, Tk_max, Hkv, _ = k_cache.shape
    k = idx.shape[-1]
    for t, n, sz in ((q, "q", 2), (k_cache, "k_cache", 2), (v_cache, "v_cache", 2),
                     (idx, "idx", 4), (count, "count", 4)):
        _need(t, n, sz)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((B, T, Hq), dtype=torch.float32, device=q.device) if with_lse else None
    st = lib().sa_sparse_attn_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx), _ptr(count),
                                      B, T, Tk_max, Hq, Hkv, D, k, scale, _ptr(out), _ptr(lse),
                                      _stream(stream))
    _check(st, "sa_sparse_attn_prefill")
    return (out, lse) if with_lse else out


def sa_sparse_attn_decode(q, k_cache, v_cache, idx, count, scale: float = 0.0, out=None,
                          with_lse: bool = False, ws=None, stream=None):
    """q [B, Hq, D]; k_cache/v_cache [B, Tk_max, Hkv, D]; idx [B, k]; count [B]."""
    torch = _torch()
    B, Hq, D = q.shape
    _, Tk_max, Hkv, _ = k_cache.shape
    k = idx.shape[-1]
    for t, n, sz in ((q, "q", 2), (k_cache, "k_cache", 2), (v_cache, "v_cache", 2),
                     (idx, "idx", 4), (count, "count", 4)):
        _need(t, n, sz)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if with_lse else None
    need = lib().sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k)
    if ws is None:
        ws = workspace(need, q.device, "attn_decode", stream)
    st = lib().sa_sparse_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx), _ptr(count),
                                     B, Tk_max, Hq, Hkv, D, k, scale, _ptr(out), _ptr(lse),
                                     _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
    _check(st, "sa_sparse_attn_decode")
    return (out, lse) if with_lse else out


def sa_gather_rows(k_cache, v_cache, idx, count, k_rows=None, v_rows=None, stream=None):
    """Compact copies [B, k, Hkv * D + 8] of the selected rows (zeros past
    count; the last 8 values of each row are a zero pad, see sa.h)."""
    torch = _torch()
    B, Tk_max, Hkv, D = k_cache.shape
    k = idx.shape[-1]
    for t, n, sz in ((k_cache, "k_cache", 2), (v_cache, "v_cache", 2), (idx, "idx", 4), (count, "count", 4)):
        _need(t, n, sz)
    if k_rows is None:
        k_rows = torch.empty((B, k, Hkv * D + 8), dtype=k_cache.dtype, device=k_cache.device)
    if v_rows is None:
        v_rows = torch.empty((B, k, Hkv * D + 8), dtype=v_cache.dtype, device=v_cache.device)
    st = lib().sa_gather_rows(_ptr(k_cache), _ptr(v_cache), _ptr(idx), _ptr(count), B, Tk_max, Hkv, D, k,
                              _ptr(k_rows), _ptr(v_rows), _stream(stream))
    _check(st, "sa_gather_rows")
    return k_rows, v_rows


def sa_sparse_attn_decode_rows(q, k_rows, v_rows, count, scale: float = 0.0, out=None, with_lse: bool = False,
                               ws=None, stream=None):
    """q [B, Hq, D]; k_rows / v_rows [B, k, Hkv * D + 8] compact rows (from
    sa_gather_rows); count [B]."""
    torch = _torch()
    B, Hq, D = q.shape
    _, k, row = k_rows.shape
    Hkv = (row - 8) // D
    for t, n, sz in ((q, "q", 2), (k_rows, "k_rows", 2), (v_rows, "v_rows", 2), (count, "count", 4)):
        _need(t, n, sz)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if with_lse else None
    need = lib().sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k)
    if ws is None:
        ws = workspace(need, q.device, "attn_decode", stream)
    st = lib().sa_sparse_attn_decode_rows(_ptr(q), _ptr(k_rows), _ptr(v_rows), _ptr(count), B, Hq, Hkv, D, k,
                                          scale, _ptr(out), _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel(),
                                          _stream(stream))
    _check(st, "sa_sparse_attn_decode_rows")
    return (out, lse) if with_lse else out


def sa_sparse_attn_decode_noalloc(q, k_cache, v_cache, idx, count, scale: float = 0.0, out=None,
                                  with_lse: bool = False, stream=None):
    """sa_sparse_attn_decode for callers that cannot allocate: no workspace
    argument; the library's fixed scratch array is used (see sa.h)."""
    torch = _torch()
    B, Hq, D = q.shape
    _, Tk_max, Hkv, _ = k_cache.shape
    k = idx.shape[-1]
    for t, n, sz in ((q, "q", 2), (k_cache, "k_cache", 2), (v_cache, "v_cache", 2),
                     (idx, "idx", 4), (count, "count", 4)):
        _need(t, n, sz)
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if with_lse else None
    st = lib().sa_sparse_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx),
                                             _ptr(count), B, Tk_max, Hq, Hkv, D, k, scale, _ptr(out),
                                             _ptr(lse), _stream(stream))
    _check(st, "sa_sparse_attn_decode_noalloc")
    return (out, lse) if with_lse else out


def sa_self_test_bounded_wait(poll_limit: int = 4096, stream=None):
    """Runs the library's bounded-wait probe on the GPU and returns its five
    result words (see sa.h): a wait nothing completes must give up with code
    77 and set its abort flag; a wait that completes must succeed."""
    import torch
    err = torch.zeros(5, dtype=torch.int32, device="cuda")
    st = lib().sa_self_test_bounded_wait(_ptr(err), poll_limit, _stream(stream))
    _check(st, "sa_self_test_bounded_wait")
    return err


def sa_gist_route_unfold(q_route, gist_key, chunk_len: int, k_chunks: int, partial_len,
                         rows_out=None, count_out=None, with_chunks: bool = False, ws=None,
                         stream=None):
    """q_route [B, d]; gist_key [B, n_chunks, d]; partial_len [B] int32 (device).
    Returns (rows [B, k_chunks*(chunk_len+1)+chunk_len], count [B][, chunks [B, k_chunks]])."""
    torch = _torch()
    B, d = q_route.shape
    n_chunks = gist_key.shape[1]
    _need(q_route, "q_route", 2)
    _need(gist_key, "gist_key", 2)
    _need(partial_len, "partial_len", 4)
    dev = q_route.device
    stride = k_chunks * (chunk_len + 1) + chunk_len
    if rows_out is None:
        rows_out = torch.empty((B, stride), dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty((B,), dtype=torch.int32, device=dev)
    chunks = torch.empty((B, k_chunks), dtype=torch.int32, device=dev) if with_chunks else None
    need = lib().sa_gist_route_unfold_workspace(B, n_chunks, d, k_chunks)
    if ws is None:
        ws = workspace(need, dev, "gist", stream)
    st = lib().sa_gist_route_unfold(_ptr(q_route), _ptr(gist_key), B, n_chunks, chunk_len, d,
                                    k_chunks, _ptr(partial_len), _ptr(rows_out), _ptr(count_out),
                                    _ptr(chunks), _ptr(ws), 0 if ws is None else ws.numel(),
                                    _stream(stream))
    _check(st, "sa_gist_route_unfold")
    return (rows_out, count_out, chunks) if with_chunks else (rows_out, count_out)


def sa_hier_gist_route_unfold(q_route, meta_key, gist_key, chunk_len: int, group_size: int, k_groups: int,
                              k_chunks: int, partial_len=None, rows_out=None, count_out=None,
                              with_chunks: bool = False, with_groups: bool = False, stream=None):
    """Two-level gist routing (see sa.h).  q_route [B, d]; meta_key
    [B, n_chunks // group_size, d]; gist_key [B, n_chunks, d].
    Returns (rows, count[, chunks][, groups])."""
    torch = _torch()
    B, d = q_route.shape
    n_chunks = gist_key.shape[1]
    _need(q_route, "q_route", 2)
    _need(meta_key, "meta_key", 2)
    _need(gist_key, "gist_key", 2)
    if partial_len is not None:
        _need(partial_len, "partial_len", 4)
    dev = q_route.device
    stride = k_chunks * (chunk_len + 1) + chunk_len
    if rows_out is None:
        rows_out = torch.empty((B, stride), dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty((B,), dtype=torch.int32, device=dev)
    chunks = torch.empty((B, k_chunks), dtype=torch.int32, device=dev) if with_chunks else None
    groups = torch.empty((B, k_groups), dtype=torch.int32, device=dev) if with_groups else None
    st = lib().sa_hier_gist_route_unfold(_ptr(q_route), _ptr(meta_key), _ptr(gist_key), B, n_chunks, chunk_len,
                                         group_size, d, k_groups, k_chunks, _ptr(partial_len), _ptr(rows_out),
                                         _ptr(count_out), _ptr(chunks), _ptr(groups), _stream(stream))
    _check(st, "sa_hier_gist_route_unfold")
    res = [rows_out, count_out]
    if with_chunks:
        res.append(chunks)
    if with_groups:
        res.append(groups)
    return tuple(res)


def sa_index_overlap(idx_a, count_a, idx_b, count_b, out=None, stream=None):
    """Per-row count of the positions two selections share.  idx_* [..., k]
    int32 (ascending rows); count_* [...] int32.  Returns int32 [rows]."""
    torch = _torch()
    k = idx_a.shape[-1]
    rows = idx_a.numel() // k
    for t, n in ((idx_a, "idx_a"), (idx_b, "idx_b"), (count_a, "count_a"), (count_b, "count_b")):
        _need(t, n, 4)
    if out is None:
        out = torch.empty((rows,), dtype=torch.int32, device=idx_a.device)
    st = lib().sa_index_overlap(_ptr(idx_a), _ptr(count_a), _ptr(idx_b), _ptr(count_b), rows, k, _ptr(out),
                                _stream(stream))
    _check(st, "sa_index_overlap")
    return out


def sa_index_pattern_greedy(overlap, n_full: int) -> str:
    """Greedy layer-role search on an [L, L] overlap matrix (host; see sa.h)."""
    import numpy as np
    ov = np.ascontiguousarray(np.asarray(overlap, dtype=np.float64))
    L = ov.shape[0]
    buf = ctypes.create_string_buffer(L + 1)
    st = lib().sa_index_pattern_greedy(ov.ctypes.data_as(ctypes.c_void_p), L, n_full, buf)
    _check(st, "sa_index_pattern_greedy")
    return buf.value.decode()


class IndexCache:
    """Shared index cache: full layers run the indexer into one buffer, shared
    layers read it (see sa_index_cache_* in sa.h).  The buffers are device
    tensors owned by this object (or passed in)."""

    def __init__(self, n_layers: int, B: int, Tq: int, k: int, pattern: str | None = None,
                 share_every: int = 4, device=None, idx_buf=None, count_buf=None):
        self._h = None
        self.idx_buf = idx_buf
        self.count_buf = count_buf
        if B > 0 and (idx_buf is None or count_buf is None):
            torch = _torch()
            self.idx_buf = torch.empty((B, Tq, k), dtype=torch.int32, device=device)
            self.count_buf = torch.empty((B, Tq), dtype=torch.int32, device=device)
        h = ctypes.c_void_p()
        pat = pattern.encode() if pattern is not None else None
        st = lib().sa_index_cache_create(n_layers, pat, share_every, B, Tq, k,
                                         _ptr(self.idx_buf), _ptr(self.count_buf), ctypes.byref(h))
        _check(st, "sa_index_cache_create")
        self._h = h
        self.n_layers, self.B, self.Tq, self.k = n_layers, B, Tq, k

    def close(self):
        if self._h is not None and self._h.value:
            lib().sa_index_cache_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def is_full(self, layer: int) -> int:
        return lib().sa_index_cache_is_full(self._h, layer)

    def owner(self, layer: int) -> int:
        return lib().sa_index_cache_owner(self._h, layer)

    def begin_step(self):
        _check(lib().sa_index_cache_begin_step(self._h), "sa_index_cache_begin_step")

    def mark_written(self, layer: int):
        _check(lib().sa_index_cache_mark_written(self._h, layer), "sa_index_cache_mark_written")

    def update(self, layer: int, q_idx, k_idx, Tk: int | None = None, q_pos0: int | None = None,
               kv_len=None, ws=None, stream=None):
        q3 = q_idx.unsqueeze(1) if q_idx.dim() == 2 else q_idx
        B, Tq, d = q3.shape
        Tk_max = k_idx.shape[1]
        Tk = Tk_max if Tk is None else Tk
        q_pos0 = Tk - Tq if q_pos0 is None else q_pos0
        need = lib().sa_index_score_topk_workspace(B, Tq, Tk_max, d, self.k)
        if ws is None:
            ws = workspace(need, q3.device, "index", stream)
        st = lib().sa_index_cache_update(self._h, layer, _ptr(q3), _ptr(k_idx), Tk, Tk_max, d, q_pos0,
                                         _ptr(kv_len), _ptr(ws), 0 if ws is None else ws.numel(),
                                         _stream(stream))
        _check(st, "sa_index_cache_update")

    def get(self, layer: int):
        """(idx_ptr, count_ptr, version) for `layer`; raises SAError on a stale read."""
        ip, cp, ver = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_uint64()
        st = lib().sa_index_cache_get(self._h, layer, ctypes.byref(ip), ctypes.byref(cp),
                                      ctypes.byref(ver))
        _check(st, "sa_index_cache_get")
        return ip.value, cp.value, ver.value

    def get_tensors(self, layer: int):
        """The index buffers for `layer` (checked against the C object)."""
        ip, cp, ver = self.get(layer)
        assert ip == self.idx_buf.data_ptr() and cp == self.count_buf.data_ptr()
        return self.idx_buf, self.count_buf, ver
