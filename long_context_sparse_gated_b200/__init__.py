"""Python binding of libcsa, the B200 (sm_100a) CSA/HCA hot-path library.

The five calls keep the C ABI's names (see include/csa.h):

    csa_compress, hca_compress, csa_index_topk, csa_sparse_attn, hca_dense_attn

This module only marshals arguments: it turns CUDA tensors into device
pointers and a torch stream into a cudaStream_t, and raises on a non-OK
status.  Every step of the computation runs in the library's kernels.  There
is no CPU fallback: without libcsa.so or without CUDA tensors the calls fail
loudly.
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "CsaParams", "CsaKv", "CsaError", "lib", "make_params",
    "csa_compress", "hca_compress", "csa_index_topk", "csa_sparse_attn", "hca_dense_attn",
    "csa_index_topk_workspace_bytes", "csa_sparse_attn_workspace_bytes",
    "hca_dense_attn_workspace_bytes", "csa_index_topk_noalloc", "csa_index_compress", "csa_index_quantize",
    "CsaState", "CsaCkpt", "csa_state_append", "csa_state_restore", "KV_F32", "KV_FP8_BF16", "IDX_F32", "IDX_MXFP4",
    "ACT_F32", "ACT_BF16", "SCORE_F32", "SCORE_BF16", "DEV_ERR_INDEX", "DEV_ERR_RANGE",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa.so")

KV_F32, KV_FP8_BF16 = 0, 1
SCORE_F32, SCORE_BF16 = 0, 1
IDX_F32, IDX_MXFP4 = 0, 1
ACT_F32, ACT_BF16 = 0, 1
DEV_ERR_INDEX, DEV_ERR_RANGE = 1, 2

STATUS = {0: "CSA_OK", -1: "CSA_ERR_INVALID", -2: "CSA_ERR_UNSUPPORTED", -3: "CSA_ERR_ALIGN",
          -4: "CSA_ERR_WORKSPACE", -5: "CSA_ERR_LAUNCH"}

EXPORTS = ["csa_compress", "hca_compress", "csa_index_topk", "csa_index_topk_workspace_bytes",
           "csa_sparse_attn", "csa_sparse_attn_workspace_bytes", "hca_dense_attn",
           "hca_dense_attn_workspace_bytes", "csa_status_string", "csa_last_error_string",
           "csa_index_topk_noalloc", "csa_index_compress", "csa_index_quantize", "csa_state_append",
           "csa_state_restore"]


class CsaError(RuntimeError):
    def __init__(self, name, status, detail=""):
        super().__init__(f"{name} returned {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))
        self.status = status


class CsaParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "d", "r", "m", "n_idx_heads", "idx_dim", "topk", "n_heads", "window",
                 "kv_fmt", "idx_fmt", "act_fmt")] + \
               [(n, ctypes.c_float) for n in ("softmax_scale", "rope_theta", "eps")] + \
               [("score_fmt", ctypes.c_int32)]


class CsaKv(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("cap", ctypes.c_int64)]


class CsaState(ctypes.Structure):
    _fields_ = [("win", CsaKv), ("a", ctypes.c_void_p), ("b", ctypes.c_void_p), ("gate", ctypes.c_void_p),
                ("s_cap", ctypes.c_int64)]


class CsaCkpt(ctypes.Structure):
    _fields_ = [("win_rows", ctypes.c_void_p), ("win_scale", ctypes.c_void_p), ("a", ctypes.c_void_p),
                ("b", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("n_slots", ctypes.c_int32),
                ("every", ctypes.c_int32)]


_lib = None

_P = ctypes.POINTER(CsaParams)
_V = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t


def lib(path: str | None = None):
    """Load libcsa.so (built by ``long_context_sparse_gated_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libcsa.so not built at {path}; run python -m long_context_sparse_gated_b200.build")
    L = ctypes.CDLL(path)
    comp = [_P, _V, _V, _V, _I64, _V, _V, _V, _I32, _V, CsaKv, _V, _V, _V]
    L.csa_compress.argtypes = comp
    L.hca_compress.argtypes = comp
    L.csa_index_topk.argtypes = [_P, _V, _V, _V, _V, _V, _I64, _V, _I32, _I32, _V, _V, _SZ, _V, _V]
    L.csa_index_topk_workspace_bytes.argtypes = [_P, _I32, _I32]
    L.csa_index_topk_workspace_bytes.restype = _SZ
    L.csa_index_topk_noalloc.argtypes = [_P, _V, _V, _V, _V, _V, _I64, _V, _I32, _I32, _V, _V, _V]
    L.csa_index_topk_noalloc.restype = _I32
    L.csa_sparse_attn.argtypes = [_P, _V, CsaKv, _V, CsaKv, _V, _V, _I32, _V, _V, _SZ, _V, _V]
    L.csa_sparse_attn_workspace_bytes.argtypes = [_P, _I32]
    L.csa_sparse_attn_workspace_bytes.restype = _SZ
    L.hca_dense_attn.argtypes = [_P, _V, CsaKv, CsaKv, _V, _V, _I32, _I32, _V, _V, _SZ, _V, _V]
    L.hca_dense_attn_workspace_bytes.argtypes = [_P, _I32, _I32]
    L.hca_dense_attn_workspace_bytes.restype = _SZ
    L.csa_index_compress.argtypes = [_P, _V, _V, _V, _I64, _V, _V, _V, _I32, _I32, _V, _V, _V, _I64, _V, _V]
    L.csa_index_compress.restype = _I32
    L.csa_index_quantize.argtypes = [_P, _V, _I64, _V, _V, _V]
    L.csa_index_quantize.restype = _I32
    L.csa_state_append.argtypes = [_P, _V, _V, _V, _V, _V, _I32, CsaState, CsaKv, _V, ctypes.POINTER(CsaCkpt),
                                   _V, _V]
    L.csa_state_append.restype = _I32
    L.csa_state_restore.argtypes = [_P, _V, ctypes.POINTER(CsaCkpt), CsaState, _V, _V]
    L.csa_state_restore.restype = _I32
    L.csa_status_string.argtypes = [_I32]
    L.csa_status_string.restype = ctypes.c_char_p
    L.csa_last_error_string.argtypes = []
    L.csa_last_error_string.restype = ctypes.c_char_p
    for n in ("csa_compress", "hca_compress", "csa_index_topk", "csa_sparse_attn", "hca_dense_attn"):
        getattr(L, n).restype = _I32
    if path == LIB_PATH:
        _lib = L
    return L


def make_params(*, B, d, r, m, n_idx_heads=1, idx_dim=64, topk=1, n_heads=1, window=1,
                kv_fmt=KV_FP8_BF16, idx_fmt=IDX_MXFP4, act_fmt=ACT_BF16, softmax_scale=1.0,
                rope_theta=1e4, eps=1e-6, score_fmt=SCORE_F32) -> CsaParams:
    return CsaParams(B, d, r, m, n_idx_heads, idx_dim, topk, n_heads, window, kv_fmt, idx_fmt,
                     act_fmt, softmax_scale, rope_theta, eps, score_fmt)


def _ptr(t):
    """Device pointer of a CUDA tensor (None -> NULL).  Host tensors are
    rejected: the library takes device pointers only."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not getattr(t, "is_cuda", False):
        raise TypeError("libcsa takes CUDA tensors (device pointers); got a host array")
    if not t.is_contiguous():
        raise ValueError("libcsa takes C-contiguous tensors")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _kv(rows, scale):
    return CsaKv(_ptr(rows), _ptr(scale), rows.shape[1])


def _check(name, st):
    if st != 0:
        detail = lib().csa_last_error_string().decode() if st == -5 else ""
        raise CsaError(name, st, detail)


def csa_compress(params, a, b, gate, tok_base, e_begin, e_end, max_entries, out_rows, out_scale=None,
                 out_pos=None, norm_w=None, err=None, stream=None, _name="csa_compress"):
    """Gated two-stream compression of entries [e_begin[b], e_end[b]) into
    ``out_rows`` ([B, cap, row_bytes]) / ``out_scale`` ([B, cap])."""
    fn = getattr(lib(), _name)
    st = fn(ctypes.byref(params), _ptr(a), _ptr(b), _ptr(gate), a.shape[1], _ptr(tok_base),
            _ptr(e_begin), _ptr(e_end), int(max_entries), _ptr(norm_w), _kv(out_rows, out_scale),
            _ptr(out_pos), _ptr(err), _stream(stream))
    _check(_name, st)


def hca_compress(params, a, b, gate, tok_base, e_begin, e_end, max_entries, out_rows, out_scale=None,
                 out_pos=None, norm_w=None, err=None, stream=None):
    csa_compress(params, a, b, gate, tok_base, e_begin, e_end, max_entries, out_rows, out_scale,
                 out_pos, norm_w, err, stream, _name="hca_compress")


def csa_index_compress(params, a, b, gate, tok_base, e_begin, e_end, max_entries, rope_dims, k_idx, k_idx_sf,
                       norm_w=None, err=None, stream=None):
    """Index keys of entries [e_begin[b], e_end[b]) from the indexer streams
    ``a``/``b`` ([B, S, idx_dim]) into ``k_idx`` ([B, k_cap, idx_dim/2]) and
    ``k_idx_sf`` ([B, k_cap, idx_dim/32])."""
    st = lib().csa_index_compress(ctypes.byref(params), _ptr(a), _ptr(b), _ptr(gate), a.shape[1], _ptr(tok_base),
                                  _ptr(e_begin), _ptr(e_end), int(max_entries), int(rope_dims), _ptr(norm_w),
                                  _ptr(k_idx), _ptr(k_idx_sf), k_idx.shape[1], _ptr(err), _stream(stream))
    _check("csa_index_compress", st)


def csa_index_quantize(params, x, out, out_sf, stream=None):
    """Rows of ``x`` ([..., idx_dim]) to MXFP4 ``out`` ([..., idx_dim/2]) and
    ``out_sf`` ([..., idx_dim/32])."""
    n_rows = x.numel() // params.idx_dim
    st = lib().csa_index_quantize(ctypes.byref(params), _ptr(x), n_rows, _ptr(out), _ptr(out_sf), _stream(stream))
    _check("csa_index_quantize", st)


def make_state(win_rows, win_scale, a_ring, b_ring, gate_ring):
    """csa_state over device tensors: window ring [B, cap, row] (+ scale
    [B, cap]), stream rings [B, s_cap, d] and gate ring [B, s_cap, 2]."""
    return CsaState(_kv(win_rows, win_scale), _ptr(a_ring), _ptr(b_ring), _ptr(gate_ring), a_ring.shape[1])


def make_ckpt(win_rows, win_scale, a, b, gate, every=1024):
    """csa_ckpt over device tensors [B, n_slots, W, row], [B, n_slots, W],
    [B, n_slots, m, d] (x2), [B, n_slots, m, 2]."""
    return CsaCkpt(_ptr(win_rows), _ptr(win_scale), _ptr(a), _ptr(b), _ptr(gate), win_rows.shape[1], int(every))


def csa_state_append(params, kv_new, a_new, b_new, gate_new, pos0, state, cache_rows, cache_scale=None,
                     cache_pos=None, ckpt=None, err=None, stream=None):
    """Append T = kv_new.shape[1] tokens per sequence at positions pos0[b]..:
    window rows, stream rings, the entries they complete, and (with a
    checkpoint store) the periodic checkpoint."""
    st = lib().csa_state_append(ctypes.byref(params), _ptr(kv_new), _ptr(a_new), _ptr(b_new), _ptr(gate_new),
                                _ptr(pos0), int(kv_new.shape[1]), state, _kv(cache_rows, cache_scale),
                                _ptr(cache_pos), None if ckpt is None else ctypes.byref(ckpt), _ptr(err),
                                _stream(stream))
    _check("csa_state_append", st)


def csa_state_restore(params, pos, ckpt, state, err=None, stream=None):
    """Put the state checkpointed at pos[b] back into the rings."""
    st = lib().csa_state_restore(ctypes.byref(params), _ptr(pos), ctypes.byref(ckpt), state, _ptr(err),
                                 _stream(stream))
    _check("csa_state_restore", st)


def csa_index_topk_workspace_bytes(params, T, n_max):
    return int(lib().csa_index_topk_workspace_bytes(ctypes.byref(params), int(T), int(n_max)))


def csa_sparse_attn_workspace_bytes(params, T):
    return int(lib().csa_sparse_attn_workspace_bytes(ctypes.byref(params), int(T)))


def hca_dense_attn_workspace_bytes(params, T, n_max):
    return int(lib().hca_dense_attn_workspace_bytes(ctypes.byref(params), int(T), int(n_max)))


def csa_index_topk(params, q_idx, q_idx_sf, w, k_idx, k_idx_sf, q_pos0, T, n_max, out_idx, ws,
                   err=None, stream=None):
    """Lightning Indexer + top-k; ``ws`` is a CUDA byte tensor of at least
    csa_index_topk_workspace_bytes(params, T, n_max)."""
    st = lib().csa_index_topk(ctypes.byref(params), _ptr(q_idx), _ptr(q_idx_sf), _ptr(w), _ptr(k_idx),
                              _ptr(k_idx_sf), k_idx.shape[1], _ptr(q_pos0), int(T), int(n_max),
                              _ptr(out_idx), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                              _ptr(err), _stream(stream))
    _check("csa_index_topk", st)


def csa_index_topk_noalloc(params, q_idx, q_idx_sf, w, k_idx, k_idx_sf, q_pos0, T, n_max, out_idx,
                           err=None, stream=None):
    """csa_index_topk without a workspace argument, for callers that cannot
    allocate device memory: the library's static 16 MiB device scratch is
    used instead (shared by every call; overlapping calls race)."""
    st = lib().csa_index_topk_noalloc(ctypes.byref(params), _ptr(q_idx), _ptr(q_idx_sf), _ptr(w),
                                      _ptr(k_idx), _ptr(k_idx_sf), k_idx.shape[1], _ptr(q_pos0), int(T),
                                      int(n_max), _ptr(out_idx), _ptr(err), _stream(stream))
    _check("csa_index_topk_noalloc", st)


def csa_sparse_attn(params, q, cache_rows, cache_scale, idx, win_rows, win_scale, sink, q_pos0, T, out,
                    ws=None, err=None, stream=None):
    st = lib().csa_sparse_attn(ctypes.byref(params), _ptr(q), _kv(cache_rows, cache_scale), _ptr(idx),
                               _kv(win_rows, win_scale), _ptr(sink), _ptr(q_pos0), int(T), _ptr(out),
                               _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                               _ptr(err), _stream(stream))
    _check("csa_sparse_attn", st)


def hca_dense_attn(params, q, cache_rows, cache_scale, win_rows, win_scale, sink, q_pos0, T, n_max, out,
                   ws=None, err=None, stream=None):
    st = lib().hca_dense_attn(ctypes.byref(params), _ptr(q), _kv(cache_rows, cache_scale),
                              _kv(win_rows, win_scale), _ptr(sink), _ptr(q_pos0), int(T), int(n_max),
                              _ptr(out), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                              _ptr(err), _stream(stream))
    _check("hca_dense_attn", st)
