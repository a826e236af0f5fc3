"""Thin Python binding of librat.so, the C ABI of the RAT+ dilated-inference hot path.

Every function here only marshals arguments (torch tensors -> device pointers, the current
CUDA stream) and calls the C entry point of the same name; all computation runs in the CUDA
kernels of librat.so.  There is no fallback: if the library is missing or a call fails, a
RatError is raised.

Entry points (see include/rat.h for layouts and error behaviour):
  rat_recur_prefill         forget-gate recurrence over k and v (chunked associative scan)
  rat_dilated_attn_prefill  causal dilated attention + local window + per-head D
  rat_kv_compress           build / extend the D-fold compressed KV cache
  rat_dilated_decode        one token per sequence against that cache
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "RatError", "lib", "library_path", "F32", "BF16", "KVCache",
    "rat_recur_workspace_bytes", "rat_recur_prefill", "rat_recur_prefill_local",
    "rat_recur_prefill_window", "rat_recur_backward", "rat_recur_backward_local",
    "rat_recur_backward_window",
    "rat_recur_backward_workspace_bytes",
    "rat_dilated_attn_backward", "rat_dilated_attn_backward_workspace_bytes",
    "rat_dilated_attn_prefill",
    "rat_kv_cache_bytes", "rat_kv_compress", "rat_kv_compress_window", "rat_kv_raw_bytes",
    "rat_decode_workspace_bytes", "rat_dilated_decode",
    "rat_workspace_init", "rat_sync_status", "rat_attn_sync_status", "rat_set_attn_block_keys", "rat_attended_keys", "rat_status_string",
    "Workspace", "rat_dilated_decode_noalloc", "PagedKVCache", "make_paged_cache", "AttnOptions",
    "rat_paged_kv_compress", "rat_paged_decode_workspace_bytes", "rat_dilated_decode_paged",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "librat.so")

F32, BF16 = 0, 1
_STATUS = {0: "RAT_OK", -1: "RAT_ERR_INVALID", -2: "RAT_ERR_UNSUPPORTED", -3: "RAT_ERR_CUDA",
           -4: "RAT_ERR_TIMEOUT", -5: "RAT_ERR_WORKSPACE"}


class RatError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (fn, _STATUS.get(status, "?"), status))


class KVCache(ctypes.Structure):
    """Mirror of struct rat_kv_cache (host struct of device pointers)."""
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32), ("W", ctypes.c_int32),
        ("Tcap", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("D", ctypes.POINTER(ctypes.c_int32)),
        ("k_dil", ctypes.c_void_p), ("v_dil", ctypes.c_void_p),
        ("k_win", ctypes.c_void_p), ("v_win", ctypes.c_void_p),
        ("h_k", ctypes.c_void_p), ("h_v", ctypes.c_void_p),
        ("pos", ctypes.c_int64), ("reset_every", ctypes.c_int64),
        ("n_sink", ctypes.c_int32), ("k_sink", ctypes.c_void_p), ("v_sink", ctypes.c_void_p),
        ("window_rec", ctypes.c_int32), ("k_raw", ctypes.c_void_p), ("v_raw", ctypes.c_void_p),
        ("a_raw", ctypes.c_void_p),
    ]


class AttnOptions(ctypes.Structure):
    """Mirror of struct rat_attn_options."""
    _fields_ = [("n_sink", ctypes.c_int32), ("top_k", ctypes.c_int32), ("lse", ctypes.c_void_p)]


class PagedKVCache(ctypes.Structure):
    """Mirror of struct rat_paged_kv_cache (host struct of device pointers)."""
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32), ("W", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("page_entries", ctypes.c_int32), ("max_pages", ctypes.c_int32),
        ("n_pages", ctypes.c_int32),
        ("D", ctypes.POINTER(ctypes.c_int32)),
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
        ("k_win", ctypes.c_void_p), ("v_win", ctypes.c_void_p),
        ("h_k", ctypes.c_void_p), ("h_v", ctypes.c_void_p),
        ("pos", ctypes.c_void_p), ("reset_every", ctypes.c_int64),
    ]


_lib = None
_vp, _sz, _i, _i64, _f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64, ctypes.c_float


def lib():
    """Load librat.so (raises if it has not been built: there is no other implementation)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RatError("load librat.so (run recurrence_augmented_dilated_b200.build)", -3)
        L = ctypes.CDLL(library_path)
        L.rat_status_string.restype = ctypes.c_char_p
        L.rat_status_string.argtypes = [_i]
        L.rat_version.restype = ctypes.c_char_p
        L.rat_workspace_init.argtypes = [_vp, _sz, _vp]
        L.rat_sync_status.argtypes = [_vp, _vp]
        L.rat_recur_workspace_bytes.restype = _sz
        L.rat_recur_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
        L.rat_recur_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _i, _i, _i, _i, _i, _i64, _f, _vp, _sz, _vp]
        L.rat_dilated_attn_backward_workspace_bytes.restype = _sz
        L.rat_dilated_attn_backward_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
        L.rat_dilated_attn_backward.argtypes = [_vp] * 8 + [_i, _i, _i, _i, _i, _i, _i,
                                                            ctypes.POINTER(ctypes.c_int32), _i,
                                                            _vp, _i64, _f, _f, _vp, _sz, _vp]
        L.rat_dilated_attn_prefill_ex.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                                  ctypes.POINTER(ctypes.c_int32), _i64, _f, _f,
                                                  ctypes.POINTER(AttnOptions), _vp]
        L.rat_dilated_attn_prefill_sinks.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                                     _i, ctypes.POINTER(ctypes.c_int32), _i,
                                                     _i64, _f, _f, _vp]
        L.rat_dilated_attn_prefill_topk.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                                    _i, ctypes.POINTER(ctypes.c_int32), _i, _i,
                                                    _i64, _f, _f, _vp]
        L.rat_recur_backward_workspace_bytes.restype = _sz
        L.rat_recur_backward_workspace_bytes.argtypes = [_i, _i, _i, _i]
        L.rat_recur_backward.argtypes = [_vp] * 16 + [_i, _i, _i, _i, _i, _i64, _f, _vp, _sz, _vp]
        L.rat_recur_backward_local.argtypes = [_vp] * 16 + [_i, _i, _i, _i, _i, _i64, _i64, _f,
                                                            _vp, _sz, _vp]
        L.rat_recur_prefill_window.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                               _i, _i, _i, _i, _i, _i64, _i64, _f, _vp, _sz, _vp]
        L.rat_recur_backward_window.argtypes = [_vp] * 14 + [_i, _i, _i, _i, _i, _i64, _i64, _f,
                                                             _vp]
        L.rat_recur_prefill_local.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                              _i, _i, _i, _i, _i, _i64, _i64, _f, _vp, _sz, _vp]
        L.rat_dilated_attn_prefill.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                               ctypes.POINTER(ctypes.c_int32), _i64, _f, _f, _vp]
        L.rat_kv_cache_bytes.argtypes = [ctypes.POINTER(KVCache), ctypes.POINTER(_sz),
                                         ctypes.POINTER(_sz), ctypes.POINTER(_sz)]
        L.rat_kv_compress.argtypes = [_vp, _vp, _vp, _vp, _i, ctypes.POINTER(KVCache), _vp]
        L.rat_kv_compress_window.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, ctypes.POINTER(KVCache), _vp]
        L.rat_kv_raw_bytes.restype = _sz
        L.rat_kv_raw_bytes.argtypes = [ctypes.POINTER(KVCache)]
        L.rat_decode_workspace_bytes.restype = _sz
        L.rat_decode_workspace_bytes.argtypes = [ctypes.POINTER(KVCache)]
        L.rat_dilated_decode.argtypes = [_vp, _vp, _vp, _vp, ctypes.POINTER(KVCache), _vp, _f, _f,
                                         _vp, _sz, _vp]
        L.rat_debug_inject_lookback_fault.argtypes = [_i64, _i64]
        L.rat_dilated_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, ctypes.POINTER(KVCache), _vp,
                                                 _f, _f, _vp]
        L.rat_paged_kv_compress.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i64,
                                             ctypes.POINTER(PagedKVCache), _vp, _sz, _vp]
        L.rat_paged_decode_workspace_bytes.restype = _sz
        L.rat_paged_decode_workspace_bytes.argtypes = [ctypes.POINTER(PagedKVCache)]
        L.rat_dilated_decode_paged.argtypes = [_vp, _vp, _vp, _vp, ctypes.POINTER(PagedKVCache),
                                               _vp, _f, _f, _vp, _sz, _vp]
        L.rat_attn_sync_status.argtypes = [_vp]
        L.rat_attn_error_site.restype = ctypes.c_uint32
        L.rat_attn_error_waiting.restype = ctypes.c_uint32
        L.rat_set_attn_block_keys.argtypes = [_i]
        L.rat_attended_keys.restype = _i64
        L.rat_attended_keys.argtypes = [_i64, _i, _i]
        _lib = L
    return _lib


def _check(fn: str, st: int):
    if st != 0:
        raise RatError(fn, st)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise RatError("dtype %s" % t.dtype, -2)


def _ptr(t: Optional[torch.Tensor]):
    """Device address of a tensor argument.  The library reads and writes every tensor as one
    dense block of device memory, so a host tensor or a strided view is refused here (a host
    address would be an illegal device access; a view would be read as if it were dense)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise RatError("tensor argument on %s (the library takes CUDA tensors)" % t.device, -1)
    if not t.is_contiguous():
        raise RatError("non-contiguous tensor argument (shape %s, strides %s)"
                       % (tuple(t.shape), t.stride()), -1)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def rat_status_string(status: int) -> str:
    return lib().rat_status_string(int(status)).decode()


def rat_attended_keys(t: int, D: int, W: int) -> int:
    return int(lib().rat_attended_keys(int(t), int(D), int(W)))


class Workspace:
    """Caller-owned device scratch (a torch uint8 buffer), zeroed once by rat_workspace_init."""

    def __init__(self, nbytes: int, device=None, stream=None):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        off = (-self.buf.data_ptr()) % 256          # 256-byte aligned view
        self.view = self.buf[off:off + self.nbytes]
        rat_workspace_init(self, stream)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.view.data_ptr())


def rat_workspace_init(ws: Workspace, stream=None):
    _check("rat_workspace_init", lib().rat_workspace_init(ws.ptr, ws.nbytes, _stream(stream)))


def rat_sync_status(ws: Workspace, stream=None) -> int:
    return int(lib().rat_sync_status(ws.ptr, _stream(stream)))


def rat_attn_sync_status(stream=None) -> int:
    return int(lib().rat_attn_sync_status(_stream(stream)))


def rat_set_attn_block_keys(block_keys: int) -> None:
    _check("rat_set_attn_block_keys", lib().rat_set_attn_block_keys(int(block_keys)))


def rat_recur_workspace_bytes(B, H, T, d, dtype) -> int:
    return int(lib().rat_recur_workspace_bytes(B, H, T, d, dtype))


def rat_recur_prefill(k, v, gate_logit, k_rec, v_rec, ws: Workspace, h0_k=None, h0_v=None,
                      hT_k=None, hT_v=None, pos0: int = 0, rope_base: float = 0.0, stream=None):
    """k, v, gate_logit -> k_rec, v_rec (all (B, H, T, d)); optional float32 (B, H, d) states."""
    B, H, T, d = k.shape
    st = lib().rat_recur_prefill(_ptr(k), _ptr(v), _ptr(gate_logit), _ptr(h0_k), _ptr(h0_v),
                                 _ptr(k_rec), _ptr(v_rec), _ptr(hT_k), _ptr(hT_v), B, H, T, d,
                                 _dtype_code(k), int(pos0), float(rope_base), ws.ptr, ws.nbytes,
                                 _stream(stream))
    _check("rat_recur_prefill", st)


def rat_recur_prefill_local(k, v, gate_logit, k_rec, v_rec, ws: Workspace, L: int,
                            h0_k=None, h0_v=None, hT_k=None, hT_v=None, pos0: int = 0,
                            rope_base: float = 0.0, stream=None):
    """rat_recur_prefill restarted before every absolute position that is a multiple of L."""
    B, H, T, d = k.shape
    st = lib().rat_recur_prefill_local(_ptr(k), _ptr(v), _ptr(gate_logit), _ptr(h0_k),
                                       _ptr(h0_v), _ptr(k_rec), _ptr(v_rec), _ptr(hT_k),
                                       _ptr(hT_v), B, H, T, d, _dtype_code(k), int(pos0), int(L),
                                       float(rope_base), ws.ptr, ws.nbytes, _stream(stream))
    _check("rat_recur_prefill_local", st)


def rat_recur_backward_workspace_bytes(B, H, T, d) -> int:
    return int(lib().rat_recur_backward_workspace_bytes(B, H, T, d))


def rat_recur_backward(k, v, gate_logit, k_rec, v_rec, dk_rec, dv_rec, dk, dv, dgate_logit,
                       ws: Workspace, h0_k=None, h0_v=None, dhT_k=None, dhT_v=None, dh0_k=None,
                       dh0_v=None, pos0: int = 0, rope_base: float = 0.0, stream=None,
                       reset_every: int = 0):
    """Gradients of the prefill recurrence step: dk, dv, dgate_logit (all (B, H, T, d)) and,
    if given, dh0_k, dh0_v (float32 (B, H, d)).  reset_every = L > 0: the chunk-local form
    (rat_recur_backward_local)."""
    B, H, T, d = k.shape
    args = [_ptr(k), _ptr(v), _ptr(gate_logit), _ptr(h0_k), _ptr(h0_v), _ptr(k_rec), _ptr(v_rec),
            _ptr(dk_rec), _ptr(dv_rec), _ptr(dhT_k), _ptr(dhT_v), _ptr(dk), _ptr(dv),
            _ptr(dgate_logit), _ptr(dh0_k), _ptr(dh0_v), B, H, T, d, _dtype_code(k), int(pos0)]
    if reset_every > 0:
        st = lib().rat_recur_backward_local(*args, int(reset_every), float(rope_base), ws.ptr,
                                            ws.nbytes, _stream(stream))
        _check("rat_recur_backward_local", st)
        return
    st = lib().rat_recur_backward(*args, float(rope_base), ws.ptr, ws.nbytes, _stream(stream))
    _check("rat_recur_backward", st)


def rat_recur_prefill_window(k, v, gate_logit, k_rec, v_rec, ws: Workspace, Lw: int = 64,
                             prev_k=None, prev_v=None, prev_gate_logit=None, pos0: int = 0,
                             rope_base: float = 0.0, stream=None):
    """Fixed-window recurrence: each state restarted Lw positions back; optional (B, H, Lw, d)
    history rows before row 0."""
    B, H, T, d = k.shape
    st = lib().rat_recur_prefill_window(_ptr(k), _ptr(v), _ptr(gate_logit), _ptr(prev_k),
                                        _ptr(prev_v), _ptr(prev_gate_logit), _ptr(k_rec),
                                        _ptr(v_rec), B, H, T, d, _dtype_code(k), int(pos0),
                                        int(Lw), float(rope_base), ws.ptr, ws.nbytes,
                                        _stream(stream))
    _check("rat_recur_prefill_window", st)


def rat_recur_backward_window(k, v, gate_logit, dk_rec, dv_rec, dk, dv, dgate_logit,
                              Lw: int = 64, prev_k=None, prev_v=None, prev_gate_logit=None,
                              dprev_k=None, dprev_v=None, dprev_gate_logit=None, pos0: int = 0,
                              rope_base: float = 0.0, stream=None):
    """Gradients of the fixed-window recurrence step: dk, dv, dgate_logit (all (B, H, T, d))
    and, with history rows, optionally dprev_k, dprev_v, dprev_gate_logit ((B, H, Lw, d))."""
    B, H, T, d = k.shape
    st = lib().rat_recur_backward_window(_ptr(k), _ptr(v), _ptr(gate_logit), _ptr(prev_k),
                                         _ptr(prev_v), _ptr(prev_gate_logit), _ptr(dk_rec),
                                         _ptr(dv_rec), _ptr(dk), _ptr(dv), _ptr(dgate_logit),
                                         _ptr(dprev_k), _ptr(dprev_v), _ptr(dprev_gate_logit),
                                         B, H, T, d, _dtype_code(k), int(pos0), int(Lw),
                                         float(rope_base), _stream(stream))
    _check("rat_recur_backward_window", st)


def rat_dilated_attn_prefill(q, k_rec, v_rec, o, D: int = 1, W: int = 0,
                             D_per_head: Optional[Sequence[int]] = None, pos0: int = 0,
                             rope_base: float = 0.0, scale: float = 0.0, stream=None,
                             n_sink: int = 0, top_k: int = 0, lse=None):
    """o = dilated attention of q over (k_rec, v_rec); all (B, H, T, d).  n_sink > 0 adds the
    first n_sink positions to every key set (rat_dilated_attn_prefill_sinks); top_k > 0 adds
    the top_k chunks by their chunk-end scores (rat_dilated_attn_prefill_topk); lse, a float32
    (B, H, T) tensor, receives log2 of every row's softmax denominator
    (rat_dilated_attn_prefill_ex)."""
    B, H, T, d = q.shape
    dph = None
    if D_per_head is not None:
        dph = (ctypes.c_int32 * H)(*[int(x) for x in D_per_head])
    if lse is not None:
        opt = AttnOptions(n_sink=int(n_sink), top_k=int(top_k), lse=_ptr(lse).value)
        st = lib().rat_dilated_attn_prefill_ex(_ptr(q), _ptr(k_rec), _ptr(v_rec), _ptr(o), B, H, T,
                                               d, _dtype_code(q), int(D), int(W), dph, int(pos0),
                                               float(rope_base), float(scale), ctypes.byref(opt),
                                               _stream(stream))
        _check("rat_dilated_attn_prefill_ex", st)
        return
    if top_k:
        st = lib().rat_dilated_attn_prefill_topk(_ptr(q), _ptr(k_rec), _ptr(v_rec), _ptr(o), B, H,
                                                 T, d, _dtype_code(q), int(D), int(W), dph,
                                                 int(n_sink), int(top_k), int(pos0),
                                                 float(rope_base), float(scale), _stream(stream))
        _check("rat_dilated_attn_prefill_topk", st)
        return
    if n_sink:
        st = lib().rat_dilated_attn_prefill_sinks(_ptr(q), _ptr(k_rec), _ptr(v_rec), _ptr(o), B, H,
                                                  T, d, _dtype_code(q), int(D), int(W), dph,
                                                  int(n_sink), int(pos0), float(rope_base),
                                                  float(scale), _stream(stream))
        _check("rat_dilated_attn_prefill_sinks", st)
        return
    st = lib().rat_dilated_attn_prefill(_ptr(q), _ptr(k_rec), _ptr(v_rec), _ptr(o), B, H, T, d,
                                        _dtype_code(q), int(D), int(W), dph, int(pos0),
                                        float(rope_base), float(scale), _stream(stream))
    _check("rat_dilated_attn_prefill", st)


def rat_dilated_attn_backward_workspace_bytes(B, H, T, d, dtype) -> int:
    return int(lib().rat_dilated_attn_backward_workspace_bytes(B, H, T, d, dtype))


def rat_dilated_attn_backward(q, k_rec, v_rec, o, dO, dq, dk_rec, dv_rec, ws: Workspace,
                              D: int = 1, W: int = 0, D_per_head: Optional[Sequence[int]] = None,
                              pos0: int = 0, rope_base: float = 0.0, scale: float = 0.0,
                              stream=None, n_sink: int = 0, lse=None):
    """Gradients of rat_dilated_attn_prefill(_sinks): dq, dk_rec, dv_rec (all (B, H, T, d));
    lse: the forward's (B, H, T) float32 output, or None (recomputed)."""
    B, H, T, d = q.shape
    dph = None
    if D_per_head is not None:
        dph = (ctypes.c_int32 * H)(*[int(x) for x in D_per_head])
    st = lib().rat_dilated_attn_backward(_ptr(q), _ptr(k_rec), _ptr(v_rec), _ptr(o), _ptr(dO),
                                         _ptr(dq), _ptr(dk_rec), _ptr(dv_rec), B, H, T, d,
                                         _dtype_code(q), int(D), int(W), dph, int(n_sink),
                                         _ptr(lse), int(pos0), float(rope_base), float(scale),
                                         ws.ptr, ws.nbytes, _stream(stream))
    _check("rat_dilated_attn_backward", st)


def make_cache(B, H, d, W, Tcap, dtype: int, D_per_head: Sequence[int], device="cuda",
               reset_every: int = 0, n_sink: int = 0, window_rec: int = 0):
    """Allocate (with torch) the buffers of a compressed cache and return (KVCache, buffers).
    reset_every = L > 0 selects the chunk-local recurrence for the decode steps; n_sink > 0
    keeps the first n_sink positions as attention sinks; window_rec = 64 selects the
    fixed-window recurrence (raw rings of the last 64 positions' k, v and gate logits)."""
    Dh = (ctypes.c_int32 * H)(*[int(x) for x in D_per_head])
    c = KVCache(B=B, H=H, d=d, W=W, Tcap=Tcap, dtype=dtype, D=Dh, reset_every=int(reset_every),
                n_sink=int(n_sink), window_rec=int(window_rec))
    dil, win, state = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check("rat_kv_cache_bytes", lib().rat_kv_cache_bytes(ctypes.byref(c), ctypes.byref(dil),
                                                          ctypes.byref(win), ctypes.byref(state)))
    tdt = torch.float32 if dtype == F32 else torch.bfloat16
    es = 4 if dtype == F32 else 2
    total = dil.value // (B * d * es)
    bufs = {
        "k_dil": torch.zeros((B, total, d), dtype=tdt, device=device),
        "v_dil": torch.zeros((B, total, d), dtype=tdt, device=device),
        "k_win": torch.zeros((B, H, max(W, 1), d), dtype=tdt, device=device),
        "v_win": torch.zeros((B, H, max(W, 1), d), dtype=tdt, device=device),
        "h_k": torch.zeros((B, H, d), dtype=torch.float32, device=device),
        "h_v": torch.zeros((B, H, d), dtype=torch.float32, device=device),
        "k_sink": torch.zeros((B, H, max(n_sink, 1), d), dtype=tdt, device=device),
        "v_sink": torch.zeros((B, H, max(n_sink, 1), d), dtype=tdt, device=device),
        "D": Dh,
    }
    for n in ("k_raw", "v_raw", "a_raw"):
        bufs[n] = torch.zeros((B, H, max(window_rec, 1), d), dtype=tdt, device=device)
    c.k_dil, c.v_dil = bufs["k_dil"].data_ptr(), bufs["v_dil"].data_ptr()
    c.k_win = bufs["k_win"].data_ptr() if W > 0 else None
    c.v_win = bufs["v_win"].data_ptr() if W > 0 else None
    c.h_k, c.h_v = bufs["h_k"].data_ptr(), bufs["h_v"].data_ptr()
    c.k_sink = bufs["k_sink"].data_ptr() if n_sink > 0 else None
    c.v_sink = bufs["v_sink"].data_ptr() if n_sink > 0 else None
    if window_rec > 0:
        c.k_raw, c.v_raw, c.a_raw = (bufs[n].data_ptr() for n in ("k_raw", "v_raw", "a_raw"))
    c.pos = 0
    return c, bufs


def rat_kv_cache_bytes(cache: KVCache):
    dil, win, state = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check("rat_kv_cache_bytes", lib().rat_kv_cache_bytes(ctypes.byref(cache), ctypes.byref(dil),
                                                          ctypes.byref(win), ctypes.byref(state)))
    return dil.value, win.value, state.value


def rat_kv_compress(k_rec, v_rec, hT_k, hT_v, cache: KVCache, stream=None):
    T = k_rec.shape[2]
    st = lib().rat_kv_compress(_ptr(k_rec), _ptr(v_rec), _ptr(hT_k), _ptr(hT_v), T,
                               ctypes.byref(cache), _stream(stream))
    _check("rat_kv_compress", st)


def rat_kv_compress_window(k_rec, v_rec, k, v, gate_logit, cache: KVCache, stream=None):
    """Append positions of the fixed-window recurrence (outputs and raw inputs) to a cache made
    with window_rec = 64."""
    T = k_rec.shape[2]
    st = lib().rat_kv_compress_window(_ptr(k_rec), _ptr(v_rec), _ptr(k), _ptr(v), _ptr(gate_logit),
                                      T, ctypes.byref(cache), _stream(stream))
    _check("rat_kv_compress_window", st)


def rat_kv_raw_bytes(cache: KVCache) -> int:
    return int(lib().rat_kv_raw_bytes(ctypes.byref(cache)))


def rat_decode_workspace_bytes(cache: KVCache) -> int:
    return int(lib().rat_decode_workspace_bytes(ctypes.byref(cache)))


def rat_dilated_decode(q, k, v, gate_logit, cache: KVCache, o, ws: Workspace,
                       rope_base: float = 0.0, scale: float = 0.0, stream=None):
    st = lib().rat_dilated_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), ctypes.byref(cache),
                                  _ptr(o), float(rope_base), float(scale), ws.ptr, ws.nbytes,
                                  _stream(stream))
    _check("rat_dilated_decode", st)


def rat_dilated_decode_noalloc(q, k, v, gate_logit, cache: KVCache, o, rope_base: float = 0.0,
                               scale: float = 0.0, stream=None):
    """rat_dilated_decode without a workspace argument: the library's fixed device scratch is used
    (for callers that cannot allocate; concurrent calls must not overlap on the GPU)."""
    st = lib().rat_dilated_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit),
                                          ctypes.byref(cache), _ptr(o), float(rope_base),
                                          float(scale), _stream(stream))
    _check("rat_dilated_decode_noalloc", st)


def make_paged_cache(B, H, d, W, dtype: int, D_per_head: Sequence[int], page_entries: int,
                     n_pages: int, page_table, device="cuda", reset_every: int = 0):
    """Allocate (with torch) the pools, ring, state and positions of a paged cache around a
    caller-filled int32 page table (B, H, max_pages) on the device; returns (PagedKVCache,
    buffers)."""
    Dh = (ctypes.c_int32 * H)(*[int(x) for x in D_per_head])
    tdt = torch.float32 if dtype == F32 else torch.bfloat16
    assert page_table.dtype == torch.int32 and page_table.is_contiguous()
    assert tuple(page_table.shape[:2]) == (B, H)
    bufs = {
        "k_pool": torch.zeros((n_pages, page_entries, d), dtype=tdt, device=device),
        "v_pool": torch.zeros((n_pages, page_entries, d), dtype=tdt, device=device),
        "k_win": torch.zeros((B, H, max(W, 1), d), dtype=tdt, device=device),
        "v_win": torch.zeros((B, H, max(W, 1), d), dtype=tdt, device=device),
        "h_k": torch.zeros((B, H, d), dtype=torch.float32, device=device),
        "h_v": torch.zeros((B, H, d), dtype=torch.float32, device=device),
        "pos": torch.zeros((B,), dtype=torch.int64, device=device),
        "page_table": page_table, "D": Dh,
    }
    c = PagedKVCache(B=B, H=H, d=d, W=W, dtype=dtype, page_entries=page_entries,
                     max_pages=int(page_table.shape[2]), n_pages=n_pages, D=Dh,
                     reset_every=int(reset_every))
    c.k_pool, c.v_pool = bufs["k_pool"].data_ptr(), bufs["v_pool"].data_ptr()
    c.page_table = page_table.data_ptr()
    c.k_win = bufs["k_win"].data_ptr() if W > 0 else None
    c.v_win = bufs["v_win"].data_ptr() if W > 0 else None
    c.h_k, c.h_v = bufs["h_k"].data_ptr(), bufs["h_v"].data_ptr()
    c.pos = bufs["pos"].data_ptr()
    return c, bufs


def rat_paged_kv_compress(k_rec, v_rec, hT_k, hT_v, b: int, pos0: int, cache: PagedKVCache,
                          ws: Workspace, stream=None):
    """Append positions pos0 .. pos0+T-1 of sequence b ((1, H, T, d) tensors) to a paged cache."""
    T = k_rec.shape[2]
    st = lib().rat_paged_kv_compress(_ptr(k_rec), _ptr(v_rec), _ptr(hT_k), _ptr(hT_v), T, int(b),
                                     int(pos0), ctypes.byref(cache), ws.ptr, ws.nbytes,
                                     _stream(stream))
    _check("rat_paged_kv_compress", st)


def rat_paged_decode_workspace_bytes(cache: PagedKVCache) -> int:
    return int(lib().rat_paged_decode_workspace_bytes(ctypes.byref(cache)))


def rat_dilated_decode_paged(q, k, v, gate_logit, cache: PagedKVCache, o, ws: Workspace,
                             rope_base: float = 0.0, scale: float = 0.0, stream=None):
    st = lib().rat_dilated_decode_paged(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit),
                                        ctypes.byref(cache), _ptr(o), float(rope_base),
                                        float(scale), ws.ptr, ws.nbytes, _stream(stream))
    _check("rat_dilated_decode_paged", st)
