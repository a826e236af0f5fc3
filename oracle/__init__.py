"""Plain float64 CPU oracle for the RAT+ dilated-inference hot path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline call this package; the CUDA library never imports it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain loops in float64, one routine per definition);
this module only builds it, marshals numpy arrays and composes the routines in the order
the pages give: recurrence over keys and values, RoPE on the recurrence output and on the
query, then attention over the dilated-plus-window key set.

Sources: "RAT+ Deep Dive" section 2.1 (full-sequence forget-gate recurrence, associative
scan prefill), section 3.1 table (FLOPs T/D), section 6 (head-wise hybrid); the RAT+
abstract (dilation D, optional local windows, D-fold KV-cache reduction); RoFormer (RoPE).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)
_lp = ctypes.POINTER(ctypes.c_long)
_bp = ctypes.POINTER(ctypes.c_uint8)
_L = ctypes.c_long


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.rat_oracle_recurrence.argtypes = [_L, _L, _L, _dp, _dp, _dp, _dp, _dp]
        lib.rat_oracle_recurrence_reset.argtypes = [_L, _L, _L, _dp, _dp, _dp, _dp, _dp, _L, _L]
        lib.rat_oracle_recurrence_window.argtypes = [_L, _L, _L, _dp, _dp, _dp, _dp, _L, _dp]
        lib.rat_oracle_dilated_attention_backward.argtypes = [_L, _L, _L, _dp, _dp, _dp, _dp,
                                                              _ip, _L, _L, ctypes.c_double, _dp,
                                                              _dp, _dp]
        lib.rat_oracle_topk_attention.argtypes = [_L, _L, _L, _dp, _dp, _dp, _ip, _L, _L, _L,
                                                  ctypes.c_double, _dp]
        lib.rat_oracle_recurrence_backward.argtypes = [_L, _L, _L, _dp, _dp, _dp, _dp, _dp, _dp,
                                                       _dp, _dp]
        lib.rat_oracle_recurrence_backward_reset.argtypes = [_L, _L, _L, _dp, _dp, _dp, _dp, _dp,
                                                             _L, _L, _dp, _dp, _dp]
        lib.rat_oracle_recurrence_window_backward.argtypes = [_L, _L, _L, _dp, _dp, _dp, _dp, _L,
                                                              _dp, _dp, _dp, _dp, _dp]
        lib.rat_oracle_rope.argtypes = [_L, _L, _L, _dp, _L, ctypes.c_double]
        lib.rat_oracle_in_key_set.argtypes = [_L, _L, _L, _L]
        lib.rat_oracle_in_key_set.restype = ctypes.c_int
        lib.rat_oracle_key_count.argtypes = [_L, _L, _L]
        lib.rat_oracle_key_count.restype = ctypes.c_long
        lib.rat_oracle_in_key_set_sinks.argtypes = [_L, _L, _L, _L, _L]
        lib.rat_oracle_in_key_set_sinks.restype = ctypes.c_int
        lib.rat_oracle_key_count_sinks.argtypes = [_L, _L, _L, _L]
        lib.rat_oracle_key_count_sinks.restype = ctypes.c_long
        lib.rat_oracle_dilated_attention.argtypes = [_L, _L, _L, _dp, _dp, _dp, _ip, _L, _L,
                                                     ctypes.c_double, _lp, _L, _dp, _dp]
        lib.rat_oracle_kv_compress.argtypes = [_L, _L, _L, _L, _L, _bp, _ip, _L, _L, _L, _bp, _bp]
        lib.rat_oracle_decode_step.argtypes = [_L, _L, _L, _ip, _L, _L, ctypes.c_double,
                                               ctypes.c_double, _dp, _dp, _dp, _dp, _dp, _dp,
                                               _dp, _dp, _L, _dp]
        lib.rat_oracle_threads.restype = ctypes.c_int
        lib.rat_oracle_set_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray, kind=_dp):
    return a.ctypes.data_as(kind)


def threads() -> int:
    return int(_load().rat_oracle_threads())


def set_threads(n: int) -> None:
    _load().rat_oracle_set_threads(int(n))


def default_scale(d: int) -> float:
    """Softmax scale 1/sqrt(d_head) (standard attention; the pages state none)."""
    return 1.0 / np.sqrt(d)


def recurrence(x, a, h0=None, pos0: int = 0, reset_every: int = 0):
    """h_t = g_t h_{t-1} + (1-g_t) x_t, g = sigmoid(a), per channel, over the full sequence.

    x, a: (..., T, d).  h0: (..., d) or None (zeros).  Returns (y, hT) in float64.
    ("RAT+ Deep Dive" section 2.1, full-sequence recurrence, L = T.)  With reset_every = L > 0
    the state is zeroed before every absolute position pos0 + t that is a multiple of L: the
    predecessor RAT's chunk-local recurrence (same section; the RAT paper's abstract).
    """
    x = _f64(x)
    a = _f64(a)
    assert x.shape == a.shape
    T, d = x.shape[-2], x.shape[-1]
    BH = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    y = np.empty_like(x)
    hT = np.empty(x.shape[:-2] + (d,), dtype=np.float64)
    h0p = None
    if h0 is not None:
        h0 = _f64(h0)
        assert h0.shape == hT.shape
        h0p = _ptr(h0)
    if reset_every and int(reset_every) > 0:
        _load().rat_oracle_recurrence_reset(BH, T, d, _ptr(x), _ptr(a), h0p, _ptr(y), _ptr(hT),
                                            int(pos0), int(reset_every))
    else:
        _load().rat_oracle_recurrence(BH, T, d, _ptr(x), _ptr(a), h0p, _ptr(y), _ptr(hT))
    return y, hT


def recurrence_window(x, a, Lw: int = 64, prev_x=None, prev_a=None):
    """Fixed-window recurrence: y_t is the forget-gate recurrence restarted from zero at
    t - Lw + 1 and run to t ("RAT+ Deep Dive" section 2.1, recurrence window L* = 64).

    x, a: (..., T, d).  prev_x, prev_a: (..., Lw, d), the Lw positions before row 0, or None
    (the window is clipped at row 0).  Returns y in float64.
    """
    x = _f64(x)
    a = _f64(a)
    assert x.shape == a.shape and int(Lw) >= 1
    T, d = x.shape[-2], x.shape[-1]
    BH = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    y = np.empty_like(x)
    px = pa = None
    if prev_x is not None:
        prev_x, prev_a = _f64(prev_x), _f64(prev_a)
        assert prev_x.shape == x.shape[:-2] + (int(Lw), d) and prev_a.shape == prev_x.shape
        px, pa = _ptr(prev_x), _ptr(prev_a)
    _load().rat_oracle_recurrence_window(BH, T, d, _ptr(x), _ptr(a), px, pa, int(Lw), _ptr(y))
    return y


def rope(x, pos0: int = 0, base: float = 10000.0):
    """Rotate-half RoPE at positions pos0 + t (RoFormer).  Returns a new float64 array."""
    x = _f64(x).copy()
    T, d = x.shape[-2], x.shape[-1]
    BH = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    _load().rat_oracle_rope(BH, T, d, _ptr(x), int(pos0), float(base))
    return x


def rope_transpose(y, pos0: int = 0, base: float = 10000.0):
    """The transpose (= inverse) of the rotate-half rotation: each pair (c, c + d/2) turned by
    -(pos0 + t) theta_c.  The backward of y = RoPE(h) is dh = RoPE^T(dy)."""
    y = _f64(y)
    T, d = y.shape[-2], y.shape[-1]
    half = d // 2
    theta = base ** (-2.0 * np.arange(half) / d)
    ang = (pos0 + np.arange(T))[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    y1, y2 = y[..., :half], y[..., half:]
    return np.concatenate([y1 * c + y2 * s, y2 * c - y1 * s], axis=-1)


def recurrence_backward(x, a, dy, h0=None, dhT=None, pos0: int = 0, reset_every: int = 0):
    """Reverse-mode derivative of recurrence(x, a, h0, pos0, reset_every): returns (dx, dg, dh0)
    for upstream gradients dy of the outputs and dhT of the final state; dg is the gradient with
    respect to the gate value g = sigmoid(a).  reset_every = L > 0 is the chunk-local form (the
    state restarts before every absolute position pos0 + t that is a multiple of L)."""
    x, a, dy = _f64(x), _f64(a), _f64(dy)
    assert x.shape == a.shape == dy.shape
    T, d = x.shape[-2], x.shape[-1]
    BH = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    dx, dg = np.empty_like(x), np.empty_like(x)
    dh0 = np.empty(x.shape[:-2] + (d,), dtype=np.float64)
    h0p = None
    if h0 is not None:
        h0 = _f64(h0)
        h0p = _ptr(h0)
    dhTp = None
    if dhT is not None:
        dhT = _f64(dhT)
        dhTp = _ptr(dhT)
    if reset_every > 0:
        _load().rat_oracle_recurrence_backward_reset(BH, T, d, _ptr(x), _ptr(a), h0p, _ptr(dy),
                                                     dhTp, int(pos0), int(reset_every), _ptr(dx),
                                                     _ptr(dg), _ptr(dh0))
    else:
        _load().rat_oracle_recurrence_backward(BH, T, d, _ptr(x), _ptr(a), h0p, _ptr(dy), dhTp,
                                               _ptr(dx), _ptr(dg), _ptr(dh0))
    return dx, dg, dh0


def recurrence_layer_backward(k, v, a, dk_rec, dv_rec, h0k=None, h0v=None, dhTk=None, dhTv=None,
                              pos0: int = 0, rope_base: float = 0.0, reset_every: int = 0):
    """Backward of the prefill recurrence step (k~ = RoPE(h^k), v~ = h^v, one gate for both):
    returns (dk, dv, da, dh0k, dh0v).  The gate is shared, so its gradient sums the k and v
    parts, through dg/da = g (1 - g).  reset_every = L > 0: the chunk-local form."""
    ek = rope_transpose(dk_rec, pos0, rope_base) if rope_base > 0 else _f64(dk_rec)
    dk, dgk, dh0k = recurrence_backward(k, a, ek, h0k, dhTk, pos0, reset_every)
    dv, dgv, dh0v = recurrence_backward(v, a, dv_rec, h0v, dhTv, pos0, reset_every)
    a = _f64(a)
    with np.errstate(over="ignore"):        # saturated logits: exp -> inf gives g = 0 or 1
        g = 1.0 / (1.0 + np.exp(-a))
        omg = 1.0 / (1.0 + np.exp(a))
    return dk, dv, g * omg * (dgk + dgv), dh0k, dh0v


def recurrence_window_backward(x, a, dy, Lw: int = 64, prev_x=None, prev_a=None):
    """Reverse-mode derivative of recurrence_window(x, a, Lw, prev_x, prev_a): returns
    (dx, dg, dprev_x, dprev_g) for upstream gradients dy of the outputs; dg is the gradient with
    respect to the gate value g = sigmoid(a); dprev_x, dprev_g are the gradients of the history
    rows (None without them)."""
    x, a, dy = _f64(x), _f64(a), _f64(dy)
    assert x.shape == a.shape == dy.shape and int(Lw) >= 1
    T, d = x.shape[-2], x.shape[-1]
    BH = int(np.prod(x.shape[:-2])) if x.ndim > 2 else 1
    dx, dg = np.empty_like(x), np.empty_like(x)
    px = pa = dpx = dpg = None
    dprev_x = dprev_g = None
    if prev_x is not None:
        prev_x, prev_a = _f64(prev_x), _f64(prev_a)
        assert prev_x.shape == x.shape[:-2] + (int(Lw), d) and prev_a.shape == prev_x.shape
        px, pa = _ptr(prev_x), _ptr(prev_a)
        dprev_x, dprev_g = np.empty_like(prev_x), np.empty_like(prev_x)
        dpx, dpg = _ptr(dprev_x), _ptr(dprev_g)
    _load().rat_oracle_recurrence_window_backward(BH, T, d, _ptr(x), _ptr(a), px, pa, int(Lw),
                                                  _ptr(dy), _ptr(dx), _ptr(dg), dpx, dpg)
    return dx, dg, dprev_x, dprev_g


def recurrence_window_layer_backward(k, v, a, dk_rec, dv_rec, Lw: int = 64, prev_k=None,
                                     prev_v=None, prev_a=None, pos0: int = 0,
                                     rope_base: float = 0.0):
    """Backward of the fixed-window prefill step (k~ = RoPE(y^k), v~ = y^v, one gate for both):
    returns (dk, dv, da, dprev_k, dprev_v, dprev_a), the last three None without history rows.
    The gate is shared, so its gradient sums the k and v parts, through dg/da = g (1 - g)."""
    ek = rope_transpose(dk_rec, pos0, rope_base) if rope_base > 0 else _f64(dk_rec)
    dk, dgk, dpk, dpgk = recurrence_window_backward(k, a, ek, Lw, prev_k, prev_a)
    dv, dgv, dpv, dpgv = recurrence_window_backward(v, a, dv_rec, Lw, prev_v, prev_a)

    def dlogit(logit, dgate):
        logit = _f64(logit)
        with np.errstate(over="ignore"):    # saturated logits: exp -> inf gives g = 0 or 1
            g = 1.0 / (1.0 + np.exp(-logit))
            omg = 1.0 / (1.0 + np.exp(logit))
        return g * omg * dgate

    da = dlogit(a, dgk + dgv)
    dpa = dlogit(prev_a, dpgk + dpgv) if prev_k is not None else None
    return dk, dv, da, dpk, dpv, dpa


def in_key_set(t: int, j: int, D: int, W: int, n_sink: int = 0) -> bool:
    """Is key j in the key set of query t (window (t-We, t] union chunk ends older than it,
    union the first n_sink positions)?"""
    if n_sink:
        return bool(_load().rat_oracle_in_key_set_sinks(int(t), int(j), int(D), int(W), int(n_sink)))
    return bool(_load().rat_oracle_in_key_set(int(t), int(j), int(D), int(W)))


def key_count(t: int, D: int, W: int, n_sink: int = 0) -> int:
    """|S(t)| by enumeration."""
    if n_sink:
        return int(_load().rat_oracle_key_count_sinks(int(t), int(D), int(W), int(n_sink)))
    return int(_load().rat_oracle_key_count(int(t), int(D), int(W)))


def _per_bh_dilation(shape_bh, D, D_per_head):
    B, H = shape_bh
    if D_per_head is None:
        Dh = np.full((H,), int(D), dtype=np.int32)
    else:
        Dh = np.asarray(D_per_head, dtype=np.int32)
        assert Dh.shape == (H,)
    return np.ascontiguousarray(np.tile(Dh, B).astype(np.int32)), Dh


def dilated_attention(q, k, v, D=1, W=0, D_per_head=None, scale=None, rows=None, n_sink=0,
                      return_lse=False):
    """Causal dilated attention (+ local window, per-head D) over (B, H, T, d) tensors.

    q, k, v are used as given (rotate them first if RoPE is in use).  rows: optional list of
    query positions; the result then has shape (B, H, len(rows), d).  n_sink > 0 adds the first
    n_sink positions to every key set (StreamingLLM attention sinks).
    (RAT+ abstract; "RAT+ Deep Dive" section 3.1 table and section 6 head-wise and layer-wise
    hybrids.)  return_lse: also return log2 of each row's softmax denominator, (B, H, rows).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, d = q.shape
    Dbh, _ = _per_bh_dilation((B, H), D, D_per_head)
    if scale is None:
        scale = default_scale(d)
    if rows is None:
        nrows, rp = T, None
        out = np.empty((B, H, T, d))
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        assert rows_a.min() >= 0 and rows_a.max() < T
        nrows, rp = len(rows_a), _ptr(rows_a, _lp)
        out = np.empty((B, H, nrows, d))
    lse = np.empty(out.shape[:-1]) if return_lse else None
    _load().rat_oracle_dilated_attention(B * H, T, d, _ptr(q), _ptr(k), _ptr(v), _ptr(Dbh, _ip),
                                         int(W), int(n_sink), float(scale), rp, nrows, _ptr(out),
                                         _ptr(lse) if return_lse else None)
    return (out, lse) if return_lse else out


def attention_over_keys(q_t, k, v, keys, scale):
    """Softmax attention of one query over an explicit list of key positions, each listed once:
    o = sum_j softmax_j(scale * <q_t, k_j>) v_j over j in keys (the attention step of the RAT+
    abstract and "RAT+ Deep Dive" section 3.1, with the key set given rather than derived).
    Used where a key set comes from a selection with several admissible outcomes (top-k chunks
    whose scores tie within rounding).  q_t (d,), k and v (T, d), keys a sequence of ints;
    returns (d,) in float64."""
    q_t, k, v = _f64(q_t), _f64(k), _f64(v)
    idx = np.asarray(list(keys), dtype=np.int64)
    s = scale * (k[idx] @ q_t)
    p = np.exp(s - s.max())
    return (p @ v[idx]) / p.sum()


def topk_attention(q, k, v, D=1, W=0, D_per_head=None, scale=None, n_sink=0, top_k=0):
    """Dilated attention plus the top_k chunks (scored by their chunk-end keys) attended at
    every position ("RAT+ Deep Dive" section 4, dilation combined with top-k selection).
    q, k, v as in dilated_attention; returns (B, H, T, d) in float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, d = q.shape
    Dbh, _ = _per_bh_dilation((B, H), D, D_per_head)
    if scale is None:
        scale = default_scale(d)
    out = np.empty((B, H, T, d))
    _load().rat_oracle_topk_attention(B * H, T, d, _ptr(q), _ptr(k), _ptr(v), _ptr(Dbh, _ip),
                                      int(W), int(n_sink), int(top_k), float(scale), _ptr(out))
    return out


def dilated_attention_backward(q, k, v, dO, D=1, W=0, D_per_head=None, scale=None,
                               rope_base=0.0, pos0=0, n_sink=0):
    """Reverse-mode derivative of dilated_attention for upstream gradients dO: returns
    (dq, dk, dv) in float64.  With rope_base > 0, q is rotated at positions pos0 + t first (as
    the attention does) and dq is the gradient with respect to the unrotated q (RoPE^T applied);
    k and v are the recurrence outputs k~, v~ as stored (k~ already rotated)."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, T, d = q.shape
    Dbh, _ = _per_bh_dilation((B, H), D, D_per_head)
    if scale is None:
        scale = default_scale(d)
    qh = rope(q, pos0, rope_base) if rope_base > 0 else q
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    _load().rat_oracle_dilated_attention_backward(B * H, T, d, _ptr(qh), _ptr(k), _ptr(v),
                                                  _ptr(dO), _ptr(Dbh, _ip), int(W), int(n_sink),
                                                  float(scale),
                                                  _ptr(dq), _ptr(dk), _ptr(dv))
    if rope_base > 0:
        dq = rope_transpose(dq, pos0, rope_base)
    return dq, dk, dv


def layer_prefill(q, k, v, a, D=1, W=0, D_per_head=None, rope_base=0.0, pos0=0, scale=None,
                  rows=None, h0_k=None, h0_v=None, reset_every=0, n_sink=0):
    """The whole prefill path in float64: recurrence -> RoPE -> dilated attention.

    Returns dict(o, k_rec, v_rec, hT_k, hT_v); k_rec is the recurrence output after RoPE
    (what the cache stores), v_rec the value recurrence output.  reset_every > 0 selects the
    chunk-local recurrence (see recurrence()).
    """
    k_rec, hT_k = recurrence(k, a, h0_k, pos0=pos0, reset_every=reset_every)
    v_rec, hT_v = recurrence(v, a, h0_v, pos0=pos0, reset_every=reset_every)
    qr = _f64(q)
    if rope_base > 0:
        k_rec = rope(k_rec, pos0, rope_base)
        qr = rope(qr, pos0, rope_base)
    o = dilated_attention(qr, k_rec, v_rec, D=D, W=W, D_per_head=D_per_head, scale=scale, rows=rows,
                          n_sink=n_sink)
    return dict(o=o, k_rec=k_rec, v_rec=v_rec, hT_k=hT_k, hT_v=hT_v)


def cache_capacity(Tcap: int, D_per_head) -> np.ndarray:
    """cap_h = floor(Tcap / D_h): the compressed cache keeps one key per chunk of D."""
    return np.asarray([Tcap // int(Dh) for Dh in D_per_head], dtype=np.int64)


def kv_compress(x, D_per_head, W: int, Tcap: int, pos0: int = 0, dil=None, ring=None):
    """Bit-exact gather of a (B, H, T, d) tensor of any element type into the cache layout.

    Returns (dil, ring): dil (B, sum_h cap_h, d), ring (B, H, W, d) (or None if W == 0), of
    x's dtype; existing dil/ring arrays are updated in place (chunked prefill).
    """
    x = np.ascontiguousarray(x)
    B, H, T, d = x.shape
    Dh = np.ascontiguousarray(np.asarray(D_per_head, dtype=np.int32))
    total = int(cache_capacity(Tcap, Dh).sum())
    if dil is None:
        dil = np.zeros((B, total, d), dtype=x.dtype)
    if ring is None and W > 0:
        ring = np.zeros((B, H, W, d), dtype=x.dtype)
    xb = x.view(np.uint8)
    _load().rat_oracle_kv_compress(B, H, T, d, x.dtype.itemsize, _ptr(xb, _bp), _ptr(Dh, _ip),
                                   int(W), int(Tcap), int(pos0), _ptr(dil.view(np.uint8), _bp),
                                   _ptr(ring.view(np.uint8), _bp) if ring is not None else None)
    return dil, ring


class DecodeState:
    """Float64 decode oracle: recurrence state plus the full history of k~ and v~.

    Keeping every position is the plain definition (the compressed cache is an optimisation
    of it); use it on a few (batch, head) slices.  Dbh gives each slice's dilation.
    window_rec = Lw > 0 selects the fixed-window recurrence (recurrence_window): the state of
    each new token is the recurrence restarted from zero Lw - 1 positions back, so the raw
    inputs (k, v, a) of every position are kept too.
    """

    def __init__(self, Dbh, d: int, W: int, Tcap: int, rope_base: float = 0.0, scale=None,
                 reset_every: int = 0, n_sink: int = 0, window_rec: int = 0):
        self.Dbh = np.ascontiguousarray(np.asarray(Dbh, dtype=np.int32))
        self.BH = len(self.Dbh)
        self.d, self.W, self.Tcap = d, int(W), int(Tcap)
        self.rope_base = float(rope_base)
        self.scale = default_scale(d) if scale is None else float(scale)
        self.hk = np.zeros((self.BH, d))
        self.hv = np.zeros((self.BH, d))
        self.khist = np.zeros((self.BH, self.Tcap, d))
        self.vhist = np.zeros((self.BH, self.Tcap, d))
        self.t = 0
        self.reset_every = int(reset_every)     # > 0: chunk-local recurrence (state zeroed at t % L == 0)
        self.n_sink = int(n_sink)               # attention sinks: the first n_sink positions
        self.window_rec = int(window_rec)       # > 0: fixed-window recurrence over the last Lw positions
        if self.window_rec > 0:
            self.raw = np.zeros((3, self.BH, self.Tcap, d))     # k, v, a of every position

    def prefill(self, k, v, a):
        """Consume a context (BH, T, d) with the sequential recurrence and record history."""
        k, v, a = _f64(k), _f64(v), _f64(a)
        T = k.shape[-2]
        if self.window_rec > 0:
            Lw, t0 = self.window_rec, self.t
            self.raw[0, :, t0:t0 + T], self.raw[1, :, t0:t0 + T], self.raw[2, :, t0:t0 + T] = k, v, a
            lo = max(0, t0 - Lw)                  # history rows before the context, where present
            yk = recurrence_window(self.raw[0, :, lo:t0 + T], self.raw[2, :, lo:t0 + T], Lw)[:, t0 - lo:]
            yv = recurrence_window(self.raw[1, :, lo:t0 + T], self.raw[2, :, lo:t0 + T], Lw)[:, t0 - lo:]
            if self.rope_base > 0:
                yk = rope(yk, t0, self.rope_base)
            self.khist[:, t0:t0 + T] = yk
            self.vhist[:, t0:t0 + T] = yv
            self.t += T
            return
        yk, hk = recurrence(k, a, self.hk, pos0=self.t, reset_every=self.reset_every)
        yv, hv = recurrence(v, a, self.hv, pos0=self.t, reset_every=self.reset_every)
        if self.rope_base > 0:
            yk = rope(yk, self.t, self.rope_base)
        self.khist[:, self.t:self.t + T] = yk
        self.vhist[:, self.t:self.t + T] = yv
        self.hk, self.hv = np.ascontiguousarray(hk), np.ascontiguousarray(hv)
        self.t += T

    def step(self, q, k, v, a):
        """One new token per slice: (BH, d) inputs -> (BH, d) output."""
        q, k, v, a = _f64(q), _f64(k), _f64(v), _f64(a)
        if self.reset_every > 0 and self.t % self.reset_every == 0:
            self.hk[:] = 0.0                    # a new block starts at this position
            self.hv[:] = 0.0
        if self.window_rec > 0:
            # the state entering the token: the recurrence from zero over the Lw - 1 positions
            # before it (those that exist); the step below adds the token itself
            t, Lw = self.t, self.window_rec
            lo = max(0, t - Lw + 1)
            zero = np.zeros((self.BH, self.d))
            _, self.hk = recurrence(self.raw[0, :, lo:t], self.raw[2, :, lo:t], zero)
            _, self.hv = recurrence(self.raw[1, :, lo:t], self.raw[2, :, lo:t], zero)
            self.hk, self.hv = np.ascontiguousarray(self.hk), np.ascontiguousarray(self.hv)
            self.raw[0, :, t], self.raw[1, :, t], self.raw[2, :, t] = k, v, a
        o = np.empty((self.BH, self.d))
        _load().rat_oracle_decode_step(self.BH, self.d, self.t, _ptr(self.Dbh, _ip), self.W,
                                       self.n_sink, self.scale, self.rope_base, _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(a), _ptr(self.hk), _ptr(self.hv), _ptr(self.khist),
                                       _ptr(self.vhist), self.Tcap, _ptr(o))
        self.t += 1
        return o
