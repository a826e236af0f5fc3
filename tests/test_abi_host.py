"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol the
header declares, and validates its arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

import recurrence_augmented_dilated_b200 as rat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from recurrence_augmented_dilated_b200 import build
    build.build()
    return rat.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"RAT_API\s+[\w\s\*]+?\b(rat_\w+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert {"rat_recur_prefill", "rat_dilated_attn_prefill", "rat_kv_compress",
            "rat_dilated_decode"} <= names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5):
        assert rat.rat_status_string(code).startswith(("RAT_OK", "RAT_ERR"))
    assert "sm_100a" in L.rat_version().decode()


def closed_form_count(t, D, W):
    We = max(W, 1)
    return min(We, t + 1) + max(0, (t - We + 1) // D)


def test_attended_keys_matches_count(L):
    for D, W in [(1, 0), (4, 0), (16, 0), (64, 128), (64, 64), (3, 7)]:
        for t in [0, 1, 2, 63, 64, 127, 128, 1000, 32767]:
            assert rat.rat_attended_keys(t, D, W) == closed_form_count(t, D, W)


def test_recur_validation(L):
    P = ctypes.c_void_p
    ws = P(4096 * 256)            # never dereferenced: validation fails first
    # B < 1
    assert L.rat_recur_prefill(P(256), P(256), P(256), None, None, P(256), P(256), None, None,
                               0, 1, 8, 128, 1, 0, 0.0, ws, 1 << 20, None) == -1
    # d unsupported
    assert L.rat_recur_prefill(P(256), P(256), P(256), None, None, P(256), P(256), None, None,
                               1, 1, 8, 96, 1, 0, 0.0, ws, 1 << 20, None) == -2
    # NULL input
    assert L.rat_recur_prefill(None, P(256), P(256), None, None, P(256), P(256), None, None,
                               1, 1, 8, 128, 1, 0, 0.0, ws, 1 << 20, None) == -1
    # misaligned input
    assert L.rat_recur_prefill(P(258), P(256), P(256), None, None, P(256), P(256), None, None,
                               1, 1, 8, 128, 1, 0, 0.0, ws, 1 << 20, None) == -1
    # workspace too small / missing
    need = rat.rat_recur_workspace_bytes(1, 1, 8, 128, 1)
    assert need > 256
    assert L.rat_recur_prefill(P(256), P(256), P(256), None, None, P(256), P(256), None, None,
                               1, 1, 8, 128, 1, 0, 0.0, ws, need - 1, None) == -5
    assert L.rat_recur_prefill(P(256), P(256), P(256), None, None, P(256), P(256), None, None,
                               1, 1, 8, 128, 1, 0, 0.0, None, need, None) == -5
    # T == 0 is a no-op
    assert L.rat_recur_prefill(None, None, None, None, None, None, None, None, None,
                               1, 1, 0, 128, 1, 0, 0.0, None, 0, None) == 0


def test_local_and_window_validation(L):
    P = ctypes.c_void_p
    ws = P(4096 * 256)
    need = rat.rat_recur_workspace_bytes(1, 1, 8, 128, 1)
    # chunk-local: the block length must be at least 1
    assert L.rat_recur_prefill_local(P(256), P(256), P(256), None, None, P(256), P(256), None,
                                     None, 1, 1, 8, 128, 1, 0, 0, 0.0, ws, need, None) == -1
    assert L.rat_recur_prefill_local(P(256), P(256), P(256), None, None, P(256), P(256), None,
                                     None, 1, 1, 8, 128, 1, 0, -3, 0.0, ws, need, None) == -1
    assert L.rat_recur_prefill_local(None, None, None, None, None, None, None, None, None,
                                     1, 1, 0, 128, 1, 0, 16, 0.0, None, 0, None) == 0
    args = lambda Lw, prev=(None, None, None), ws_=ws, wsb=256, T=8: (
        P(256), P(256), P(256), *prev, P(256), P(256), 1, 1, T, 128, 1, 0, Lw, 0.0, ws_, wsb, None)
    # window: below 1 invalid, other lengths than 64 unsupported
    assert L.rat_recur_prefill_window(*args(0)) == -1
    assert L.rat_recur_prefill_window(*args(32)) == -2
    # history rows: all three or none
    assert L.rat_recur_prefill_window(*args(64, prev=(P(256), None, None))) == -1
    assert L.rat_recur_prefill_window(*args(64, prev=(P(256), P(256), P(258)))) == -1
    # workspace header missing, too small or misaligned
    assert L.rat_recur_prefill_window(*args(64, ws_=None)) == -5
    assert L.rat_recur_prefill_window(*args(64, wsb=255)) == -5
    assert L.rat_recur_prefill_window(*args(64, ws_=P(4096 * 256 + 16))) == -5
    # T == 0 is a no-op
    assert L.rat_recur_prefill_window(*args(64, T=0)) == 0


def test_window_backward_validation(L):
    P = ctypes.c_void_p
    three = (P(256), P(512), P(768))
    bargs = lambda Lw=64, prev=(None, None, None), dprev=(None, None, None), T=8, d=128, dt=1, \
        pos0=0, out=P(1024): (P(256), P(256), P(256), *prev, P(256), P(256), out, P(256), P(256),
                              *dprev, 1, 1, T, d, dt, pos0, Lw, 0.0, None)
    assert L.rat_recur_backward_window(*bargs(Lw=0)) == -1
    assert L.rat_recur_backward_window(*bargs(Lw=32)) == -2
    assert L.rat_recur_backward_window(*bargs(d=96)) == -2
    assert L.rat_recur_backward_window(*bargs(dt=7)) == -1
    assert L.rat_recur_backward_window(*bargs(pos0=-1)) == -1
    # history rows and their gradients: all three or none; gradients only with the rows
    assert L.rat_recur_backward_window(*bargs(prev=(P(256), None, None))) == -1
    assert L.rat_recur_backward_window(*bargs(dprev=three)) == -1
    assert L.rat_recur_backward_window(*bargs(prev=three, dprev=(P(256), P(256), None))) == -1
    # misaligned or missing output
    assert L.rat_recur_backward_window(*bargs(out=P(1032))) == -1
    assert L.rat_recur_backward_window(*bargs(out=None)) == -1
    assert L.rat_recur_backward_window(*bargs(prev=three, dprev=(P(256), P(264), P(256)))) == -1
    # T == 0 is a no-op (no pointer is read)
    assert L.rat_recur_backward_window(*bargs(T=0, out=None)) == 0


def test_empty_inputs_are_no_ops(L):
    # T = 0: every entry point returns RAT_OK before touching a pointer or the GPU
    P = ctypes.c_void_p
    Dh = (ctypes.c_int32 * 2)(4, 16)
    assert L.rat_dilated_attn_prefill(None, None, None, None, 1, 2, 0, 128, 1, 4, 0, None, 0, 0.0,
                                      0.0, None) == 0
    assert L.rat_dilated_attn_prefill_sinks(None, None, None, None, 1, 2, 0, 128, 1, 4, 0, Dh, 4, 0,
                                            0.0, 0.0, None) == 0
    assert L.rat_dilated_attn_prefill_topk(None, None, None, None, 1, 2, 0, 128, 1, 4, 0, None, 0, 8,
                                           0, 0.0, 0.0, None) == 0
    assert L.rat_dilated_attn_backward(*([None] * 8), 1, 2, 0, 128, 1, 4, 0, None, 0, None, 0, 0.0,
                                       0.0, None, 0, None) == 0
    assert L.rat_recur_backward(*([None] * 16), 1, 2, 0, 128, 1, 0, 0.0, None, 0, None) == 0
    c = cache()
    c.k_dil = c.v_dil = c.k_win = c.v_win = c.h_k = c.h_v = 256
    assert L.rat_kv_compress(None, None, None, None, 0, ctypes.byref(c), None) == 0
    assert c.pos == 0


def test_option_limits(L):
    P = ctypes.c_void_p
    args = lambda top_k, n_sink: (P(256), P(256), P(256), P(256), 1, 1, 8, 128, 1, 4, 0, None,
                                  n_sink, top_k, 0, 0.0, 0.0, None)
    assert L.rat_dilated_attn_prefill_topk(*args(17, 0)) == -2      # at most 16 chunks
    assert L.rat_dilated_attn_prefill_topk(*args(-1, 0)) == -1
    assert L.rat_dilated_attn_prefill_topk(*args(2, -1)) == -1


def test_recur_workspace_grows_with_chunks(L):
    a = rat.rat_recur_workspace_bytes(1, 1, 128, 128, 1)
    b = rat.rat_recur_workspace_bytes(1, 1, 129, 128, 1)
    c = rat.rat_recur_workspace_bytes(4, 16, 4096, 128, 1)
    assert 256 < a < b < c
    assert rat.rat_recur_workspace_bytes(0, 1, 8, 128, 1) == 0


def test_attn_validation(L):
    P = ctypes.c_void_p
    ok = dict(q=P(256), k=P(256), v=P(256), o=P(256))
    args = lambda **kw: [kw.get(n, ok.get(n)) for n in ("q", "k", "v", "o")]
    # D < 1 with no per-head table
    assert L.rat_dilated_attn_prefill(*args(), 1, 1, 8, 128, 1, 0, 0, None, 0, 0.0, 0.0, None) == -1
    # W < 0
    assert L.rat_dilated_attn_prefill(*args(), 1, 1, 8, 128, 1, 1, -1, None, 0, 0.0, 0.0, None) == -1
    # per-head D with a zero
    Dh = (ctypes.c_int32 * 2)(4, 0)
    assert L.rat_dilated_attn_prefill(*args(), 1, 2, 8, 128, 1, 1, 0, Dh, 0, 0.0, 0.0, None) == -1
    # misaligned output
    assert L.rat_dilated_attn_prefill(*args(o=P(260)), 1, 1, 8, 128, 1, 1, 0, None, 0, 0.0, 0.0, None) == -1
    # unsupported head dim
    assert L.rat_dilated_attn_prefill(*args(), 1, 1, 8, 80, 1, 1, 0, None, 0, 0.0, 0.0, None) == -2
    # too many heads for the per-head table
    assert L.rat_dilated_attn_prefill(*args(), 1, 300, 8, 128, 1, 1, 0, None, 0, 0.0, 0.0, None) == -2


def cache(**kw):
    D = (ctypes.c_int32 * kw.get("H", 2))(*kw.get("Dlist", [1, 64]))
    c = rat.KVCache(B=kw.get("B", 2), H=kw.get("H", 2), d=kw.get("d", 128), W=kw.get("W", 16),
                    Tcap=kw.get("Tcap", 1024), dtype=kw.get("dtype", 1), D=D)
    c._keep = D
    return c


def test_cache_bytes_layout(L):
    c = cache()
    dil, win, state = rat.rat_kv_cache_bytes(c)
    # cap_h = floor(Tcap / D_h): 1024 + 16 entries per sequence, bf16 rows of 256 bytes
    assert dil == 2 * (1024 + 16) * 256
    assert win == 2 * 2 * 16 * 256
    assert state == 2 * 2 * 128 * 4
    bad = cache(Dlist=[1, 0])
    with pytest.raises(rat.RatError):
        rat.rat_kv_cache_bytes(bad)


def test_compress_and_decode_validation(L):
    P = ctypes.c_void_p
    c = cache()
    c.k_dil = c.v_dil = c.k_win = c.v_win = c.h_k = c.h_v = 256
    # beyond capacity
    c.pos = 1000
    assert L.rat_kv_compress(P(256), P(256), None, None, 100, ctypes.byref(c), None) == -1
    # decode at pos == Tcap
    c.pos = 1024
    ws = P(256 * 4096)
    assert L.rat_dilated_decode(P(256), P(256), P(256), P(256), ctypes.byref(c), P(256), 0.0, 0.0,
                                ws, 1 << 30, None) == -1
    # decode with a too-small workspace
    c.pos = 5
    need = rat.rat_decode_workspace_bytes(c)
    assert need > 256
    assert L.rat_dilated_decode(P(256), P(256), P(256), P(256), ctypes.byref(c), P(256), 0.0, 0.0,
                                ws, need - 1, None) == -5
    # fp32 decode is not provided
    c32 = cache(dtype=0)
    c32.k_dil = c32.v_dil = c32.k_win = c32.v_win = c32.h_k = c32.h_v = 256
    assert L.rat_dilated_decode(P(256), P(256), P(256), P(256), ctypes.byref(c32), P(256), 0.0, 0.0,
                                ws, 1 << 30, None) == -2


def test_cache_rejects_negative_block_length(L):
    c = cache()
    c.reset_every = -1
    sz = ctypes.c_size_t()
    assert L.rat_kv_cache_bytes(ctypes.byref(c), ctypes.byref(sz), None, None) == -1
    c.reset_every = 16
    assert L.rat_kv_cache_bytes(ctypes.byref(c), ctypes.byref(sz), None, None) == 0


def test_window_cache_validation(L):
    # the fixed-window form: window_rec 64 only, no chunk-local restarts, raw rings required by
    # the calls that use them (not by the size helpers)
    P = ctypes.c_void_p
    c = cache()
    c.window_rec = 64
    assert rat.rat_kv_raw_bytes(c) == 2 * 2 * 64 * 128 * 2
    sz = ctypes.c_size_t()
    assert L.rat_kv_cache_bytes(ctypes.byref(c), ctypes.byref(sz), None, None) == 0
    c.window_rec = 32
    assert rat.rat_kv_raw_bytes(c) == 0
    assert L.rat_kv_cache_bytes(ctypes.byref(c), ctypes.byref(sz), None, None) == -1
    c.window_rec = 64
    c.reset_every = 16
    assert L.rat_kv_cache_bytes(ctypes.byref(c), ctypes.byref(sz), None, None) == -1
    c.reset_every = 0
    c.k_dil = c.v_dil = c.k_win = c.v_win = c.h_k = c.h_v = 256
    # raw rings missing: refused by the window compress and by decode
    assert L.rat_kv_compress_window(P(256), P(256), P(256), P(256), P(256), 10, ctypes.byref(c), None) == -1
    ws = P(256 * 4096)
    assert L.rat_dilated_decode(P(256), P(256), P(256), P(256), ctypes.byref(c), P(256), 0.0, 0.0,
                                ws, 1 << 30, None) == -1
    # the plain compress refuses a window cache even with its rings
    c.k_raw = c.v_raw = c.a_raw = 256
    assert L.rat_kv_compress(P(256), P(256), None, None, 10, ctypes.byref(c), None) == -1
    # and the window compress refuses a cache without the window form
    c2 = cache()
    c2.k_dil = c2.v_dil = c2.k_win = c2.v_win = c2.h_k = c2.h_v = 256
    assert L.rat_kv_compress_window(P(256), P(256), P(256), P(256), P(256), 10, ctypes.byref(c2), None) == -1
    assert rat.rat_kv_raw_bytes(c2) == 0


def paged(**kw):
    D = (ctypes.c_int32 * kw.get("H", 2))(*kw.get("Dlist", [1, 64]))
    c = rat.PagedKVCache(B=kw.get("B", 2), H=kw.get("H", 2), d=kw.get("d", 128), W=kw.get("W", 16),
                         dtype=kw.get("dtype", 1), page_entries=kw.get("pe", 64),
                         max_pages=kw.get("max_pages", 8), n_pages=kw.get("n_pages", 32), D=D)
    c._keep = D
    c.k_pool = c.v_pool = c.k_win = c.v_win = c.h_k = c.h_v = c.pos = c.page_table = 256
    return c


def test_paged_validation(L):
    P = ctypes.c_void_p
    ws = P(256 * 4096)
    ok = paged()
    need = rat.rat_paged_decode_workspace_bytes(ok)
    assert need > 256
    args = lambda c, wsb=need: (P(256), P(256), P(256), P(256), ctypes.byref(c), P(256), 0.0, 0.0,
                                ws, wsb, None)
    # page_entries must be a power of two; pool and table sizes at least 1
    for bad in (paged(pe=48), paged(pe=0), paged(max_pages=0), paged(n_pages=0)):
        assert rat.rat_paged_decode_workspace_bytes(bad) == 0
        assert L.rat_dilated_decode_paged(*args(bad)) == -1
    # missing page table or positions
    c = paged()
    c.page_table = None
    assert L.rat_dilated_decode_paged(*args(c)) == -1
    c = paged()
    c.pos = None
    assert L.rat_dilated_decode_paged(*args(c)) == -1
    # float32 decode is not provided; the workspace must be large enough
    assert L.rat_dilated_decode_paged(*args(paged(dtype=0))) == -2
    assert L.rat_dilated_decode_paged(*args(ok, need - 1)) == -5
    # compress: sequence index in range, workspace header present
    assert L.rat_paged_kv_compress(P(256), P(256), None, None, 8, 2, 0, ctypes.byref(ok), ws, 256,
                                   None) == -1
    assert L.rat_paged_kv_compress(P(256), P(256), None, None, 8, 0, -1, ctypes.byref(ok), ws, 256,
                                   None) == -1
    assert L.rat_paged_kv_compress(P(256), P(256), None, None, 8, 0, 0, ctypes.byref(ok), None, 256,
                                   None) == -5
    assert L.rat_paged_kv_compress(None, None, None, None, 0, 0, 0, ctypes.byref(ok), ws, 256,
                                   None) == 0


def test_workspace_init_rejects_null(L):
    assert L.rat_workspace_init(None, 1024, None) == -5
    assert L.rat_sync_status(None, None) == -5


def test_binding_refuses_host_tensors():
    # the binding passes device addresses only: a host tensor is refused before any library call
    import torch
    k = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16)
    with pytest.raises(rat.RatError) as e:
        rat.rat_recur_prefill(k, k, k, k, k, ws=None)
    assert e.value.status == -1
    with pytest.raises(rat.RatError) as e:
        rat.rat_dilated_attn_prefill(k, k, k, k, D=4)
    assert e.value.status == -1
    assert rat._ptr(None) is None
