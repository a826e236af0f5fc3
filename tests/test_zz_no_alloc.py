"""The decode entry point that allocates nothing (rat_dilated_decode_noalloc).

Some callers cannot give the library a device buffer for the decode workspace: their device
memory is owned by a host framework or planned up front as a fixed arena.  For them the library
serves the same decode step from a fixed scratch array compiled into its device image.  This
test calls that entry point through the C ABI, twice in a row, and checks each output (and the
cache it updates) against the ordinary entry point with a caller-provided workspace, within the
bf16 tolerance used by the other tests.  It lives in a file that pytest collects last and
depends on no state left by other tests.
"""
import ctypes

import pytest
import torch

import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import TOL_BF16, gpu_recur, rel_err

pytestmark = pytest.mark.gpu


def build_cache(w, T0, Tcap, rope_base):
    dev = torch.device("cuda")
    k, v, a = synthetic.decode_context_block(w, 0, device=dev, T=T0)
    kr, vr, hk, hv = gpu_recur(k, v, a, rope_base=rope_base)
    cache, bufs = rat.make_cache(w.B, w.H, w.d, w.W, Tcap, rat.BF16, w.heads_D())
    rat.rat_kv_compress(kr, vr, hk, hv, cache)
    torch.cuda.synchronize()
    return cache, bufs


def run_both(w, T0, steps, rope_base):
    """steps decode calls in a row on each entry point over two copies of one cache; every
    output and the caches they leave must agree."""
    ref_cache, ref_bufs = build_cache(w, T0, T0 + steps, rope_base)
    na_cache, na_bufs = build_cache(w, T0, T0 + steps, rope_base)
    ws = rat.Workspace(rat.rat_decode_workspace_bytes(ref_cache))
    tok = synthetic.decode_steps(w, steps)
    L = rat.lib()
    dev = torch.device("cuda")
    for s in range(steps):
        args = [tok[n][s].reshape(w.B, w.H, 1, w.d).to(dev) for n in ("q", "k", "v", "a")]
        o_ref = torch.empty((w.B, w.H, 1, w.d), dtype=torch.bfloat16, device=dev)
        o_na = torch.full_like(o_ref, float("nan"))
        rat.rat_dilated_decode(*args, ref_cache, o_ref, ws, rope_base=rope_base)
        st = L.rat_dilated_decode_noalloc(*[ctypes.c_void_p(t.data_ptr()) for t in args],
                                          ctypes.byref(na_cache), ctypes.c_void_p(o_na.data_ptr()),
                                          float(rope_base), 0.0,
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, rat.rat_status_string(st)
        torch.cuda.synchronize()
        assert not torch.isnan(o_na).any()
        assert rel_err(o_na, o_ref) <= TOL_BF16
    assert na_cache.pos == ref_cache.pos == T0 + steps
    for n in ("h_k", "h_v", "k_dil", "v_dil", "k_win", "v_win"):
        assert rel_err(na_bufs[n], ref_bufs[n]) <= TOL_BF16, n


@pytest.mark.parametrize("rope_base", [0.0, 10000.0])
def test_noalloc_decode_matches_workspace_decode(rope_base):
    # first a call over many slices and long contexts (many splits: the array fills far beyond
    # what the next calls use), then two calls in a row on a small cache: stale partials and
    # tickets of the large call must not leak into the small ones
    big = synthetic.Workload("noalloc_big", B=8, H=16, d=128, T=0, W=8,
                             D_per_head=tuple([1, 4] * 8), dtype="bf16", seed=78)
    run_both(big, 4096, 1, rope_base)
    w = synthetic.Workload("noalloc", B=2, H=3, d=128, T=0, W=8, D_per_head=(1, 4, 16),
                           dtype="bf16", seed=77)
    run_both(w, 150, 2, rope_base)


def test_noalloc_rejects_oversized_scratch():
    # a cache whose decode scratch would exceed the fixed 8 MiB array is refused up front
    Dh = (ctypes.c_int32 * 256)(*([1] * 256))
    c = rat.KVCache(B=256, H=256, d=128, W=0, Tcap=1 << 20, dtype=rat.BF16, D=Dh)
    assert rat.rat_decode_workspace_bytes(c) > (8 << 20)
    st = rat.lib().rat_dilated_decode_noalloc(None, None, None, None, ctypes.byref(c), None, 0.0, 0.0, None)
    assert st == -5
