"""GPU parity of rat_kv_compress (bit-exact cache layout) and rat_dilated_decode."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import TOL_BF16, TOL_F32, f64, gpu_recur, rel_err

pytestmark = pytest.mark.gpu

POISON = -12345.0     # exactly representable in bf16 and float32


def tagged(B, H, T, d, dtype, pos0=0):
    """Rows whose channels encode their own (position, slice) index, exact in the dtype."""
    x = torch.zeros((B, H, T, d), dtype=torch.float32)
    t = torch.arange(pos0, pos0 + T, dtype=torch.float32)
    if dtype == torch.float32:
        x[..., 0] = t
        x[..., 1] = (torch.arange(B)[:, None] * H + torch.arange(H)[None, :]).float()[:, :, None]
        x[..., 2:] = torch.arange(2, d).float()
    else:
        x[..., 0] = torch.floor(t / 256)
        x[..., 1] = t % 256
        x[..., 2] = (torch.arange(B)[:, None] * H + torch.arange(H)[None, :]).float()[:, :, None]
        x[..., 3:] = (torch.arange(3, d) % 256).float()
    return x.to(dtype)


def as_np(t):
    """Raw element storage as a numpy array (bf16 viewed as uint16)."""
    t = t.cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_compress_index_layout_bit_exact(dtype, d):
    B, H, T, W, Tcap = 2, 3, 1000, 16, 1100
    Dh = [1, 4, 64]
    kr = tagged(B, H, T, d, dtype)
    vr = -tagged(B, H, T, d, dtype)
    cache, bufs = rat.make_cache(B, H, d, W, Tcap, rat.F32 if dtype == torch.float32 else rat.BF16, Dh)
    for n in ("k_dil", "v_dil", "k_win", "v_win"):
        bufs[n].fill_(POISON)
    hk = torch.randn((B, H, d)).cuda()
    hv = torch.randn((B, H, d)).cuda()
    rat.rat_kv_compress(kr.cuda(), vr.cuda(), hk, hv, cache)
    torch.cuda.synchronize()
    assert cache.pos == T
    for name, src in (("k", kr), ("v", vr)):
        dil0 = np.full(bufs[name + "_dil"].shape, as_np(torch.tensor([POISON], dtype=dtype))[0])
        win0 = np.full(bufs[name + "_win"].shape, as_np(torch.tensor([POISON], dtype=dtype))[0])
        dil, win = oracle.kv_compress(as_np(src), Dh, W, Tcap, dil=dil0, ring=win0)
        assert np.array_equal(as_np(bufs[name + "_dil"]), dil)
        assert np.array_equal(as_np(bufs[name + "_win"]), win)
    assert torch.equal(bufs["h_k"], hk) and torch.equal(bufs["h_v"], hv)


def test_compress_chunked_equals_whole():
    B, H, T, d, W, Tcap = 1, 2, 700, 128, 32, 800
    Dh = [4, 16]
    kr = tagged(B, H, T, d, torch.bfloat16)
    c1, b1 = rat.make_cache(B, H, d, W, Tcap, rat.BF16, Dh)
    c2, b2 = rat.make_cache(B, H, d, W, Tcap, rat.BF16, Dh)
    h = torch.zeros((B, H, d)).cuda()
    rat.rat_kv_compress(kr.cuda(), kr.cuda(), h, h, c1)
    for lo, hi in ((0, 250), (250, 251), (251, 700)):
        part = kr[:, :, lo:hi].contiguous().cuda()
        rat.rat_kv_compress(part, part, h, h, c2)
    torch.cuda.synchronize()
    assert c1.pos == c2.pos == T
    for n in ("k_dil", "v_dil", "k_win", "v_win"):
        assert torch.equal(b1[n], b2[n]), n


def run_decode(w, T0, steps, heads_check, B=None, H=None, rope_base=0.0, reset_every=0, n_sink=0):
    """GPU: prefill a T0-token context, compress, then decode `steps` tokens.
    Oracle: the same from the same raw inputs on the (b, h) slices in heads_check."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    d, W = w.d, w.W
    Dh = w.heads_D()[:H]
    Tcap = T0 + steps
    dev = torch.device("cuda")
    cache, bufs = rat.make_cache(B, H, d, W, Tcap, rat.BF16, Dh, reset_every=reset_every,
                                 n_sink=n_sink)
    hk = torch.zeros((B, H, d), dtype=torch.float32, device=dev)
    hv = torch.zeros_like(hk)
    nchunks = (T0 + synthetic.CTX_CHUNK - 1) // synthetic.CTX_CHUNK
    for c in range(nchunks):     # chunked prefill of the context: state carried, cache appended
        k, v, a = synthetic.decode_context_block(w, c, device=dev, T=T0, B=B, H=H)
        kr, vr, hk, hv = gpu_recur(k, v, a, rope_base=rope_base, pos0=cache.pos, h0k=hk, h0v=hv,
                                   reset_every=reset_every)
        rat.rat_kv_compress(kr, vr, hk, hv, cache)
        del k, v, a, kr, vr
    tok = synthetic.decode_steps(w, steps)
    tok = {n: t[:, :B, :H].contiguous() for n, t in tok.items()}
    ws = rat.Workspace(rat.rat_decode_workspace_bytes(cache))
    outs = []
    for s in range(steps):
        o = torch.empty((B, H, 1, d), dtype=torch.bfloat16, device=dev)
        args = [tok[n][s].reshape(B, H, 1, d).to(dev) for n in ("q", "k", "v", "a")]
        rat.rat_dilated_decode(*args, cache, o, ws, rope_base=rope_base)
        outs.append(o)
    assert rat.rat_sync_status(ws) == 0
    assert cache.pos == Tcap
    got = torch.stack(outs)[:, :, :, 0]            # (steps, B, H, d)
    # oracle on the checked slices
    st = oracle.DecodeState([Dh[h] for _, h in heads_check], d, W, Tcap, rope_base=rope_base,
                            reset_every=reset_every, n_sink=n_sink)
    ctx = [synthetic.decode_context_slice(w, b, h, device=dev, T=T0) for b, h in heads_check]
    st.prefill(np.stack([f64(x[0]) for x in ctx]), np.stack([f64(x[1]) for x in ctx]),
               np.stack([f64(x[2]) for x in ctx]))
    del ctx
    errs = []
    for s in range(steps):
        sel = lambda n: np.stack([f64(tok[n][s, b, h]) for b, h in heads_check])
        ref = st.step(sel("q"), sel("k"), sel("v"), sel("a"))
        errs.append(rel_err(torch.stack([got[s, b, h] for b, h in heads_check]), ref))
    hk_ref = st.hk
    hk_got = np.stack([f64(bufs["h_k"][b, h]) for b, h in heads_check])
    return max(errs), rel_err(hk_got, hk_ref)


@pytest.mark.parametrize("rope_base", [0.0, 10000.0])
def test_decode_small(rope_base):
    w = synthetic.Workload("dec_small", B=2, H=3, d=128, T=0, W=8, D_per_head=(1, 4, 16),
                           dtype="bf16", seed=40)
    heads = [(b, h) for b in range(2) for h in range(3)]
    err, herr = run_decode(w, T0=100, steps=40, heads_check=heads, rope_base=rope_base)
    assert err <= TOL_BF16, err
    assert herr <= TOL_F32, herr


def test_decode_no_window():
    w = synthetic.Workload("dec_w0", B=1, H=2, d=128, T=0, W=0, D_per_head=(4, 64), dtype="bf16", seed=41)
    err, herr = run_decode(w, T0=130, steps=70, heads_check=[(0, 0), (0, 1)])
    assert err <= TOL_BF16 and herr <= TOL_F32


def test_decode_full_size_sampled():
    w = synthetic.WORKLOADS["decode_7p6b"]
    err, herr = run_decode(w, T0=w.T, steps=8, heads_check=[(0, 0), (w.B - 1, w.H - 1), (5, 17)])
    assert err <= TOL_BF16, err
    assert herr <= TOL_F32, herr


@pytest.mark.parametrize("L", [1, 16, 50])
def test_decode_local_recurrence(L):
    # RAT's chunk-local recurrence in decode: the context ends inside a block (100 mod L != 0 for
    # L = 16, 50) and the decoded tokens cross block starts; L = 16 equals the largest head's D
    w = synthetic.Workload("dec_local", B=2, H=3, d=128, T=0, W=8, D_per_head=(1, 4, 16),
                           dtype="bf16", seed=42)
    heads = [(b, h) for b in range(2) for h in range(3)]
    err, herr = run_decode(w, T0=100, steps=40, heads_check=heads, rope_base=10000.0,
                           reset_every=L)
    assert err <= TOL_BF16, err
    assert herr <= TOL_F32, herr


# ---- decode with the fixed-window recurrence (L* = 64): raw rings of the last 64 positions
def run_window_decode(w, T0, steps, chunk, rope_base=0.0):
    """GPU: the context prefilled in chunks by rat_recur_prefill_window (each chunk with the 64
    raw rows before it as history) and appended by rat_kv_compress_window, then `steps` decode
    tokens.  Oracle: DecodeState(window_rec=64) from the same raw inputs on every slice."""
    B, H, d, W = w.B, w.H, w.d, w.W
    Dh = w.heads_D()
    Tcap = T0 + steps
    dev = torch.device("cuda")
    cache, bufs = rat.make_cache(B, H, d, W, Tcap, rat.BF16, Dh, window_rec=64)
    for n in ("k_raw", "v_raw", "a_raw"):
        bufs[n].fill_(POISON)
    x = synthetic.prefill_inputs(w, T=T0)
    ws = rat.Workspace(256)
    for lo in range(0, T0, chunk):
        hi = min(T0, lo + chunk)
        k, v, a = (x[n][:, :, lo:hi].contiguous().to(dev) for n in ("k", "v", "a"))
        kr, vr = torch.empty_like(k), torch.empty_like(v)
        prev = {}
        if lo >= 64:
            prev = {n: x[m][:, :, lo - 64:lo].contiguous().to(dev)
                    for n, m in (("prev_k", "k"), ("prev_v", "v"), ("prev_gate_logit", "a"))}
        rat.rat_recur_prefill_window(k, v, a, kr, vr, ws, 64, pos0=lo, rope_base=rope_base, **prev)
        rat.rat_kv_compress_window(kr, vr, k, v, a, cache)
    assert rat.rat_sync_status(ws) == 0
    assert cache.pos == T0
    # the raw rings hold the last 64 raw rows, position p in slot p mod 64, bit for bit
    for n, m in (("k_raw", "k"), ("v_raw", "v"), ("a_raw", "a")):
        exp = torch.full((B, H, 64, d), POISON, dtype=torch.bfloat16)
        for p in range(max(0, T0 - 64), T0):
            exp[:, :, p % 64] = x[m][:, :, p]
        assert torch.equal(bufs[n].cpu(), exp), n
    tok = synthetic.decode_steps(w, steps)
    wsd = rat.Workspace(rat.rat_decode_workspace_bytes(cache))
    st = oracle.DecodeState([Dh[h] for b in range(B) for h in range(H)], d, W, Tcap,
                            rope_base=rope_base, window_rec=64)
    st.prefill(f64(x["k"]).reshape(B * H, T0, d), f64(x["v"]).reshape(B * H, T0, d),
               f64(x["a"]).reshape(B * H, T0, d))
    worst = 0.0
    for s in range(steps):
        o = torch.empty((B, H, 1, d), dtype=torch.bfloat16, device=dev)
        args = [tok[n][s].reshape(B, H, 1, d).to(dev) for n in ("q", "k", "v", "a")]
        rat.rat_dilated_decode(*args, cache, o, wsd, rope_base=rope_base)
        ref = st.step(*(f64(tok[n][s]).reshape(B * H, d) for n in ("q", "k", "v", "a")))
        worst = max(worst, rel_err(o.reshape(B * H, d), ref))
    assert rat.rat_sync_status(wsd) == 0
    assert cache.pos == Tcap
    return worst


@pytest.mark.parametrize("T0,chunk,rope_base", [(200, 200, 0.0), (300, 128, 10000.0), (40, 40, 10000.0)])
def test_window_decode(T0, chunk, rope_base):
    # contexts longer than the window (in one chunk and in three), and shorter than it (the
    # window still filling during the decode steps)
    w = synthetic.Workload("wdec", B=2, H=3, d=128, T=T0, W=8, D_per_head=(1, 4, 16),
                           dtype="bf16", seed=T0 + chunk)
    assert run_window_decode(w, T0, 70, chunk, rope_base) <= TOL_BF16


def test_window_cache_refuses_the_plain_compress():
    # a window cache must also receive the raw rows: rat_kv_compress refuses it
    cache, _ = rat.make_cache(1, 1, 128, 4, 100, rat.BF16, [4], window_rec=64)
    x = torch.zeros((1, 1, 10, 128), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((1, 1, 128), device="cuda")
    with pytest.raises(rat.RatError):
        rat.rat_kv_compress(x, x, h, h, cache)
