"""GPU parity of attention sinks (StreamingLLM layers: the first n_sink positions join every key
set): prefill attention and its backward, the cache's sink rows, and decode."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import TOL_BF16, TOL_F32, f64, gpu_recur, rel_err, tol_for
from test_gpu_cache import run_decode

pytestmark = pytest.mark.gpu

NO_CHUNK_ENDS = 1 << 30          # a StreamingLLM layer: no dilated keys


def inputs(B, H, T, d, dtype, seed):
    w = synthetic.Workload("s", B=B, H=H, d=d, T=T, dtype="f32" if dtype == torch.float32 else "bf16",
                           seed=seed)
    return synthetic.prefill_inputs(w)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("D,W,n_sink", [(NO_CHUNK_ENDS, 16, 4), (NO_CHUNK_ENDS, 1, 7), (16, 8, 4),
                                        (4, 0, 10)])
def test_prefill_attention_with_sinks(dtype, d, D, W, n_sink):
    x = inputs(2, 2, 300, d, dtype, seed=n_sink + W)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    rat.rat_dilated_attn_prefill(q, k, v, o, D=D, W=W, n_sink=n_sink, rope_base=10000.0, pos0=3)
    qr = oracle.rope(f64(x["q"]), 3, 10000.0)
    ref = oracle.dilated_attention(qr, f64(x["k"]), f64(x["v"]), D=D, W=W, n_sink=n_sink)
    assert rel_err(o, ref) <= tol_for(dtype)


def test_sinks_with_per_head_dilation():
    x = inputs(1, 3, 513, 128, torch.bfloat16, seed=9)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    Dh = [1, 8, NO_CHUNK_ENDS]
    rat.rat_dilated_attn_prefill(q, k, v, o, W=32, D_per_head=Dh, n_sink=4)
    ref = oracle.dilated_attention(f64(x["q"]), f64(x["k"]), f64(x["v"]), W=32, D_per_head=Dh,
                                   n_sink=4)
    assert rel_err(o, ref) <= TOL_BF16


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_attention_backward_with_sinks(dtype):
    x = inputs(1, 2, 257, 128, dtype, seed=11)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    kw = dict(D=16, W=8, n_sink=4, rope_base=10000.0)
    rat.rat_dilated_attn_prefill(q, k, v, o, **kw)
    g = torch.Generator().manual_seed(12)
    dO = torch.randn(q.shape, generator=g).to(dtype)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = rat.Workspace(rat.rat_dilated_attn_backward_workspace_bytes(1, 2, 257, 128,
                                                                     0 if dtype == torch.float32 else 1))
    rat.rat_dilated_attn_backward(q, k, v, o, dO.to(dev), dq, dk, dv, ws, **kw)
    ref = oracle.dilated_attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(dO), **kw)
    for got, r in zip((dq, dk, dv), ref):
        assert rel_err(got, r) <= tol_for(dtype)


def test_compress_keeps_the_sink_rows_bit_exact():
    w = synthetic.Workload("sk", B=2, H=2, d=128, T=0, W=8, D_per_head=(4, 16), dtype="bf16", seed=13)
    dev = torch.device("cuda")
    cache, bufs = rat.make_cache(2, 2, 128, 8, 200, rat.BF16, [4, 16], n_sink=6)
    k, v, a = synthetic.decode_context_block(w, 0, device=dev, T=100, B=2, H=2)
    kr, vr, hk, hv = gpu_recur(k[:, :, :3].contiguous(), v[:, :, :3].contiguous(), a[:, :, :3].contiguous())
    rat.rat_kv_compress(kr, vr, hk, hv, cache)               # positions 0..2
    kr2, vr2, hk2, hv2 = gpu_recur(k[:, :, 3:].contiguous(), v[:, :, 3:].contiguous(),
                                   a[:, :, 3:].contiguous(), pos0=3, h0k=hk, h0v=hv)
    rat.rat_kv_compress(kr2, vr2, hk2, hv2, cache)           # positions 3..99
    assert torch.equal(bufs["k_sink"][:, :, :3], kr[:, :, :3])
    assert torch.equal(bufs["k_sink"][:, :, 3:6], kr2[:, :, :3])
    assert torch.equal(bufs["v_sink"][:, :, 3:6], vr2[:, :, :3])


@pytest.mark.parametrize("D_per_head,W", [((NO_CHUNK_ENDS, NO_CHUNK_ENDS, 16), 8), ((1, 4, 64), 0)])
def test_decode_with_sinks(D_per_head, W):
    # the context ends before, at and after the sinks are filled (T0 = 2 < n_sink on one run)
    w = synthetic.Workload("dec_sink", B=2, H=3, d=128, T=0, W=W, D_per_head=D_per_head,
                           dtype="bf16", seed=14)
    heads = [(b, h) for b in range(2) for h in range(3)]
    for T0 in (2, 100):
        err, herr = run_decode(w, T0=T0, steps=30, heads_check=heads, rope_base=10000.0, n_sink=4)
        assert err <= TOL_BF16, (T0, err)
        assert herr <= TOL_F32, herr
