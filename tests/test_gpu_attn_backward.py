"""GPU parity of rat_dilated_attn_backward (gradients of the dilated attention) against the
float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import TOL_BF16, TOL_F32, f64, gpu_attn, rel_err, tol_for

pytestmark = pytest.mark.gpu


def run(B, H, T, d, dtype, D=1, W=0, D_per_head=None, rope_base=0.0, pos0=0, seed=0, heads=None,
        x=None):
    if x is None:
        w = synthetic.Workload("ab", B=B, H=H, d=d, T=T, dtype="f32" if dtype == torch.float32 else "bf16",
                               seed=seed)
        x = synthetic.prefill_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))     # k, v stand in for k~, v~
    g = torch.Generator().manual_seed(seed + 1)
    dO = torch.randn(q.shape, generator=g).to(dtype)
    o = gpu_attn(q, k, v, D=D, W=W, D_per_head=D_per_head, rope_base=rope_base, pos0=pos0)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = rat.Workspace(rat.rat_dilated_attn_backward_workspace_bytes(B, H, T, d, 0 if dtype == torch.float32 else 1))
    rat.rat_dilated_attn_backward(q, k, v, o, dO.to(dev), dq, dk, dv, ws, D=D, W=W,
                                  D_per_head=D_per_head, pos0=pos0, rope_base=rope_base)
    torch.cuda.synchronize()
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    errs = {}
    for b, h in sel:
        Dh = [D_per_head[h]] if D_per_head is not None else None
        ref = oracle.dilated_attention_backward(
            f64(x["q"][b:b + 1, h:h + 1]), f64(x["k"][b:b + 1, h:h + 1]), f64(x["v"][b:b + 1, h:h + 1]),
            f64(dO[b:b + 1, h:h + 1]), D=D, W=W, D_per_head=Dh, rope_base=rope_base, pos0=pos0)
        for n, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            errs[(b, h, n)] = rel_err(got[b, h], r[0, 0])
    tol = tol_for(dtype)
    worst = max(errs.values())
    assert worst <= tol, {k_: v_ for k_, v_ in errs.items() if v_ > tol}
    return worst


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("D,W", [(1, 0), (4, 0), (16, 0), (4, 8), (64, 128), (7, 3)])
def test_attention_backward_key_sets(dtype, d, D, W):
    run(1, 2, 300, d, dtype, D=D, W=W, seed=D * 10 + W)


@pytest.mark.parametrize("T", [1, 2, 65, 129])
def test_attention_backward_short_and_ragged(T):
    run(2, 2, T, 128, torch.bfloat16, D=4, W=2, seed=T)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_attention_backward_rope_and_head_hybrid(dtype):
    run(1, 4, 257, 128, dtype, D_per_head=[1, 4, 16, 64], W=8, rope_base=10000.0, pos0=4000, seed=3)


def test_attention_backward_full_size_sampled_heads():
    # the prefill_1p5b workload (B 4, H 16, T 4096, d 128, D 16, RoPE), two heads checked whole
    w = synthetic.WORKLOADS["prefill_1p5b"]
    x = synthetic.prefill_inputs(w)
    run(w.B, w.H, w.T, w.d, torch.bfloat16, D=w.D, W=w.W, rope_base=w.rope_base, x=x,
        heads=[(0, 0), (w.B - 1, w.H - 1)], seed=5)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_forward_lse_and_backward_with_it(dtype, d):
    # the forward's log-sum-exp (tensor-core kernel for bf16 d 128, CUDA-core otherwise) against
    # the oracle's, and the backward fed with it equal to the backward that recomputes it
    B, H, T = 1, 3, 333
    w = synthetic.Workload("lse", B=B, H=H, d=d, T=T, dtype="f32" if dtype == torch.float32 else "bf16",
                           seed=21)
    x = synthetic.prefill_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    kw = dict(D_per_head=[1, 16, 64], W=0, rope_base=10000.0)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    rat.rat_dilated_attn_prefill(q, k, v, o, lse=lse, **kw)
    qr = oracle.rope(f64(x["q"]), 0, 10000.0)
    _, ref = oracle.dilated_attention(qr, f64(x["k"]), f64(x["v"]), W=0, D_per_head=[1, 16, 64],
                                      return_lse=True)
    tol_abs = 2e-2 if dtype == torch.bfloat16 else 1e-4
    assert float(np.max(np.abs(f64(lse) - ref))) <= tol_abs * max(1.0, float(np.max(np.abs(ref))))
    g = torch.Generator().manual_seed(22)
    dO = torch.randn(q.shape, generator=g).to(dtype).to(dev)
    ws = rat.Workspace(rat.rat_dilated_attn_backward_workspace_bytes(B, H, T, d,
                                                                     0 if dtype == torch.float32 else 1))
    outs = []
    for given in (None, lse):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        rat.rat_dilated_attn_backward(q, k, v, o, dO, dq, dk, dv, ws, lse=given, **kw)
        outs.append((dq, dk, dv))
    ref_b = oracle.dilated_attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(dO), **kw)
    for got in outs:
        for gg, r in zip(got, ref_b):
            assert rel_err(gg, r) <= tol_for(dtype)


# bf16, d 128 without sinks runs on the tensor cores (dq and dk/dv launches): several query tiles
# and key blocks with ragged tails, every key-set shape (dense, chunk ends only, chunk ends plus
# a wide window, no chunk end inside the sequence, self key only), RoPE at an offset
@pytest.mark.parametrize("T", [63, 64, 130, 1000])
@pytest.mark.parametrize("D,W", [(1, 0), (3, 0), (8, 100), (600, 0), (16, 1)])
def test_attention_backward_tensor_core_tiles(T, D, W):
    run(1, 2, T, 128, torch.bfloat16, D=D, W=W, seed=T + D + W, rope_base=10000.0, pos0=7)


def test_attention_backward_head_hybrid_lse_given():
    # a dense head and four dilations in one launch, the forward's log-sum-exp passed in
    B, H, T, d = 2, 6, 700, 128
    Dh = [1, 2, 5, 64, 300, 1]
    w = synthetic.Workload("hy", B=B, H=H, d=d, T=T, dtype="bf16", seed=31)
    x = synthetic.prefill_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    rat.rat_dilated_attn_prefill(q, k, v, o, D_per_head=Dh, W=4, rope_base=500.0, lse=lse)
    g = torch.Generator().manual_seed(32)
    dO = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = rat.Workspace(rat.rat_dilated_attn_backward_workspace_bytes(B, H, T, d, 1))
    rat.rat_dilated_attn_backward(q, k, v, o, dO.to(dev), dq, dk, dv, ws, D_per_head=Dh, W=4,
                                  rope_base=500.0, lse=lse)
    assert rat.rat_sync_status(ws) == 0
    ref = oracle.dilated_attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(dO),
                                            W=4, D_per_head=Dh, rope_base=500.0)
    for got, r in zip((dq, dk, dv), ref):
        assert rel_err(got, r) <= TOL_BF16


def test_attention_backward_five_dilations_take_the_cuda_core_path():
    # more than four distinct dilations in one call: the CUDA-core kernels, same results (the
    # bf16 forward takes at most four, so o comes from the oracle, rounded to bf16)
    B, H, T, d = 1, 5, 200, 128
    Dh = [2, 3, 4, 5, 6]
    w = synthetic.Workload("d5", B=B, H=H, d=d, T=T, dtype="bf16", seed=41)
    x = synthetic.prefill_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.from_numpy(oracle.dilated_attention(f64(x["q"]), f64(x["k"]), f64(x["v"]), W=2,
                                                  D_per_head=Dh)).to(torch.bfloat16).to(dev)
    g = torch.Generator().manual_seed(42)
    dO = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = rat.Workspace(rat.rat_dilated_attn_backward_workspace_bytes(B, H, T, d, 1))
    rat.rat_dilated_attn_backward(q, k, v, o, dO.to(dev), dq, dk, dv, ws, D_per_head=Dh, W=2)
    assert rat.rat_sync_status(ws) == 0
    ref = oracle.dilated_attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(dO), W=2,
                                            D_per_head=Dh)
    for got, r in zip((dq, dk, dv), ref):
        assert rel_err(got, r) <= TOL_BF16


def test_attention_backward_window_2p6b_sampled_heads():
    # the window_2p6b workload (B 2, H 20, T 16384, D 64, W 128) at full size, two heads checked
    w = synthetic.WORKLOADS["window_2p6b"]
    x = synthetic.prefill_inputs(w)
    run(w.B, w.H, w.T, w.d, torch.bfloat16, D=w.D, W=w.W, x=x, heads=[(0, 3), (1, 19)], seed=6)


# chunk-end key blocks whose query walks span many 64-query tiles (T > 1024), with ragged last
# tiles, blocks whose first key lies deep in the sequence, a window beside the chunk ends, and a
# launch that mixes a dense head (64-key dq blocks) with dilated ones
@pytest.mark.parametrize("T,D,W", [(1025, 16, 0), (2500, 37, 3), (3000, 200, 70)])
def test_attention_backward_long_walks(T, D, W):
    run(1, 2, T, 128, torch.bfloat16, D=D, W=W, seed=T + D, rope_base=10000.0, pos0=11)


def test_attention_backward_long_walks_head_hybrid():
    run(1, 3, 2100, 128, torch.bfloat16, D_per_head=[1, 16, 64], W=4, seed=99)
