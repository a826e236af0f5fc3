"""GPU parity of rat_recur_backward (gradients of the prefill recurrence step) against the
float64 oracle's reverse loop."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import TOL_BF16, TOL_F32, f64, gpu_recur, rel_err, tol_for

pytestmark = pytest.mark.gpu


def inputs(B, H, T, d, dtype, seed=0, mu=2.0, sigma=1.0):
    w = synthetic.Workload("b", B=B, H=H, d=d, T=T, dtype="f32" if dtype == torch.float32 else "bf16",
                           gate_mu=mu, gate_sigma=sigma, seed=seed)
    return synthetic.prefill_inputs(w)


def gpu_backward(x, dyk, dyv, h0=None, dhT=None, pos0=0, rope_base=0.0, reset_every=0):
    dev = torch.device("cuda")
    k, v, a = (x[n].to(dev) for n in ("k", "v", "a"))
    B, H, T, d = k.shape
    h0k = h0v = dhk = dhv = None
    if h0 is not None:
        h0k, h0v = (t.to(dev) for t in h0)
    if dhT is not None:
        dhk, dhv = (t.to(dev) for t in dhT)
    kr, vr, _, _ = gpu_recur(k, v, a, rope_base=rope_base, pos0=pos0, h0k=h0k, h0v=h0v,
                             reset_every=reset_every)
    dk, dv, da = torch.empty_like(k), torch.empty_like(v), torch.empty_like(a)
    dh0k = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    dh0v = torch.empty_like(dh0k)
    ws = rat.Workspace(rat.rat_recur_backward_workspace_bytes(B, H, T, d))
    rat.rat_recur_backward(k, v, a, kr, vr, dyk.to(dev), dyv.to(dev), dk, dv, da, ws,
                           h0_k=h0k, h0_v=h0v, dhT_k=dhk, dhT_v=dhv, dh0_k=dh0k, dh0_v=dh0v,
                           pos0=pos0, rope_base=rope_base, reset_every=reset_every)
    assert rat.rat_sync_status(ws) == 0
    return dk, dv, da, dh0k, dh0v


def check(x, dyk, dyv, h0=None, dhT=None, pos0=0, rope_base=0.0, heads=None, reset_every=0):
    got = gpu_backward(x, dyk, dyv, h0, dhT, pos0, rope_base, reset_every)
    B, H = x["k"].shape[:2]
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    bi, hi = [b for b, _ in sel], [h for _, h in sel]
    pick = lambda t: None if t is None else f64(t[bi, hi])
    ref = oracle.recurrence_layer_backward(
        pick(x["k"]), pick(x["v"]), pick(x["a"]), pick(dyk), pick(dyv),
        None if h0 is None else pick(h0[0]), None if h0 is None else pick(h0[1]),
        None if dhT is None else pick(dhT[0]), None if dhT is None else pick(dhT[1]),
        pos0=pos0, rope_base=rope_base, reset_every=reset_every)
    tol = tol_for(x["k"].dtype)
    names = ("dk", "dv", "da", "dh0k", "dh0v")
    errs = {n: rel_err(g[bi, hi], r) for n, g, r in zip(names, got, ref)}
    for n in names[:3]:
        assert errs[n] <= tol, errs
    # the initial-state gradients are float32 arithmetic on inputs the oracle sees exactly
    for n in names[3:]:
        assert errs[n] <= TOL_F32, errs
    return errs


def grads(B, H, T, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((B, H, T, d), generator=g).to(dtype),
            torch.randn((B, H, T, d), generator=g).to(dtype))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000])
def test_backward_ragged_lengths(dtype, d, T):
    x = inputs(2, 3, T, d, dtype, seed=T + d)
    dyk, dyv = grads(2, 3, T, d, dtype, seed=T)
    check(x, dyk, dyv)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("pos0", [0, 5000])
def test_backward_state_gradients_and_rope(dtype, pos0):
    x = inputs(2, 2, 333, 128, dtype, seed=pos0 + 3)
    dyk, dyv = grads(2, 2, 333, 128, dtype, seed=9)
    g = torch.Generator().manual_seed(11)
    h0 = (torch.randn((2, 2, 128), generator=g), torch.randn((2, 2, 128), generator=g))
    dhT = (torch.randn((2, 2, 128), generator=g), torch.randn((2, 2, 128), generator=g))
    check(x, dyk, dyv, h0=h0, dhT=dhT, pos0=pos0, rope_base=10000.0)


def test_backward_slow_gates():
    # gates near 1 carry the gradient far back (logits around 5: g ~ 0.993)
    x = inputs(1, 2, 1500, 128, torch.float32, seed=4, mu=5.0, sigma=0.5)
    dyk, dyv = grads(1, 2, 1500, 128, torch.float32, seed=5)
    check(x, dyk, dyv)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_zero_gate_passes_the_gradient_through(dtype):
    # g = 0 exactly: k~ = k, so dk = dk~ bit for bit and the gate gets no gradient
    x = inputs(1, 2, 300, 128, dtype, seed=12)
    x["a"] = torch.full_like(x["a"], -1.0e4)
    dyk, dyv = grads(1, 2, 300, 128, dtype, seed=13)
    dk, dv, da, dh0k, _ = gpu_backward(x, dyk, dyv)
    assert torch.equal(dk.cpu(), dyk) and torch.equal(dv.cpu(), dyv)
    assert torch.count_nonzero(da).item() == 0 and torch.count_nonzero(dh0k).item() == 0


def test_backward_full_size_sampled_heads():
    # the prefill_1p5b workload (B 4, H 16, T 4096, d 128, bf16, RoPE)
    w = synthetic.WORKLOADS["prefill_1p5b"]
    x = synthetic.prefill_inputs(w)
    dyk, dyv = grads(w.B, w.H, w.T, w.d, torch.bfloat16, seed=21)
    check(x, dyk, dyv, rope_base=w.rope_base, heads=[(0, 0), (w.B - 1, w.H - 1), (2, 5)])


# ---- the chunk-local form (rat_recur_backward_local): both recurrences cut at block starts
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("L", [1, 5, 16, 64, 100, 5000])
def test_local_backward_block_lengths(dtype, d, L):
    x = inputs(2, 2, 300, d, dtype, seed=L + d)
    dyk, dyv = grads(2, 2, 300, d, dtype, seed=L + 1)
    g = torch.Generator().manual_seed(L + 2)
    h0 = (torch.randn((2, 2, d), generator=g), torch.randn((2, 2, d), generator=g))
    dhT = (torch.randn((2, 2, d), generator=g), torch.randn((2, 2, d), generator=g))
    check(x, dyk, dyv, h0=h0, dhT=dhT, reset_every=L)


@pytest.mark.parametrize("pos0", [0, 3, 16, 1000])
def test_local_backward_offsets_and_rope(pos0):
    # block starts at absolute positions: row 0 starts a block when pos0 is a multiple of L (h0
    # then gets no gradient)
    x = inputs(1, 3, 257, 128, torch.bfloat16, seed=pos0 + 9)
    dyk, dyv = grads(1, 3, 257, 128, torch.bfloat16, seed=pos0 + 10)
    g = torch.Generator().manual_seed(pos0)
    h0 = (torch.randn((1, 3, 128), generator=g), torch.randn((1, 3, 128), generator=g))
    check(x, dyk, dyv, h0=h0, pos0=pos0, rope_base=10000.0, reset_every=16)


def test_local_backward_full_size_sampled_heads():
    # the prefill_1p5b workload with RAT's block length 16
    w = synthetic.WORKLOADS["prefill_1p5b"]
    x = synthetic.prefill_inputs(w)
    dyk, dyv = grads(w.B, w.H, w.T, w.d, torch.bfloat16, seed=19)
    check(x, dyk, dyv, rope_base=w.rope_base, heads=[(0, 0), (3, 15)], reset_every=16)


def test_backward_workspace_reused_across_calls():
    # one workspace, several calls of both forms and both dtypes: the look-back records carry a
    # per-launch tag, so no call reads another's records (every result matches the oracle)
    B, H, T, d = 1, 2, 700, 128
    for i, (dtype, L) in enumerate([(torch.bfloat16, 0), (torch.float32, 16), (torch.bfloat16, 5),
                                    (torch.float32, 0), (torch.bfloat16, 0)]):
        x = inputs(B, H, T, d, dtype, seed=40 + i)
        dyk, dyv = grads(B, H, T, d, dtype, seed=50 + i)
        check(x, dyk, dyv, rope_base=10000.0, reset_every=L)


def test_backward_lookback_timeout_is_reported():
    # failure detection: one chunk withholds its publication (test hook); the chunks before it
    # wait for it until their bound runs out, the workspace reports RAT_ERR_TIMEOUT, nothing hangs
    # and the next call on the same workspace is correct again
    L = rat.lib()
    B, H, T, d = 1, 2, 1024, 128
    x = inputs(B, H, T, d, torch.bfloat16, seed=31)
    dyk, dyv = grads(B, H, T, d, torch.bfloat16, seed=32)
    dev = torch.device("cuda")
    k, v, a = (x[n].to(dev) for n in ("k", "v", "a"))
    kr, vr, _, _ = gpu_recur(k, v, a)
    dk, dv, da = torch.empty_like(k), torch.empty_like(v), torch.empty_like(a)
    ws = rat.Workspace(rat.rat_recur_backward_workspace_bytes(B, H, T, d))
    L.rat_debug_inject_lookback_fault(5, 20_000_000)      # chunk 5, 20 ms waits, next call only
    rat.rat_recur_backward(k, v, a, kr, vr, dyk.to(dev), dyv.to(dev), dk, dv, da, ws)
    assert rat.rat_sync_status(ws) == -4
    rat.rat_recur_backward(k, v, a, kr, vr, dyk.to(dev), dyv.to(dev), dk, dv, da, ws)
    assert rat.rat_sync_status(ws) == 0
    ref = oracle.recurrence_layer_backward(f64(x["k"]), f64(x["v"]), f64(x["a"]), f64(dyk), f64(dyv),
                                           None, None, None, None)
    for g, r in zip((dk, dv, da), ref[:3]):
        assert rel_err(g, r) <= TOL_BF16
