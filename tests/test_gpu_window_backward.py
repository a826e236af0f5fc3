"""GPU parity of rat_recur_backward_window (gradients of the fixed-window recurrence step)
against the float64 oracle, which differentiates every output's restarted recurrence on its own."""
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import f64, rel_err, tol_for

pytestmark = pytest.mark.gpu


def inputs(B, H, T, d, dtype, seed=0):
    w = synthetic.Workload("wb", B=B, H=H, d=d, T=T, dtype="f32" if dtype == torch.float32 else "bf16",
                           gate_mu=2.0, gate_sigma=1.0, seed=seed)
    return synthetic.prefill_inputs(w)


def grads(B, H, T, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((B, H, T, d), generator=g).to(dtype),
            torch.randn((B, H, T, d), generator=g).to(dtype))


def gpu_window_backward(x, dyk, dyv, prev=None, want_dprev=False, pos0=0, rope_base=0.0):
    dev = torch.device("cuda")
    k, v, a = (x[n].to(dev) for n in ("k", "v", "a"))
    dk, dv, da = torch.empty_like(k), torch.empty_like(v), torch.empty_like(a)
    pk = pv = pa = dpk = dpv = dpa = None
    if prev is not None:
        pk, pv, pa = (t.to(dev) for t in prev)
        if want_dprev:
            dpk, dpv, dpa = (torch.full_like(pk, float("nan")) for _ in range(3))
    rat.rat_recur_backward_window(k, v, a, dyk.to(dev), dyv.to(dev), dk, dv, da, 64,
                                  prev_k=pk, prev_v=pv, prev_gate_logit=pa, dprev_k=dpk,
                                  dprev_v=dpv, dprev_gate_logit=dpa, pos0=pos0,
                                  rope_base=rope_base)
    torch.cuda.synchronize()
    return dk, dv, da, dpk, dpv, dpa


def check(x, dyk, dyv, prev=None, want_dprev=False, pos0=0, rope_base=0.0, heads=None):
    got = gpu_window_backward(x, dyk, dyv, prev, want_dprev, pos0, rope_base)
    B, H = x["k"].shape[:2]
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    bi, hi = [b for b, _ in sel], [h for _, h in sel]
    pick = lambda t: None if t is None else f64(t[bi, hi])
    ref = oracle.recurrence_window_layer_backward(
        pick(x["k"]), pick(x["v"]), pick(x["a"]), pick(dyk), pick(dyv), 64,
        *(pick(t) for t in (prev or (None, None, None))), pos0=pos0, rope_base=rope_base)
    tol = tol_for(x["k"].dtype)
    names = ("dk", "dv", "da", "dprev_k", "dprev_v", "dprev_a")
    n_out = 6 if want_dprev else 3
    errs = {n: rel_err(g[bi, hi], r) for n, g, r in list(zip(names, got, ref))[:n_out]}
    for n in names[:n_out]:
        assert errs[n] <= tol, errs
    return errs, got


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000, 2049])
def test_window_backward_ragged_lengths(dtype, d, T):
    # B 2 x H 4 x 33 blocks at T = 2049 gives more (slice, block) items than SMs: CTA ranges
    # span several blocks and cross (b, h) and slice boundaries
    x = inputs(2, 4, T, d, dtype, seed=T + 3 * d)
    dyk, dyv = grads(2, 4, T, d, dtype, seed=T + 1)
    check(x, dyk, dyv)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("want_dprev", [False, True])
@pytest.mark.parametrize("T,pos0", [(777, 5000), (40, 64), (2049, 0)])
def test_window_backward_history_rows_and_rope(dtype, want_dprev, T, pos0):
    # history rows before row 0; with their gradients (the oldest row, outside every window,
    # gets exactly 0); RoPE at positions below and above the float32-angle bound
    x = inputs(2, 3, T, 128, dtype, seed=17 + T)
    p = inputs(2, 3, 64, 128, dtype, seed=18 + T)
    prev = (p["k"], p["v"], p["a"])
    dyk, dyv = grads(2, 3, T, 128, dtype, seed=19 + T)
    _, got = check(x, dyk, dyv, prev=prev, want_dprev=want_dprev, pos0=pos0, rope_base=10000.0)
    if want_dprev:
        for t in got[3:]:
            assert torch.count_nonzero(t[:, :, 0]).item() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_window_backward_history_gradients_many_ranges(dtype, d):
    # B 3 x H 5 x (blocks -1 .. 20) x slices: more items than CTAs, so ranges start inside a
    # (b, h), on its history block and right after it; no RoPE, and RoPE at positions past the
    # float32-angle bound
    for pos0, base in ((0, 0.0), (9000, 10000.0)):
        x = inputs(3, 5, 1300, d, dtype, seed=40 + d + pos0)
        p = inputs(3, 5, 64, d, dtype, seed=41 + d + pos0)
        dyk, dyv = grads(3, 5, 1300, d, dtype, seed=42 + d + pos0)
        check(x, dyk, dyv, prev=(p["k"], p["v"], p["a"]), want_dprev=True, pos0=pos0,
              rope_base=base)


def test_window_backward_two_calls_equal_one():
    # a sequence cut in two, the second call given the last 64 rows of the first as history:
    # the second call's history gradients add to the first call's last 64 rows
    B, H, T, d, cut = 1, 3, 700, 128, 320
    x = inputs(B, H, T, d, torch.float32, seed=23)
    dyk, dyv = grads(B, H, T, d, torch.float32, seed=24)
    whole = gpu_window_backward(x, dyk, dyv, rope_base=10000.0)
    first = gpu_window_backward({n: t[:, :, :cut].contiguous() for n, t in x.items() if n in "kva"},
                                dyk[:, :, :cut].contiguous(), dyv[:, :, :cut].contiguous(),
                                rope_base=10000.0)
    prev = tuple(x[n][:, :, cut - 64:cut].contiguous() for n in ("k", "v", "a"))
    second = gpu_window_backward({n: t[:, :, cut:].contiguous() for n, t in x.items() if n in "kva"},
                                 dyk[:, :, cut:].contiguous(), dyv[:, :, cut:].contiguous(),
                                 prev=prev, want_dprev=True, pos0=cut, rope_base=10000.0)
    for i in range(3):
        joined = torch.cat([first[i], second[i]], 2).clone()
        joined[:, :, cut - 64:cut] += second[3 + i]
        assert rel_err(joined, whole[i]) <= 1e-5


def test_window_backward_short_sequence_is_the_full_backward():
    # T <= 64 without history: every window starts at row 0, so the window form's gradients are
    # the full-sequence backward's (h0 = 0, no final-state gradient)
    x = inputs(2, 2, 64, 128, torch.float32, seed=29)
    dyk, dyv = grads(2, 2, 64, 128, torch.float32, seed=30)
    dk, dv, da, _, _, _ = gpu_window_backward(x, dyk, dyv, rope_base=500.0)
    dev = torch.device("cuda")
    k, v, a = (x[n].to(dev) for n in ("k", "v", "a"))
    kr, vr = torch.empty_like(k), torch.empty_like(v)
    ws = rat.Workspace(rat.rat_recur_workspace_bytes(2, 2, 64, 128, 0))
    rat.rat_recur_prefill(k, v, a, kr, vr, ws, rope_base=500.0)
    fk, fv, fa = torch.empty_like(k), torch.empty_like(v), torch.empty_like(a)
    wsb = rat.Workspace(rat.rat_recur_backward_workspace_bytes(2, 2, 64, 128))
    rat.rat_recur_backward(k, v, a, kr, vr, dyk.to(dev), dyv.to(dev), fk, fv, fa, wsb,
                           rope_base=500.0)
    assert rat.rat_sync_status(wsb) == 0
    for mine, ref in ((dk, fk), (dv, fv), (da, fa)):
        assert rel_err(mine, ref) <= 1e-4


@pytest.mark.parametrize("name", ["prefill_1p5b", "window_2p6b"])
def test_window_backward_full_size_sampled_heads(name):
    # the whole workload runs on the GPU (bf16, RoPE); the oracle checks sampled heads
    w = synthetic.WORKLOADS[name]
    x = synthetic.prefill_inputs(w)
    dyk, dyv = grads(w.B, w.H, w.T, w.d, torch.bfloat16, seed=31)
    heads = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2)]
    check(x, dyk, dyv, rope_base=w.rope_base, heads=heads)
