"""GPU parity of rat_recur_prefill (chunked associative scan) against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import TOL_BF16, TOL_F32, f64, gpu_recur, rel_err, tol_for

pytestmark = pytest.mark.gpu


def check(k, v, a, rope_base=0.0, pos0=0, heads=None, h0=None, reset_every=0):
    """GPU vs oracle on all (b, h) or on `heads` (list of (b, h))."""
    h0k = h0v = None
    if h0 is not None:
        h0k, h0v = (x.cuda() for x in h0)
    kr, vr, hTk, hTv = gpu_recur(k, v, a, rope_base=rope_base, pos0=pos0, h0k=h0k, h0v=h0v,
                                 reset_every=reset_every)
    sel = heads if heads is not None else [(b, h) for b in range(k.shape[0]) for h in range(k.shape[1])]
    bi = [b for b, _ in sel]
    hi = [h for _, h in sel]
    ok_, ov_ = f64(k[bi, hi]), f64(v[bi, hi])
    oa_ = f64(a[bi, hi])
    o_h0k = f64(h0[0][bi, hi]) if h0 is not None else None
    o_h0v = f64(h0[1][bi, hi]) if h0 is not None else None
    yk, hk = oracle.recurrence(ok_, oa_, o_h0k, pos0=pos0, reset_every=reset_every)
    yv, hv = oracle.recurrence(ov_, oa_, o_h0v, pos0=pos0, reset_every=reset_every)
    if rope_base > 0:
        yk = oracle.rope(yk, pos0, rope_base)
    tol = tol_for(k.dtype)
    errs = dict(k=rel_err(kr[bi, hi], yk), v=rel_err(vr[bi, hi], yv), hk=rel_err(hTk[bi, hi], hk),
                hv=rel_err(hTv[bi, hi], hv))
    # the float32 state is exact up to float32 rounding even on the bf16 path
    assert errs["hk"] <= TOL_F32, errs
    assert errs["hv"] <= TOL_F32, errs
    assert errs["k"] <= tol and errs["v"] <= tol, errs
    return errs


def inputs(B, H, T, d, dtype, mu=2.0, sigma=1.0, seed=0):
    w = synthetic.Workload("t", B=B, H=H, d=d, T=T, dtype="f32" if dtype == torch.float32 else "bf16",
                           gate_mu=mu, gate_sigma=sigma, seed=seed)
    return synthetic.prefill_inputs(w)


# bf16 d128 full-sequence scans with T a multiple of 16 run in 64-channel slices with 128-row
# chunks; these lengths end in partial chunks (and, for the last (b, h), a box past the tensor)
@pytest.mark.parametrize("T", [16, 48, 208, 1008, 4096 + 16])
def test_sliced_scan_partial_chunks(T):
    x = inputs(2, 3, T, 128, torch.bfloat16, seed=T + 7)
    g = torch.Generator().manual_seed(T)
    h0 = (torch.randn((2, 3, 128), generator=g), torch.randn((2, 3, 128), generator=g))
    check(x["k"], x["v"], x["a"], rope_base=10000.0, pos0=37, h0=h0)


def test_tiny_fp32_workload():
    w = synthetic.WORKLOADS["tiny_fp32"]
    x = synthetic.prefill_inputs(w)
    check(x["k"], x["v"], x["a"])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 64, 129, 1000, 2049])
def test_ragged_lengths(dtype, d, T):
    x = inputs(2, 3, T, d, dtype, seed=T + d)
    check(x["k"], x["v"], x["a"])


@pytest.mark.parametrize("pos0", [0, 5000, 70000])
def test_rope_positions(pos0):
    x = inputs(1, 2, 777, 128, torch.bfloat16, seed=pos0 + 1)
    check(x["k"], x["v"], x["a"], rope_base=10000.0, pos0=pos0)


def test_rope_fp32_precision():
    x = inputs(1, 2, 300, 64, torch.float32, seed=9)
    check(x["k"], x["v"], x["a"], rope_base=10000.0, pos0=123456)


def test_initial_state_and_chunked_prefill():
    x = inputs(2, 2, 500, 128, torch.float32, seed=3)
    g = torch.Generator().manual_seed(5)
    h0 = (torch.randn((2, 2, 128), generator=g), torch.randn((2, 2, 128), generator=g))
    check(x["k"], x["v"], x["a"], h0=h0)
    # two GPU calls chained through hT equal one call
    k, v, a = (t.cuda() for t in (x["k"], x["v"], x["a"]))
    kr, vr, hk, hv = gpu_recur(k, v, a)
    kr1, vr1, hk1, hv1 = gpu_recur(k[:, :, :200].contiguous(), v[:, :, :200].contiguous(), a[:, :, :200].contiguous())
    kr2, vr2, hk2, hv2 = gpu_recur(k[:, :, 200:].contiguous(), v[:, :, 200:].contiguous(), a[:, :, 200:].contiguous(),
                                   h0k=hk1, h0v=hv1)
    assert rel_err(torch.cat([kr1, kr2], 2), kr) <= 1e-5
    assert rel_err(hk2, hk) <= 1e-5 and rel_err(hv2, hv) <= 1e-5


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_zero_gate_is_identity_exactly(dtype):
    # logit -1e4: g = 0 and 1-g = 1 exactly, so k~ = k and v~ = v bit for bit
    x = inputs(1, 2, 300, 128, dtype, seed=11)
    a = torch.full_like(x["a"], -1.0e4)
    kr, vr, _, _ = gpu_recur(x["k"], x["v"], a)
    assert torch.equal(kr.cpu(), x["k"]) and torch.equal(vr.cpu(), x["v"])


def test_unit_gate_holds_initial_state():
    x = inputs(1, 1, 200, 64, torch.float32, seed=12)
    a = torch.full_like(x["a"], 1.0e4)
    h0k = torch.randn((1, 1, 64)).cuda()
    h0v = torch.randn((1, 1, 64)).cuda()
    kr, vr, hk, hv = gpu_recur(x["k"], x["v"], a, h0k=h0k, h0v=h0v)
    assert torch.equal(kr[0, 0], h0k[0, 0].expand(200, 64))
    assert torch.equal(hv, h0v)


@pytest.mark.parametrize("T", [1500, 1536])
def test_repeated_launches_reuse_workspace(T):
    # the launch epoch lets one workspace serve many calls without clearing: every call matches
    # the oracle (a stale look-back record would corrupt whole chunks).  Calls agree with each
    # other to rounding, not bit for bit: the look-back may group the predecessors differently.
    # T 1500 runs the full-row scan, T 1536 the channel-sliced one.
    x = inputs(2, 4, T, 128, torch.bfloat16, seed=21)
    ws = rat.Workspace(rat.rat_recur_workspace_bytes(2, 4, T, 128, 1))
    yk, hk = oracle.recurrence(f64(x["k"]), f64(x["a"]), None)
    for _ in range(6):
        kr, _, hTk, _ = gpu_recur(x["k"], x["v"], x["a"], ws=ws)
        assert rel_err(kr, yk) <= TOL_BF16
        assert rel_err(hTk, hk) <= TOL_F32


@pytest.mark.parametrize("name", ["prefill_1p5b", "window_2p6b", "hybrid_7p6b"])
def test_full_size_workloads_sampled_heads(name):
    w = synthetic.WORKLOADS[name]
    x = synthetic.prefill_inputs(w)
    heads = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2)]
    check(x["k"], x["v"], x["a"], rope_base=w.rope_base, heads=heads)


def test_lookback_timeout_is_reported():
    # failure detection: one chunk withholds its publication (test hook); its successors' bounded
    # waits run out, the device error word reads RAT_ERR_TIMEOUT, and the context stays usable.
    L = rat.lib()
    x = inputs(1, 1, 1024, 128, torch.bfloat16, seed=30)
    L.rat_debug_inject_lookback_fault(2, 20_000_000)      # chunk 2, 20 ms waits, next call only
    k, v, a = (t.cuda() for t in (x["k"], x["v"], x["a"]))
    ws = rat.Workspace(rat.rat_recur_workspace_bytes(1, 1, 1024, 128, 1))
    kr, vr = torch.empty_like(k), torch.empty_like(v)
    rat.rat_recur_prefill(k, v, a, kr, vr, ws)
    assert rat.rat_sync_status(ws) == -4
    # the next call (no fault armed) is correct again
    check(x["k"], x["v"], x["a"])


# ---- chunk-local recurrence (RAT: the state restarts every L positions)
# The scan's chunk holds 32 (float32, d 128), 64 (float32 d 64, bf16 d 128) or 128 (bf16 d 64)
# rows, split into segments of 4 or 8 rows per lane; L is chosen below, equal to and above those
# sizes, as a divisor and a non-divisor of them, and beyond the sequence.
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("L", [1, 3, 8, 16, 37, 64, 128, 200, 5000])
def test_local_recurrence(dtype, d, L):
    x = inputs(2, 2, 1100, d, dtype, seed=L + d)
    check(x["k"], x["v"], x["a"], reset_every=L)


@pytest.mark.parametrize("pos0", [5, 63, 64, 1000003])
def test_local_recurrence_offsets_and_initial_state(pos0):
    # blocks are aligned to absolute positions; h0 reaches only the rows before the first start
    x = inputs(2, 2, 700, 128, torch.float32, seed=pos0 % 97)
    g = torch.Generator().manual_seed(pos0 % 89)
    h0 = (torch.randn((2, 2, 128), generator=g), torch.randn((2, 2, 128), generator=g))
    for L in (16, 64, 100):
        check(x["k"], x["v"], x["a"], pos0=pos0, h0=h0, reset_every=L, rope_base=10000.0)


def test_local_recurrence_chained_equals_whole():
    # float32 outputs: the two forms differ only in float32 rounding order, which can flip a
    # bf16 rounding
    x = inputs(1, 3, 900, 128, torch.float32, seed=77)
    k, v, a = (t.cuda() for t in (x["k"], x["v"], x["a"]))
    L = 48
    kr, vr, hk, hv = gpu_recur(k, v, a, reset_every=L)
    cut = 301
    parts = [slice(0, cut), slice(cut, 900)]
    kr1, vr1, hk1, hv1 = gpu_recur(*(t[:, :, parts[0]].contiguous() for t in (k, v, a)), reset_every=L)
    kr2, vr2, hk2, hv2 = gpu_recur(*(t[:, :, parts[1]].contiguous() for t in (k, v, a)), reset_every=L,
                                   pos0=cut, h0k=hk1, h0v=hv1)
    assert rel_err(torch.cat([kr1, kr2], 2), kr) <= 1e-5
    assert rel_err(torch.cat([vr1, vr2], 2), vr) <= 1e-5
    assert rel_err(hk2, hk) <= 1e-5 and rel_err(hv2, hv) <= 1e-5


def test_local_recurrence_block_one_is_the_input_term():
    # L = 1: every row starts a block, so k~_t = (1 - g_t) k_t exactly as the kernel rounds it
    # (one float32 product of the gate complement and the input)
    x = inputs(1, 2, 257, 64, torch.float32, seed=5)
    kr, vr, hk, _ = gpu_recur(x["k"], x["v"], x["a"], reset_every=1)
    ref = oracle.recurrence(f64(x["k"]), f64(x["a"]), reset_every=1)[0]
    assert rel_err(kr, ref) <= TOL_F32
    assert rel_err(hk, ref[..., -1, :]) <= TOL_F32


def test_local_recurrence_full_size_sampled_heads():
    # the prefill_1p5b workload (B 4, H 16, T 4096, d 128, bf16, RoPE) with RAT's chunk size 16
    w = synthetic.WORKLOADS["prefill_1p5b"]
    x = synthetic.prefill_inputs(w)
    heads = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2)]
    check(x["k"], x["v"], x["a"], rope_base=w.rope_base, heads=heads, reset_every=16)


# ---- fixed-window recurrence (each state covers the last 64 positions)
def gpu_window(k, v, a, prev=None, pos0=0, rope_base=0.0):
    dev = torch.device("cuda")
    k, v, a = (x.to(dev) for x in (k, v, a))
    kr, vr = torch.empty_like(k), torch.empty_like(v)
    ws = rat.Workspace(256)
    pk = pv = pa = None
    if prev is not None:
        pk, pv, pa = (x.to(dev) for x in prev)
    rat.rat_recur_prefill_window(k, v, a, kr, vr, ws, 64, prev_k=pk, prev_v=pv,
                                 prev_gate_logit=pa, pos0=pos0, rope_base=rope_base)
    st = rat.rat_sync_status(ws)
    assert st == 0, rat.rat_status_string(st)
    return kr, vr


def check_window(k, v, a, prev=None, pos0=0, rope_base=0.0, heads=None):
    kr, vr = gpu_window(k, v, a, prev=prev, pos0=pos0, rope_base=rope_base)
    sel = heads if heads is not None else [(b, h) for b in range(k.shape[0]) for h in range(k.shape[1])]
    bi = [b for b, _ in sel]
    hi = [h for _, h in sel]
    px = pv = pa = None
    if prev is not None:
        px, pv, pa = (f64(x[bi, hi]) for x in prev)
    oa = f64(a[bi, hi])
    yk = oracle.recurrence_window(f64(k[bi, hi]), oa, 64, prev_x=px, prev_a=pa)
    yv = oracle.recurrence_window(f64(v[bi, hi]), oa, 64, prev_x=pv, prev_a=pa)
    if rope_base > 0:
        yk = oracle.rope(yk, pos0, rope_base)
    tol = tol_for(k.dtype)
    errs = dict(k=rel_err(kr[bi, hi], yk), v=rel_err(vr[bi, hi], yv))
    assert errs["k"] <= tol and errs["v"] <= tol, errs
    return errs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000, 2049])
def test_window_recurrence(dtype, d, T):
    # B 2 x H 4 x 33 blocks at T = 2049 is more blocks than SMs: CTA ranges span several blocks
    # and cross (b, h) boundaries
    x = inputs(2, 4, T, d, dtype, seed=T + 3 * d)
    check_window(x["k"], x["v"], x["a"])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_window_history_rows_and_rope(dtype):
    x = inputs(2, 3, 777, 128, dtype, seed=17)
    p = inputs(2, 3, 64, 128, dtype, seed=18)
    prev = (p["k"], p["v"], p["a"])
    check_window(x["k"], x["v"], x["a"], prev=prev, pos0=5000, rope_base=10000.0)


def test_window_continues_a_sequence():
    # two calls, the second given the last 64 rows of the first as history, equal one call
    x = inputs(1, 2, 640, 128, torch.float32, seed=23)
    k, v, a = (t.cuda() for t in (x["k"], x["v"], x["a"]))
    kr, vr = gpu_window(k, v, a)
    cut = 320
    kr1, vr1 = gpu_window(*(t[:, :, :cut].contiguous() for t in (k, v, a)))
    prev = tuple(t[:, :, cut - 64:cut].contiguous() for t in (k, v, a))
    kr2, vr2 = gpu_window(*(t[:, :, cut:].contiguous() for t in (k, v, a)), prev=prev)
    assert rel_err(torch.cat([kr1, kr2], 2), kr) <= 1e-5
    assert rel_err(torch.cat([vr1, vr2], 2), vr) <= 1e-5


def test_window_short_sequence_is_the_full_recurrence():
    # T <= 64 without history: no position ever leaves the window
    x = inputs(2, 2, 64, 128, torch.float32, seed=29)
    kr, vr = gpu_window(x["k"], x["v"], x["a"])
    kf, vf, _, _ = gpu_recur(x["k"], x["v"], x["a"])
    assert rel_err(kr, kf) <= 1e-5 and rel_err(vr, vf) <= 1e-5


def test_window_full_size_sampled_heads():
    # the prefill_1p5b workload (B 4, H 16, T 4096, d 128, bf16, RoPE)
    w = synthetic.WORKLOADS["prefill_1p5b"]
    x = synthetic.prefill_inputs(w)
    heads = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2), (1, 7)]
    check_window(x["k"], x["v"], x["a"], rope_base=w.rope_base, heads=heads)
