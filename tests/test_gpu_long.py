"""GPU parity at the size limits: sequences far beyond the workloads' (262,144 positions for the
recurrence forms, 131,072 for the attention, checked on sampled rows) and the largest head count
one call takes (256 heads with four different dilations)."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import TOL_BF16, TOL_F32, f64, gpu_attn, gpu_recur, rel_err

pytestmark = pytest.mark.gpu


def long_inputs(B, H, T, d, seed):
    w = synthetic.Workload("long", B=B, H=H, d=d, T=T, dtype="bf16", seed=seed)
    return synthetic.prefill_inputs(w)


def test_scan_and_window_over_262144_positions():
    T = 262144
    x = long_inputs(1, 1, T, 128, seed=60)
    kr, vr, hk, hv = gpu_recur(x["k"], x["v"], x["a"], rope_base=10000.0)
    yk, hk_ref = oracle.recurrence(f64(x["k"]), f64(x["a"]))
    yv, _ = oracle.recurrence(f64(x["v"]), f64(x["a"]))
    yk = oracle.rope(yk, 0, 10000.0)
    assert rel_err(kr, yk) <= TOL_BF16 and rel_err(vr, yv) <= TOL_BF16
    assert rel_err(hk, hk_ref) <= TOL_F32
    # the window form over the same rows (its oracle is O(T Lw); checked on the first 40,000)
    dev = torch.device("cuda")
    k, v, a = (x[n].to(dev) for n in ("k", "v", "a"))
    wk, wv = torch.empty_like(k), torch.empty_like(v)
    ws = rat.Workspace(256)
    rat.rat_recur_prefill_window(k, v, a, wk, wv, ws, 64)
    assert rat.rat_sync_status(ws) == 0
    n = 40000
    ref = oracle.recurrence_window(f64(x["k"][:, :, :n]), f64(x["a"][:, :, :n]), 64)
    assert rel_err(wk[:, :, :n], ref) <= TOL_BF16


def test_attention_over_131072_positions_sampled_rows():
    T = 131072
    x = long_inputs(1, 2, T, 128, seed=61)
    dev = torch.device("cuda")
    o = gpu_attn(x["q"], x["k"], x["v"], D_per_head=[64, 1024], W=128, rope_base=10000.0)
    rows = [0, 1, 127, 128, 4095, 65536, 100003, T - 1]
    qr = oracle.rope(f64(x["q"]), 0, 10000.0)
    ref = oracle.dilated_attention(qr, f64(x["k"]), f64(x["v"]), W=128, D_per_head=[64, 1024],
                                   rows=rows)
    assert rel_err(o[:, :, rows], ref) <= TOL_BF16


def test_256_heads_four_dilations():
    B, H, T, d = 1, 256, 384, 128
    x = long_inputs(B, H, T, d, seed=62)
    Dh = [[1, 4, 16, 64][h % 4] for h in range(H)]
    o = gpu_attn(x["q"], x["k"], x["v"], D_per_head=Dh, W=0)
    heads = [0, 1, 2, 3, 130, 255]
    ref = oracle.dilated_attention(f64(x["q"][:, heads]), f64(x["k"][:, heads]),
                                   f64(x["v"][:, heads]), W=0, D_per_head=[Dh[h] for h in heads])
    assert rel_err(o[:, heads], ref) <= TOL_BF16
