"""GPU parity of the top-k chunk selection combined with dilation (prefill) against the float64
oracle.  The selection is an integer decision taken on float32 scores by the kernel and on
float64 scores by the oracle: rows whose k-th and (k+1)-th chunk scores are within rounding of
each other may legitimately select differently, so those rows (rare, counted) are left out of
the element-wise comparison."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import f64, rel_err, tol_for

pytestmark = pytest.mark.gpu


def unambiguous_rows(qr, k, D, W, top_k, scale, margin=1e-3):
    """(T,) mask of query rows whose top-k chunk choice is separated by more than `margin`."""
    T = qr.shape[0]
    We = max(W, 1)
    ok = np.ones(T, dtype=bool)
    ends = k[D - 1::D]
    for t in range(T):
        nc = (t - We + 1) // D if t - We + 1 >= D else 0
        if nc <= top_k:
            continue
        sc = np.sort(scale * (ends[:nc] @ qr[t]))[::-1]
        if sc[top_k - 1] - sc[top_k] <= margin * (1.0 + abs(sc[top_k - 1])):
            ok[t] = False
    return ok


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D,W,n_sink,top_k", [(16, 0, 0, 4), (8, 16, 0, 8), (4, 4, 6, 16),
                                              (32, 1, 4, 1)])
def test_topk_attention(dtype, D, W, n_sink, top_k):
    B, H, T, d = 1, 2, 600, 128
    w = synthetic.Workload("tk", B=B, H=H, d=d, T=T, dtype="f32" if dtype == torch.float32 else "bf16",
                           seed=D + top_k)
    x = synthetic.prefill_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    rat.rat_dilated_attn_prefill(q, k, v, o, D=D, W=W, n_sink=n_sink, top_k=top_k,
                                 rope_base=10000.0)
    qr = oracle.rope(f64(x["q"]), 0, 10000.0)
    ref = oracle.topk_attention(qr, f64(x["k"]), f64(x["v"]), D=D, W=W, n_sink=n_sink, top_k=top_k)
    scale = oracle.default_scale(d)
    skipped = 0
    for h in range(H):
        rows = unambiguous_rows(qr[0, h], f64(x["k"])[0, h], D, W, top_k, scale)
        skipped += int((~rows).sum())
        assert rel_err(o[0, h][torch.from_numpy(rows).to(dev)], ref[0, h][rows]) <= tol_for(dtype)
    assert skipped <= 0.05 * H * T, skipped


def test_topk_zero_equals_plain_attention():
    w = synthetic.Workload("tk0", B=1, H=2, d=128, T=300, dtype="bf16", seed=3)
    x = synthetic.prefill_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    rat.rat_dilated_attn_prefill(q, k, v, o, D=8, W=0)
    ref = oracle.dilated_attention(f64(x["q"]), f64(x["k"]), f64(x["v"]), D=8, W=0)
    assert rel_err(o, ref) <= tol_for(torch.bfloat16)


def test_topk_above_16_is_refused():
    w = synthetic.Workload("tk17", B=1, H=1, d=128, T=64, dtype="bf16", seed=4)
    x = synthetic.prefill_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    with pytest.raises(rat.RatError) as e:
        rat.rat_dilated_attn_prefill(q, k, v, o, D=4, top_k=17)
    assert e.value.status == -2
