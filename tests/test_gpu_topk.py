"""GPU parity of the top-k chunk selection combined with dilation (prefill) against the float64
oracle.  The selection is an integer decision taken on float32 scores by the kernel and on
float64 scores by the oracle: in a row whose k-th and (k+1)-th chunk scores tie within rounding
either choice is correct.  Rows with a clear choice are compared with the oracle element by
element; every other row must match the oracle's attention over one of its admissible
selections (each chunk scoring clearly above the k-th is taken, the rest of the k are any of
the chunks that tie with the k-th)."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import f64, rel_err, tol_for

pytestmark = pytest.mark.gpu

MARGIN = 1e-3       # score gap (relative to 1 + |s_k|) beyond float32 rounding of a 128-term dot


def chunk_scores(qr_t, k, t, D, W, scale):
    We = max(W, 1)
    nc = (t - We + 1) // D if t - We + 1 >= D else 0
    return scale * (k[D - 1::D][:nc] @ qr_t)


def tie_zone(sc, top_k):
    """(sure, zone, need): the chunks clearly above the k-th score, the chunks within MARGIN of
    it, and how many of the zone a correct selection takes; None when the choice is clear."""
    nc = len(sc)
    if nc <= top_k:
        return None
    order = np.sort(sc)[::-1]
    sk = order[top_k - 1]
    m = MARGIN * (1.0 + abs(sk))
    if sk - order[top_k] > m:
        return None
    sure = [c for c in range(nc) if sc[c] > sk + m]
    zone = [c for c in range(nc) if abs(sc[c] - sk) <= m]
    return sure, zone, top_k - len(sure)


def admissible_rows(qr_t, k, v, t, D, W, n_sink, scale, sel):
    """The oracle's output row for every admissible selection of a tied row."""
    sure, zone, need = sel
    base = [j for j in range(t + 1) if oracle.in_key_set(t, j, D, W, n_sink)]
    combos = list(itertools.combinations(zone, need))
    assert len(combos) <= 512, (len(zone), need)
    outs = []
    for combo in combos:
        # a selected chunk adds its positions below the chunk end (the end is a dilated key
        # already; positions below n_sink are sinks, listed already)
        extra = [j for c in list(sure) + list(combo) for j in range(c * D, c * D + D - 1)
                 if j >= n_sink]
        outs.append(oracle.attention_over_keys(qr_t, k, v, base + extra, scale))
    return outs


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
    kf, vf = f64(x["k"]), f64(x["v"])
    ref = oracle.topk_attention(qr, kf, vf, D=D, W=W, n_sink=n_sink, top_k=top_k)
    scale = oracle.default_scale(d)
    tol = tol_for(dtype)
    og = f64(o)
    tied = 0
    for h in range(H):
        den = float(np.max(np.abs(ref[0, h])))
        clear = np.ones(T, dtype=bool)
        for t in range(T):
            sel = tie_zone(chunk_scores(qr[0, h, t], kf[0, h], t, D, W, scale), top_k)
            if sel is None:
                continue
            clear[t] = False
            tied += 1
            errs = [float(np.max(np.abs(og[0, h, t] - r))) / den
                    for r in admissible_rows(qr[0, h, t], kf[0, h], vf[0, h], t, D, W, n_sink,
                                             scale, sel)]
            assert min(errs) <= tol, (h, t, errs)
        assert rel_err(o[0, h][torch.from_numpy(clear).to(dev)], ref[0, h][clear]) <= tol
    # near-ties are rare on random scores: a large count would point at the scores themselves
    assert tied <= 0.05 * H * T, tied


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
