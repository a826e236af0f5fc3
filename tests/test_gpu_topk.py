"""GPU parity of the top-k chunk selection combined with dilation (prefill) against the float64
oracle.  The selection is an integer decision on scores, so the test takes it in the kernel's
precision: the tensor-core path (bf16, d 128, no sinks) scores chunks with q^ rounded to bf16 (the
MMA operand), the CUDA-core path with q^ in float32 (within rounding of float64).  In a row whose
k-th and (k+1)-th chunk scores tie within rounding either choice is correct.  Every row is
compared element by element with the oracle's attention over its key set: S(t) plus the
selected chunks for a row with a clear choice, and for a tied row any of its admissible
selections (each chunk scoring clearly above the k-th is taken, the rest of the k are any of the
chunks that tie with the k-th)."""
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


def keys_with(t, D, W, n_sink, chunks):
    """S(t) and the positions of the given chunks below their chunk ends (the ends are keys
    already; positions below n_sink are sinks, listed already)."""
    base = [j for j in range(t + 1) if oracle.in_key_set(t, j, D, W, n_sink)]
    return base + [j for c in chunks for j in range(c * D, c * D + D - 1) if j >= n_sink]


def admissible_rows(qr_t, k, v, t, D, W, n_sink, scale, sel):
    """The oracle's output row for every admissible selection of a tied row."""
    sure, zone, need = sel
    combos = list(itertools.combinations(zone, need))
    assert len(combos) <= 512, (len(zone), need)
    return [oracle.attention_over_keys(qr_t, k, v, keys_with(t, D, W, n_sink, list(sure) + list(c)),
                                       scale) for c in combos]


def check_topk(x, D, W, n_sink, top_k, D_per_head=None, rope_base=10000.0, pos0=0, heads=None):
    """GPU top-k attention on x's q, k, v against the oracle on the heads given (all by default)."""
    q_, k_, v_ = x["q"], x["k"], x["v"]
    B, H, T, d = q_.shape
    dtype = q_.dtype
    tc_path = dtype == torch.bfloat16 and d == 128 and n_sink == 0 and T <= 65536
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in (q_, k_, v_))
    o = torch.empty_like(q)
    rat.rat_dilated_attn_prefill(q, k, v, o, D=D, W=W, D_per_head=D_per_head, n_sink=n_sink,
                                 top_k=top_k, rope_base=rope_base, pos0=pos0)
    assert rat.rat_attn_sync_status() == 0
    heads = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    scale = oracle.default_scale(d)
    tol = tol_for(dtype)
    og = f64(o)
    tied = 0
    for b, h in heads:
        Dh = D_per_head[h] if D_per_head is not None else D
        qr = f64(q_[b:b + 1, h:h + 1])
        if rope_base > 0:
            qr = oracle.rope(qr, pos0, rope_base)
        # the query the selection is taken with: as the kernel scores chunks
        qs = torch.from_numpy(qr).to(torch.bfloat16).double().numpy() if tc_path else qr
        kf, vf = f64(k_[b:b + 1, h:h + 1])[0, 0], f64(v_[b:b + 1, h:h + 1])[0, 0]
        if Dh == 1:       # a dense head: no chunks, top-k adds nothing
            ref = oracle.dilated_attention(qr, kf[None, None], vf[None, None], D=1, W=W)[0, 0]
            assert rel_err(og[b, h], ref) <= tol, (b, h)
            continue
        ref = np.empty((T, d))
        rows = []
        for t in range(T):
            sc = chunk_scores(qs[0, 0, t], kf, t, Dh, W, scale)
            sel = tie_zone(sc, top_k)
            if sel is None:
                best = sorted(range(len(sc)), key=lambda c: (-sc[c], c))[:top_k]
                ref[t] = oracle.attention_over_keys(qr[0, 0, t], kf, vf,
                                                    keys_with(t, Dh, W, n_sink, best), scale)
            else:
                tied += 1
                rows.append((t, admissible_rows(qr[0, 0, t], kf, vf, t, Dh, W, n_sink, scale, sel)))
                ref[t] = rows[-1][1][0]
        den = float(np.max(np.abs(ref)))
        for t, outs in rows:
            errs = [float(np.max(np.abs(og[b, h, t] - r))) / den for r in outs]
            assert min(errs) <= tol, (b, h, t, errs)
        clear = np.ones(T, dtype=bool)
        clear[[t for t, _ in rows]] = False
        assert rel_err(og[b, h][clear], ref[clear]) <= tol, (b, h)
    # near-ties are rare on random scores: a large count would point at the scores themselves
    assert tied <= 0.05 * len(heads) * T, tied


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D,W,n_sink,top_k", [(16, 0, 0, 4), (8, 16, 0, 8), (4, 4, 6, 16),
                                              (32, 1, 4, 1)])
def test_topk_attention(dtype, D, W, n_sink, top_k):
    B, H, T, d = 1, 2, 600, 128
    w = synthetic.Workload("tk", B=B, H=H, d=d, T=T, dtype="f32" if dtype == torch.float32 else "bf16",
                           seed=D + top_k)
    check_topk(synthetic.prefill_inputs(w), D, W, n_sink, top_k)


# bf16, d 128 without sinks: the tensor-core kernel (selection phase, then the selected chunks'
# key blocks beside the chunk-end and window blocks); chunks shorter, equal and longer than a
# 64-key block, several tiles with a ragged tail, top_k 1 .. 16, RoPE at an offset
@pytest.mark.parametrize("D,W,top_k", [(2, 0, 3), (16, 0, 16), (64, 64, 8), (100, 5, 2),
                                       (24, 130, 1), (5, 1, 7)])
@pytest.mark.parametrize("T", [333, 1000])
def test_topk_tensor_cores(D, W, top_k, T):
    w = synthetic.Workload("tkc", B=2, H=2, d=128, T=T, dtype="bf16", seed=D * 7 + top_k + T)
    check_topk(synthetic.prefill_inputs(w), D, W, 0, top_k, pos0=11)


def test_topk_tensor_cores_head_hybrid():
    # a dense head (no chunks: top-k adds nothing) beside three dilations in one launch
    w = synthetic.Workload("tkh", B=1, H=4, d=128, T=777, dtype="bf16", seed=55)
    check_topk(synthetic.prefill_inputs(w), 1, 16, 0, 4, D_per_head=[1, 8, 32, 64])


def test_topk_prefill_1p5b_sampled_heads():
    # the prefill_1p5b workload (B 4, H 16, T 4096, D 16, RoPE) with the top 8 chunks
    w = synthetic.WORKLOADS["prefill_1p5b"]
    x = synthetic.prefill_inputs(w)
    check_topk(x, w.D, w.W, 0, 8, rope_base=w.rope_base, heads=[(0, 0), (3, 15)])


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
