"""GPU parity of the paged compressed cache with per-sequence positions: rat_paged_kv_compress
(bit-exact layout through the page table) and rat_dilated_decode_paged (ragged positions, each
sequence against its own float64 decode oracle)."""
import numpy as np
import pytest
import torch

import oracle
import recurrence_augmented_dilated_b200 as rat
import synthetic
from gpu_util import TOL_BF16, TOL_F32, f64, gpu_recur, rel_err

pytestmark = pytest.mark.gpu


def page_table_for(B, H, max_pages, seed=0, spare=3):
    """Every (b, h) slice gets max_pages distinct pages of one pool, in a shuffled order (so the
    indirection is exercised); `spare` pages stay unused.  Returns (table, n_pages)."""
    n_pages = B * H * max_pages + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)[: B * H * max_pages]
    return perm.to(torch.int32).reshape(B, H, max_pages).contiguous(), n_pages


def gather_entries(pool, table, b, h, n, pe):
    """Dil entries 0 .. n-1 of slice (b, h), read through the page table on the host."""
    rows = [int(table[b, h, i // pe]) * pe + i % pe for i in range(n)]
    return pool.reshape(-1, pool.shape[-1])[rows]


def build(w, lengths, page_entries, max_pages, rope_base=0.0, reset_every=0, seed=0):
    """Prefill every sequence b (its own length) through the scan and the paged compress."""
    B, H, d, W = len(lengths), w.H, w.d, w.W
    Dh = w.heads_D()[:H]
    table, n_pages = page_table_for(B, H, max_pages, seed=seed)
    dev = torch.device("cuda")
    cache, bufs = rat.make_paged_cache(B, H, d, W, rat.BF16, Dh, page_entries, n_pages,
                                       table.to(dev), reset_every=reset_every)
    ws = rat.Workspace(256)
    ctx = []
    for b, T in enumerate(lengths):
        sl = [synthetic.decode_context_slice(w, b, h, device=dev, T=T) for h in range(H)]
        k, v, a = (torch.stack([x[i] for x in sl]).unsqueeze(0).contiguous() for i in range(3))
        kr, vr, hk, hv = gpu_recur(k, v, a, rope_base=rope_base, reset_every=reset_every)
        rat.rat_paged_kv_compress(kr, vr, hk, hv, b, 0, cache, ws)
        ctx.append((k, v, a, kr, vr, hk, hv))
    assert rat.rat_sync_status(ws) == 0
    return cache, bufs, table, ctx


@pytest.mark.parametrize("page_entries", [1, 4, 64])
def test_paged_compress_layout_bit_exact(page_entries):
    w = synthetic.Workload("paged", B=3, H=3, d=128, T=0, W=8, D_per_head=(1, 4, 16),
                           dtype="bf16", seed=50)
    lengths = [200, 37, 129]
    max_pages = (200 + page_entries - 1) // page_entries
    cache, bufs, table, ctx = build(w, lengths, page_entries, max_pages)
    assert bufs["pos"].cpu().tolist() == lengths
    Dh = w.heads_D()
    for b, T in enumerate(lengths):
        _, _, _, kr, vr, hk, hv = ctx[b]
        for h in range(w.H):
            D = Dh[h]
            n = T // D
            want_k = kr[0, h, D - 1::D][:n].cpu()
            want_v = vr[0, h, D - 1::D][:n].cpu()
            got_k = gather_entries(bufs["k_pool"].cpu(), table, b, h, n, page_entries)
            got_v = gather_entries(bufs["v_pool"].cpu(), table, b, h, n, page_entries)
            assert torch.equal(got_k, want_k) and torch.equal(got_v, want_v)
            for p in range(max(0, T - w.W), T):          # the ring holds the last W positions
                assert torch.equal(bufs["k_win"][b, h, p % w.W].cpu(), kr[0, h, p].cpu())
                assert torch.equal(bufs["v_win"][b, h, p % w.W].cpu(), vr[0, h, p].cpu())
        assert torch.equal(bufs["h_k"][b].cpu(), hk[0].cpu())
        assert torch.equal(bufs["h_v"][b].cpu(), hv[0].cpu())


def run_ragged(w, lengths, steps, page_entries, rope_base=0.0, reset_every=0, graph=False):
    B, H, d, W = len(lengths), w.H, w.d, w.W
    Dh = w.heads_D()[:H]
    cap = max((T + steps) // min(Dh) for T in lengths) + 1
    max_pages = (cap + page_entries - 1) // page_entries
    cache, bufs, table, ctx = build(w, lengths, page_entries, max_pages, rope_base=rope_base,
                                    reset_every=reset_every, seed=7)
    dev = torch.device("cuda")
    tok = synthetic.decode_steps(synthetic.Workload("tok", B=B, H=H, d=d, T=0, W=W,
                                                    D_per_head=tuple(Dh), dtype="bf16",
                                                    seed=w.seed + 1), steps)
    ws = rat.Workspace(rat.rat_paged_decode_workspace_bytes(cache))
    ins = {n: t.to(dev) for n, t in tok.items()}
    outs = torch.empty((steps, B, H, 1, d), dtype=torch.bfloat16, device=dev)

    def step(s):
        rat.rat_dilated_decode_paged(*(ins[n][s].reshape(B, H, 1, d) for n in ("q", "k", "v", "a")),
                                     cache, outs[s], ws, rope_base=rope_base)

    if graph:
        # inputs of every step are views of resident tensors, positions advance on the device:
        # one capture of all steps replays them with no host involvement
        st = torch.cuda.Stream()
        st.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(st):
            with torch.cuda.graph(g, stream=st):
                for s in range(steps):
                    step(s)
        torch.cuda.current_stream().wait_stream(st)
        g.replay()
    else:
        for s in range(steps):
            step(s)
    torch.cuda.synchronize()
    assert rat.rat_sync_status(ws) == 0
    assert bufs["pos"].cpu().tolist() == [T + steps for T in lengths]
    errs, herrs = [], []
    for b, T in enumerate(lengths):
        st_ = oracle.DecodeState(Dh, d, W, T + steps, rope_base=rope_base, reset_every=reset_every)
        k, v, a = ctx[b][:3]
        st_.prefill(f64(k[0]), f64(v[0]), f64(a[0]))
        for s in range(steps):
            ref = st_.step(*(f64(tok[n][s, b]) for n in ("q", "k", "v", "a")))
            errs.append(rel_err(outs[s, b, :, 0], ref))
        herrs.append(rel_err(bufs["h_k"][b], st_.hk))
    return max(errs), max(herrs)


@pytest.mark.parametrize("rope_base", [0.0, 10000.0])
def test_paged_decode_ragged_positions(rope_base):
    # three sequences at different positions; D = 16 entries are appended at different steps
    w = synthetic.Workload("ragged", B=3, H=3, d=128, T=0, W=8, D_per_head=(1, 4, 16),
                           dtype="bf16", seed=51)
    err, herr = run_ragged(w, [100, 37, 250], 40, page_entries=16, rope_base=rope_base)
    assert err <= TOL_BF16, err
    assert herr <= TOL_F32, herr


def test_paged_decode_graph_replay_and_local_recurrence():
    # positions advance on the device, so one captured graph of all steps is correct; the
    # chunk-local recurrence (L = 16) crosses block starts at different steps per sequence
    w = synthetic.Workload("ragged_g", B=4, H=2, d=128, T=0, W=0, D_per_head=(4, 64),
                           dtype="bf16", seed=52)
    err, herr = run_ragged(w, [300, 1, 64, 129], 24, page_entries=8, rope_base=10000.0,
                           reset_every=16, graph=True)
    assert err <= TOL_BF16, err
    assert herr <= TOL_F32, herr


def test_paged_decode_d64():
    w = synthetic.Workload("ragged64", B=2, H=2, d=64, T=0, W=4, D_per_head=(2, 8),
                           dtype="bf16", seed=53)
    err, herr = run_ragged(w, [77, 150], 20, page_entries=32)
    assert err <= TOL_BF16, err


def test_page_index_outside_the_pool_is_reported():
    # a table entry naming no page: the kernels' own bounds checks skip it and record
    # RAT_ERR_INVALID in the workspace header; nothing outside the pool is touched
    w = synthetic.Workload("badpage", B=1, H=1, d=128, T=0, W=0, D_per_head=(4,),
                           dtype="bf16", seed=54)
    table, n_pages = page_table_for(1, 1, 4, seed=1)
    table[0, 0, 1] = n_pages + 7
    dev = torch.device("cuda")
    cache, bufs = rat.make_paged_cache(1, 1, 128, 0, rat.BF16, [4], 4, n_pages, table.to(dev))
    sl = synthetic.decode_context_slice(w, 0, 0, device=dev, T=40)
    k, v, a = (sl[i][None, None].contiguous() for i in range(3))
    kr, vr, hk, hv = gpu_recur(k, v, a)
    ws = rat.Workspace(256)
    rat.rat_paged_kv_compress(kr, vr, hk, hv, 0, 0, cache, ws)
    assert rat.rat_sync_status(ws) == -1
    # the pages that exist hold their entries
    assert torch.equal(gather_entries(bufs["k_pool"].cpu(), table, 0, 0, 4, 4), kr[0, 0, 3:16:4].cpu())
