#!/usr/bin/env python3
"""Benchmark of the RAT+ dilated-inference hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload hybrid_7p6b] [--only] [--no-decode]

One step = one pass of the prefill path over one batch of the workload: the forget-gate
recurrence over k and v (rat_recur_prefill), dilated attention (rat_dilated_attn_prefill) and
the compressed-cache build (rat_kv_compress), on synthetic inputs already resident in HBM.
`value` is prefill tokens/s over all ranks on the headline workload (the largest one, the
7.6B-like hybrid head composition; B*T tokens per rank per step; weak scaling: every rank runs
its own batch, no data-path collective).  The `workloads` object holds every other workload,
each with its own kernels, roofline, clocks and CPU baseline: the 1.5B-like and 2.6B-like
prefill, the tiny float32 layer, and decode (256 one-token steps against the compressed
cache).  Each kernel's average duration is measured with CUDA events on its
own stream inside the timed region and turned into a roofline fraction with the algorithmic
bytes (or FLOPs) of one launch.

--impl reference times the float64 CPU oracle (the only other implementation of the method)
on a bounded sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synthetic  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# device-code headers every kernel file includes
KERNEL_HEADERS = ("common.cuh", "internal.h", "tc.cuh")


def headers_sha():
    h = hashlib.sha256()
    for n in KERNEL_HEADERS:
        with open(os.path.join(ROOT, "recurrence_augmented_dilated_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel is unchanged since: its
    source file's hash, and (for entries that record it) the shared headers' hash, must match."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        table = json.load(f)
    e = table.get(kernel_file, {}).get(workload)
    src = os.path.join(ROOT, "recurrence_augmented_dilated_b200", "csrc", kernel_file)
    if not e or not os.path.exists(src) or e.get("source_sha") != file_sha(src):
        return None
    if "headers_sha" in e and e["headers_sha"] != headers_sha():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if not self.path or not os.path.exists(self.path):
            return out
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if sm:
            out.update(sm_mhz=statistics.median(sm), sm_max_mhz=max(mx), samples=len(sm))
        out["reasons"] = sorted(reasons)
        return out


class EventTimer:
    """Per-kernel CUDA-event durations on one stream, accumulated over the timed steps."""

    def __init__(self, stream):
        self.stream = stream
        self.pairs = {}

    def span(self, name):
        timer = self

        class _S:
            def __enter__(self):
                self.a = torch.cuda.Event(enable_timing=True)
                self.b = torch.cuda.Event(enable_timing=True)
                self.a.record(timer.stream)

            def __exit__(self, *exc):
                self.b.record(timer.stream)
                timer.pairs.setdefault(name, []).append((self.a, self.b))
        return _S()

    def mean_ms(self):
        return {k: sum(a.elapsed_time(b) for a, b in v) / len(v) for k, v in self.pairs.items()}


# ----------------------------------------------------------------------------- distributed
def dist_setup(want_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


# ----------------------------------------------------------------------------- our arm
def algorithmic(w: synthetic.Workload, n_sink: int = 0, top_k: int = 0):
    """Algorithmic bytes / FLOPs of one launch of each kernel on workload w (with n_sink
    attention sinks and top_k selected chunks added to every key set)."""
    import recurrence_augmented_dilated_b200 as rat
    eb = 4 if w.dtype == "f32" else 2
    N = w.B * w.H * w.T * w.d
    We = max(w.W, 1)
    keys = 0
    for D in w.heads_D():
        # sum over queries of |S(t)| (closed form per t, summed in C by the library helper)
        keys += sum(rat.rat_attended_keys(t, D, w.W) for t in range(w.T))
        for t in range(w.T):
            lim = min(n_sink, max(0, t - We + 1))           # sinks older than the window
            keys += lim - lim // D if D > 1 else 0
            n_dil = (t - We + 1) // D if t - We + 1 >= D else 0
            if top_k and D > 1:
                # the positions of the selected chunks, less those that are sinks already
                # (counted at most: every selected chunk taken in full)
                keys += min(top_k, n_dil) * (D - 1)
    keys *= w.B
    cache_rows = sum(w.T // D for D in w.heads_D()) * w.B + w.B * w.H * min(w.W, w.T)
    return {
        "recur_bytes": 5 * N * eb,                      # read k, v, a; write k~, v~
        "attn_bytes": 4 * N * eb,                       # read q, k~, v~; write o
        "attn_flops": 4 * w.d * keys,                   # QK^T and PV over the attended keys only
        "attended_keys": keys,
        "compress_bytes": 2 * 2 * cache_rows * w.d * eb,  # k and v rows, read + write
    }


class ProfiledRegion:
    """cudaProfilerStart/Stop around a bench leg's warm-up and timed steps, so that
    `ncu --profile-from-start off` lists exactly those launches (no effect without a profiler)."""

    def __enter__(self):
        torch.cuda.synchronize()
        torch.cuda.profiler.start()
        return self

    def __exit__(self, *exc):
        torch.cuda.synchronize()
        torch.cuda.profiler.stop()
        return False


def run_prefill(w: synthetic.Workload, steps: int, warmup: int, rank: int, world: int, peaks,
                peak_kind, with_e2e: bool, min_warmup_s: float = 1.0, reset_every: int = 0,
                window: int = 0, n_sink: int = 0, top_k: int = 0):
    import recurrence_augmented_dilated_b200 as rat
    dev = torch.device("cuda")
    x = synthetic.prefill_inputs(w, seed=w.seed + 1000 * rank)
    q, k, v, a = (x[n].to(dev) for n in ("q", "k", "v", "a"))
    B, H, T, d = q.shape
    kr, vr, o = torch.empty_like(k), torch.empty_like(v), torch.empty_like(q)
    hk = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    hv = torch.empty_like(hk)
    dtc = rat.F32 if w.dtype == "f32" else rat.BF16
    cache, bufs = rat.make_cache(B, H, d, w.W, T, dtc, w.heads_D())
    ws = rat.Workspace(rat.rat_recur_workspace_bytes(B, H, T, d, dtc))
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream()          # the cache append runs beside the attention
    side_timer = EventTimer(side)
    Dph = list(w.D_per_head) if w.D_per_head else None

    def step(timer=None, qq=q, kk=k, vv=v, aa=a):
        span = timer.span if timer else (lambda n: _Null())
        sspan = side_timer.span if timer else (lambda n: _Null())
        with span("recur"):
            if window > 0:
                rat.rat_recur_prefill_window(kk, vv, aa, kr, vr, ws, window, rope_base=w.rope_base)
            elif reset_every > 0:
                rat.rat_recur_prefill_local(kk, vv, aa, kr, vr, ws, reset_every, hT_k=hk, hT_v=hv,
                                            rope_base=w.rope_base)
            else:
                rat.rat_recur_prefill(kk, vv, aa, kr, vr, ws, hT_k=hk, hT_v=hv,
                                      rope_base=w.rope_base)
        # the attention and the cache append both read only the recurrence outputs: the append
        # runs on a second stream while the attention runs, and the step ends when both have
        side.wait_stream(stream)
        cache.pos = 0
        with torch.cuda.stream(side):
            with sspan("compress"):
                rat.rat_kv_compress(kr, vr, hk, hv, cache, stream=side)
        with span("attn"):
            rat.rat_dilated_attn_prefill(qq, kr, vr, o, D=w.D, W=w.W, D_per_head=Dph,
                                         rope_base=w.rope_base, n_sink=n_sink, top_k=top_k)
        stream.wait_stream(side)

    timer = EventTimer(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # clocks are sampled from the start of the warm-up (at least ~1 s of it) through the timed
    # steps: a timed region of a few ms is shorter than the 200 ms sampling period
    with ClockSampler(torch.cuda.current_device()) as clk, ProfiledRegion():
        t_w = time.perf_counter()
        n_w = 0
        while n_w < warmup or time.perf_counter() - t_w < min_warmup_s:
            step()
            n_w += 1
            if n_w % 16 == 0:
                torch.cuda.synchronize()
        st = rat.rat_sync_status(ws)
        if st != 0:
            raise RuntimeError("device error " + rat.rat_status_string(st))
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            step(timer)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1) / steps
    ms_max = max_over_ranks(ms, world)
    kern = timer.mean_ms()
    span = side_timer.mean_ms()
    # the append's own duration: timed alone on the main stream after the step loop (beside the
    # attention its span also counts the time it waits for SM slots)
    # (back to back between two events: one launch between events would also count the host's
    # submission time of each call)
    n_solo = max(8, steps)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cache.pos = 0
    rat.rat_kv_compress(kr, vr, hk, hv, cache)
    c0.record(stream)
    for _ in range(n_solo):
        cache.pos = 0
        rat.rat_kv_compress(kr, vr, hk, hv, cache)
    c1.record(stream)
    torch.cuda.synchronize()
    kern["compress"] = c0.elapsed_time(c1) / n_solo
    st = rat.rat_sync_status(ws)
    if st != 0:
        raise RuntimeError("device error " + rat.rat_status_string(st))
    alg = algorithmic(w, n_sink, top_k)
    res = {
        "ms_per_step": ms_max,
        "tokens_per_s": world * B * T / (ms_max / 1e3),
        "kernels": {},
        "clocks": clk.summary(),
        "gpu_launches_per_step": 3,
    }
    hbm = peaks["hbm_gbs"]
    # a step of a few ms timed over tens of steps is a burst, not a seconds-long loop under the
    # power cap: the tensor-bound fraction is taken against the burst GEMM peak (the sustained
    # one is reported beside it)
    tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tc_sus = peaks.get("bf16_tflops_sustained", tc)
    step_kern = {n: t for n, t in kern.items() if n != "compress"}
    for name, t in kern.items():
        e = {"ms": t}
        if name in step_kern:
            e["share_of_kernel_time"] = t / sum(step_kern.values())
        if name == "recur":
            e.update(bound="hbm", achieved=alg["recur_bytes"] / (t * 1e-3) / 1e9, peak=hbm, unit="GB/s")
        elif name == "attn":
            gbs = alg["attn_bytes"] / (t * 1e-3) / 1e9
            tfs = alg["attn_flops"] / (t * 1e-3) / 1e12
            # below the ridge (FLOP/byte < peak ratio) attention is bound by HBM, above it by bf16 MMA
            ridge = tc * 1e12 / (hbm * 1e9)
            if alg["attn_flops"] / alg["attn_bytes"] < ridge or w.dtype == "f32":
                e.update(bound="hbm", achieved=gbs, peak=hbm, unit="GB/s", tflops=tfs)
            else:
                e.update(bound="tensor", achieved=tfs, peak=tc, unit="TFLOP/s", gbs=gbs,
                         peak_kind="burst", frac_of_sustained=tfs / tc_sus)
        elif name == "compress":
            # standalone duration; in the step it runs on a second stream beside the attention
            e.update(bound="hbm", achieved=alg["compress_bytes"] / (t * 1e-3) / 1e9, peak=hbm, unit="GB/s",
                     overlapped_with="attn", span_beside_attn_ms=span.get("compress"))
        e["frac"] = e["achieved"] / e["peak"]
        e["of"] = peak_kind
        res["kernels"][name] = e
    res["algorithmic"] = alg
    if with_e2e:
        o_ref = o.clone()
        res["e2e"] = run_e2e(w, steps, warmup, x, {"q": q, "k": k, "v": v, "a": a, "kr": kr, "vr": vr,
                                                  "o": o, "hk": hk, "hv": hv}, world)
        # the host-buffer path must reproduce the device path's output (up to the rounding order
        # of the scan's look-back)
        diff = (res["e2e"].pop("out").float() - o_ref.cpu().float()).abs().max().item()
        scale = o_ref.float().abs().max().item()
        if not diff <= 1e-2 * max(scale, 1e-30):
            raise RuntimeError("end-to-end output differs from the device path: %g" % diff)
    return res


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def e2e_chunks(B: int, H: int, min_chunks: int = 4):
    """(b, h0, h1) pieces of a (B, H, T, d) batch for the end-to-end pipeline: whole batch rows,
    or, when there are fewer rows than min_chunks, groups of heads of one row (each piece
    x[b:b+1, h0:h1] is one contiguous range)."""
    per_row = 1
    while B * per_row < min_chunks and per_row < H:
        per_row *= 2
    while H % per_row:
        per_row -= 1
    g = H // per_row
    return [(b, i * g, (i + 1) * g) for b in range(B) for i in range(per_row)]


def run_e2e(w, steps, warmup, x, dev, world):
    """The layer step through the public API from host buffers: for each piece of the batch (a
    batch row, or a group of heads of one row), the H2D copy of its q, k, v, a from pinned
    memory, the three calls, and the D2H copy of its output, on three streams (copy in, compute,
    copy out) so that one piece's copies overlap another piece's compute. Every copy of the step
    is inside the timed region."""
    import recurrence_augmented_dilated_b200 as rat
    names = ("q", "k", "v", "a")
    host = {n: x[n].pin_memory() for n in names}
    o, kr, vr, hk, hv = dev["o"], dev["kr"], dev["vr"], dev["hk"], dev["hv"]
    out_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    B, H, T, d = o.shape
    dtc = rat.F32 if w.dtype == "f32" else rat.BF16
    Dh = w.heads_D()
    pieces = e2e_chunks(B, H)
    P = len(pieces)
    # one cache and one scan workspace per piece (calls on one piece never overlap themselves)
    caches = [rat.make_cache(1, h1 - h0, d, w.W, T, dtc, Dh[h0:h1]) for (_, h0, h1) in pieces]
    ws = [rat.Workspace(rat.rat_recur_workspace_bytes(1, h1 - h0, T, d, dtc)) for (_, h0, h1) in pieces]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(P)]
    ev_comp = [torch.cuda.Event() for _ in range(P)]
    ev_out = [torch.cuda.Event() for _ in range(P)]

    def e2e_step():
        for i, (b, h0, h1) in enumerate(pieces):
            r = (slice(b, b + 1), slice(h0, h1))
            Dph = Dh[h0:h1] if w.D_per_head else None
            s_in.wait_event(ev_comp[i])          # the previous step's piece i no longer needs its inputs
            with torch.cuda.stream(s_in):
                for n in names:
                    dev[n][r].copy_(host[n][r], non_blocking=True)
                ev_in[i].record(s_in)
            s_comp.wait_event(ev_in[i])
            s_comp.wait_event(ev_out[i])         # the previous step's piece i output has been read
            with torch.cuda.stream(s_comp):
                rat.rat_recur_prefill(dev["k"][r], dev["v"][r], dev["a"][r], kr[r], vr[r], ws[i],
                                      hT_k=hk[r], hT_v=hv[r], rope_base=w.rope_base)
                rat.rat_dilated_attn_prefill(dev["q"][r], kr[r], vr[r], o[r], D=w.D, W=w.W,
                                             D_per_head=Dph, rope_base=w.rope_base)
                cache = caches[i][0]
                cache.pos = 0
                rat.rat_kv_compress(kr[r], vr[r], hk[r], hv[r], cache)
                ev_comp[i].record(s_comp)
            s_out.wait_event(ev_comp[i])
            with torch.cuda.stream(s_out):
                out_host[r].copy_(o[r], non_blocking=True)
                ev_out[i].record(s_out)

    cur = torch.cuda.current_stream()
    for _ in range(max(1, warmup)):
        e2e_step()
    torch.cuda.synchronize()
    for i in range(P):
        if rat.rat_sync_status(ws[i]) != 0:
            raise RuntimeError("device error in the end-to-end leg")
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for s_ in (s_in, s_comp, s_out):
        s_.wait_event(e0)
    for _ in range(steps):
        e2e_step()
    done = torch.cuda.Event()
    done.record(s_out)
    cur.wait_event(done)
    e1.record(cur)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()
    return {"value": world * w.B * w.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "method": "%d pieces (batch row x head group): H2D, recurrence + attention + compress, "
                      "D2H on three streams" % P,
            "out": out_host}


def run_decode(w: synthetic.Workload, steps_timed: int, warmup: int, rank: int, world: int, peaks,
               peak_kind, window_rec: int = 0):
    """Decode workload: context prefill + compress (untimed), then w.steps one-token steps per
    timed repetition, captured in one CUDA graph and replayed.  window_rec = 64: the
    fixed-window recurrence (context by rat_recur_prefill_window with each chunk's history rows,
    rat_kv_compress_window; every step reruns the recurrence over the raw ring)."""
    import recurrence_augmented_dilated_b200 as rat
    dev = torch.device("cuda")
    B, H, d, W, T0 = w.B, w.H, w.d, w.W, w.T
    nsteps = w.steps
    Tcap = T0 + nsteps
    cache, bufs = rat.make_cache(B, H, d, W, Tcap, rat.BF16, w.heads_D(), window_rec=window_rec)
    hk = torch.zeros((B, H, d), dtype=torch.float32, device=dev)
    hv = torch.zeros_like(hk)
    nchunks = (T0 + synthetic.CTX_CHUNK - 1) // synthetic.CTX_CHUNK
    ws_r = rat.Workspace(rat.rat_recur_workspace_bytes(B, H, synthetic.CTX_CHUNK, d, rat.BF16))
    hist = {}
    for c in range(nchunks):
        k, v, a = synthetic.decode_context_block(w, c, device=dev, T=T0)
        kr, vr = torch.empty_like(k), torch.empty_like(v)
        if window_rec:
            rat.rat_recur_prefill_window(k, v, a, kr, vr, ws_r, window_rec, pos0=cache.pos,
                                         rope_base=w.rope_base, **hist)
            rat.rat_kv_compress_window(kr, vr, k, v, a, cache)
            hist = {n: x[:, :, -window_rec:].contiguous()
                    for n, x in (("prev_k", k), ("prev_v", v), ("prev_gate_logit", a))}
        else:
            hk2, hv2 = torch.empty_like(hk), torch.empty_like(hv)
            rat.rat_recur_prefill(k, v, a, kr, vr, ws_r, h0_k=hk, h0_v=hv, hT_k=hk2, hT_v=hv2,
                                  pos0=cache.pos, rope_base=w.rope_base)
            rat.rat_kv_compress(kr, vr, hk2, hv2, cache)
            hk, hv = hk2, hv2
        del k, v, a, kr, vr
    del hist
    del ws_r
    torch.cuda.synchronize()
    torch.cuda.empty_cache()      # only the cache and the step inputs stay on the device
    tok = synthetic.decode_steps(w)
    tq, tk, tv, ta = (tok[n].to(dev).reshape(nsteps, B, H, 1, d) for n in ("q", "k", "v", "a"))
    out = torch.empty((nsteps, B, H, 1, d), dtype=torch.bfloat16, device=dev)
    ws = rat.Workspace(rat.rat_decode_workspace_bytes(cache))
    # snapshot of the mutable cache state (state and ring), restored before every repetition
    snap = {n: bufs[n].clone() for n in ("h_k", "h_v", "k_win", "v_win") +
            (("k_raw", "v_raw", "a_raw") if window_rec else ())}
    pos_ctx = cache.pos

    def reset():
        for n in snap:
            bufs[n].copy_(snap[n])
        cache.pos = pos_ctx

    def all_steps():
        for s in range(nsteps):
            rat.rat_dilated_decode(tq[s], tk[s], tv[s], ta[s], cache, out[s], ws, rope_base=w.rope_base)

    # capture the 256 launches once (positions baked into the graph), replay per repetition
    reset()
    torch.cuda.synchronize()
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s_cap):
        with torch.cuda.graph(g, stream=s_cap):
            all_steps()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    prof = ProfiledRegion().__enter__()
    for _ in range(warmup):
        reset()
        g.replay()
    torch.cuda.synchronize()
    st = rat.rat_sync_status(ws)
    if st != 0:
        prof.__exit__()
        raise RuntimeError("decode device error " + rat.rat_status_string(st))
    times = []
    barrier(world)
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(steps_timed):
            reset()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
    prof.__exit__()
    ms_total = max_over_ranks(sum(times) / len(times), world)
    ms_step = ms_total / nsteps
    # algorithmic bytes per step: K and V rows of every attended cache entry + the ring window
    # (window form: + the raw k, v, a rows of the 63 positions before the token)
    eb = 2
    rows = 0
    for D in w.heads_D():
        for s in range(nsteps):
            t = T0 + s
            rows += rat.rat_attended_keys(t, D, W) - 1      # the token itself comes from registers
    rows = rows * B / nsteps
    step_bytes = 2 * rows * d * eb
    if window_rec:
        step_bytes += 3 * (window_rec - 1) * B * H * d * eb
    achieved = step_bytes / (ms_step * 1e-3) / 1e9
    return {
        "workload": w.name + ("_window%d" % window_rec if window_rec else ""),
        "metric": "decode tokens/s", "unit": "tokens/s",
        "value": world * B * nsteps / (ms_total / 1e3), "ms_per_token_step": ms_step,
        "steps_per_repetition": nsteps, "repetitions": steps_timed, "cuda_graph": True,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "of": peak_kind,
                     "traffic": recorded_traffic("decode.cu", w.name + ("_window%d" % window_rec
                                                                          if window_rec else ""))},
        "clocks": clk.summary(),
        "gpu_launches": nsteps * steps_timed,
    }


def run_decode_paged(w: synthetic.Workload, steps_timed: int, warmup: int, rank: int, world: int,
                     peaks, peak_kind, page_entries: int = 64):
    """Ragged decode: the sequences of the batch hold different context lengths
    (synthetic.ragged_lengths), in a paged compressed cache; every sequence decodes w.steps
    tokens at its own position.  The steps of a repetition replay as one CUDA graph (positions
    advance on the device)."""
    import recurrence_augmented_dilated_b200 as rat
    dev = torch.device("cuda")
    B, H, d, W = w.B, w.H, w.d, w.W
    nsteps = w.steps
    lengths = synthetic.ragged_lengths(w)
    Dh = w.heads_D()
    cap = (max(lengths) + nsteps) // min(Dh) + 1
    max_pages = (cap + page_entries - 1) // page_entries
    n_pages = B * H * max_pages
    g = torch.Generator().manual_seed(w.seed)
    table = torch.randperm(n_pages, generator=g).to(torch.int32).reshape(B, H, max_pages)
    cache, bufs = rat.make_paged_cache(B, H, d, W, rat.BF16, Dh, page_entries, n_pages,
                                       table.contiguous().to(dev))
    ws_c = rat.Workspace(256)
    ws_r = rat.Workspace(rat.rat_recur_workspace_bytes(1, H, synthetic.CTX_CHUNK, d, rat.BF16))
    for b, T in enumerate(lengths):
        hk = torch.zeros((1, H, d), dtype=torch.float32, device=dev)
        hv = torch.zeros_like(hk)
        for c in range((T + synthetic.CTX_CHUNK - 1) // synthetic.CTX_CHUNK):
            kva = torch.stack([synthetic.decode_context_chunk(w, b, h, c, dev, T) for h in range(H)], 1)
            k, v, a = (kva[i].unsqueeze(0).contiguous() for i in range(3))
            kr, vr = torch.empty_like(k), torch.empty_like(v)
            hk2, hv2 = torch.empty_like(hk), torch.empty_like(hv)
            pos0 = c * synthetic.CTX_CHUNK
            rat.rat_recur_prefill(k, v, a, kr, vr, ws_r, h0_k=hk, h0_v=hv, hT_k=hk2, hT_v=hv2,
                                  pos0=pos0, rope_base=w.rope_base)
            rat.rat_paged_kv_compress(kr, vr, hk2, hv2, b, pos0, cache, ws_c)
            hk, hv = hk2, hv2
    if rat.rat_sync_status(ws_c) != 0:
        raise RuntimeError("paged compress reported an error")
    del ws_r
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    tok = synthetic.decode_steps(w)
    tq, tk, tv, ta = (tok[n].to(dev).reshape(nsteps, B, H, 1, d) for n in ("q", "k", "v", "a"))
    out = torch.empty((nsteps, B, H, 1, d), dtype=torch.bfloat16, device=dev)
    ws = rat.Workspace(rat.rat_paged_decode_workspace_bytes(cache))
    snap = {n: bufs[n].clone() for n in ("h_k", "h_v", "k_win", "v_win", "pos")}

    def reset():
        for n in snap:
            bufs[n].copy_(snap[n])

    reset()
    torch.cuda.synchronize()
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s_cap):
        with torch.cuda.graph(gr, stream=s_cap):
            for s in range(nsteps):
                rat.rat_dilated_decode_paged(tq[s], tk[s], tv[s], ta[s], cache, out[s], ws,
                                             rope_base=w.rope_base)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    prof = ProfiledRegion().__enter__()
    for _ in range(warmup):
        reset()
        gr.replay()
    torch.cuda.synchronize()
    st = rat.rat_sync_status(ws)
    if st != 0:
        prof.__exit__()
        raise RuntimeError("paged decode device error " + rat.rat_status_string(st))
    if bufs["pos"].cpu().tolist() != [T + nsteps for T in lengths]:
        raise RuntimeError("paged decode positions did not advance")
    times = []
    barrier(world)
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(steps_timed):
            reset()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            gr.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
    prof.__exit__()
    ms_total = max_over_ranks(sum(times) / len(times), world)
    ms_step = ms_total / nsteps
    rows = 0
    for T in lengths:
        for D in Dh:
            for s in range(nsteps):
                rows += rat.rat_attended_keys(T + s, D, W) - 1
    step_bytes = 2 * (rows / nsteps) * d * 2
    achieved = step_bytes / (ms_step * 1e-3) / 1e9
    return {
        "workload": w.name + "_ragged_paged", "metric": "decode tokens/s", "unit": "tokens/s",
        "value": world * B * nsteps / (ms_total / 1e3), "ms_per_token_step": ms_step,
        "context_lengths": [min(lengths), max(lengths)], "page_entries": page_entries,
        "steps_per_repetition": nsteps, "repetitions": steps_timed, "cuda_graph": True,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "of": peak_kind,
                     "traffic": recorded_traffic("decode.cu", w.name + "_ragged_paged")},
        "clocks": clk.summary(),
        "gpu_launches": nsteps * steps_timed,
    }


def run_backward(w: synthetic.Workload, steps: int, warmup: int, world: int, peaks, peak_kind,
                 reset_every: int = 0, window: int = 0):
    """Backward of the recurrence step on the prefill workload: the forward outputs and
    upstream gradients are resident; each timed step is one rat_recur_backward call
    (rat_recur_backward_local with reset_every = L > 0, rat_recur_backward_window with
    window = 64, which reads the forward inputs only)."""
    import recurrence_augmented_dilated_b200 as rat
    dev = torch.device("cuda")
    x = synthetic.prefill_inputs(w)
    k, v, a = (x[n].to(dev) for n in ("k", "v", "a"))
    B, H, T, d = k.shape
    dtc = rat.F32 if w.dtype == "f32" else rat.BF16
    kr, vr = torch.empty_like(k), torch.empty_like(v)
    ws_f = rat.Workspace(rat.rat_recur_workspace_bytes(B, H, T, d, dtc))
    if window:
        rat.rat_recur_prefill_window(k, v, a, kr, vr, ws_f, window, rope_base=w.rope_base)
    elif reset_every > 0:
        rat.rat_recur_prefill_local(k, v, a, kr, vr, ws_f, reset_every, rope_base=w.rope_base)
    else:
        rat.rat_recur_prefill(k, v, a, kr, vr, ws_f, rope_base=w.rope_base)
    g = torch.Generator(device=dev).manual_seed(w.seed + 77)
    dyk = torch.randn(k.shape, generator=g, device=dev).to(k.dtype)
    dyv = torch.randn(k.shape, generator=g, device=dev).to(k.dtype)
    dk, dv, da = torch.empty_like(k), torch.empty_like(v), torch.empty_like(a)
    ws = rat.Workspace(rat.rat_recur_backward_workspace_bytes(B, H, T, d))
    stream = torch.cuda.current_stream()

    def step():
        if window:
            rat.rat_recur_backward_window(k, v, a, dyk, dyv, dk, dv, da, window,
                                          rope_base=w.rope_base)
        else:
            rat.rat_recur_backward(k, v, a, kr, vr, dyk, dyv, dk, dv, da, ws,
                                   rope_base=w.rope_base, reset_every=reset_every)

    with ProfiledRegion():
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
    if rat.rat_sync_status(ws) != 0:
        raise RuntimeError("backward device error")
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk, ProfiledRegion():
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    eb = 2 if w.dtype == "bf16" else 4
    # read k, v, a, k~, v~ (not the window form), dk~, dv~; write dk, dv, da
    nbytes = (8 if window else 10) * B * H * T * d * eb
    achieved = nbytes / (ms * 1e-3) / 1e9
    res = {"workload": w.name, "ms": ms,
           "step": ("rat_recur_backward_window(Lw=%d) (1 launch: blocks of Lw rows, no waits)" % window
                    if window else
                    ("rat_recur_backward_local(L=%d)" % reset_every if reset_every else
                     "rat_recur_backward") + " (1 launch: scan from the end, decoupled look-back)"),
           "tokens_per_s": world * B * T / (ms * 1e-3),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "of": peak_kind,
                        "algorithmic_bytes": nbytes},
           "clocks": clk.summary(), "gpu_launches": steps}
    # attention backward on the same shapes: q, k~, v~, o, dO resident
    q = x["q"].to(dev)
    o = torch.empty_like(q)
    Dph = list(w.D_per_head) if w.D_per_head else None
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)    # saved by the forward
    rat.rat_dilated_attn_prefill(q, kr, vr, o, D=w.D, W=w.W, D_per_head=Dph, rope_base=w.rope_base,
                                 lse=lse)
    dO = torch.randn(q.shape, generator=g, device=dev).to(q.dtype)
    dq, dkr, dvr = torch.empty_like(q), torch.empty_like(kr), torch.empty_like(vr)
    ws_a = rat.Workspace(rat.rat_dilated_attn_backward_workspace_bytes(B, H, T, d, dtc))

    def astep():
        rat.rat_dilated_attn_backward(q, kr, vr, o, dO, dq, dkr, dvr, ws_a, D=w.D, W=w.W,
                                      D_per_head=Dph, rope_base=w.rope_base, lse=lse)

    with ProfiledRegion():
        for _ in range(warmup):
            astep()
        torch.cuda.synchronize()
    barrier(world)
    with ProfiledRegion():
        e0.record(stream)
        for _ in range(steps):
            astep()
        e1.record(stream)
        torch.cuda.synchronize()
    ams = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    abytes = 8 * B * H * T * d * eb        # read q, k~, v~, o, dO; write dq, dk~, dv~
    pairs = sum(rat.rat_attended_keys(t, D_, w.W) for D_ in w.heads_D() for t in range(T)) * B
    aflops = 10 * d * pairs                 # per pair: recomputed score, dp, dq, dk, dv
    a_ach = abytes / (ams * 1e-3) / 1e9
    tc_path = w.dtype == "bf16" and w.d == 128
    res["attention"] = {"step": "rat_dilated_attn_backward (%s, the forward's log-sum-exp given)" % (
                            "prep on CUDA cores, dq and dk/dv launches on tcgen05 tensor cores"
                            if tc_path else "3 CUDA-core launches"), "ms": ams,
                        "roofline": {"bound": "hbm", "achieved": a_ach, "peak": peaks["hbm_gbs"],
                                     "unit": "GB/s", "frac": a_ach / peaks["hbm_gbs"],
                                     "of": peak_kind, "algorithmic_bytes": abytes,
                                     "tflops": aflops / (ams * 1e-3) / 1e12},
                        "gpu_launches": 3 * steps}
    return res


# ----------------------------------------------------------------------------- oracle (CPU)
def oracle_sample(w: synthetic.Workload, budget_s: float = 12.0):
    """Time the float64 oracle on whole (b, h) slices of w (recurrence + RoPE + attention over
    every query row, or over evenly spaced rows when a slice does not fit the budget).  Heads
    are sampled per dilation class (a hybrid's dense and dilated heads cost very different
    amounts), each class's time scaled by its own slice count; returns (tokens/s scaled to the
    whole workload, threads, description, seconds spent)."""
    import numpy as np
    import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    Dh = w.heads_D()
    x = synthetic.prefill_inputs(w)
    classes = {}
    for i in range(w.B * w.H):
        classes.setdefault(Dh[i % w.H], []).append(i)
    budget_c = budget_s / len(classes)

    def run(slices, rows, threads):
        b_idx = [i // w.H for i in slices]
        h_idx = [i % w.H for i in slices]
        sl = {n: x[n][b_idx, h_idx].unsqueeze(0).double().numpy() for n in ("q", "k", "v", "a")}
        oracle.set_threads(threads)
        t0 = time.perf_counter()
        oracle.layer_prefill(sl["q"], sl["k"], sl["v"], sl["a"], D_per_head=[Dh[h] for h in h_idx],
                             W=w.W, rope_base=w.rope_base, rows=rows)
        return time.perf_counter() - t0

    total_s, spent, used, descs = 0.0, 0.0, 1, []
    for D, members in sorted(classes.items()):
        nsl = len(members)
        # probe one wave of slices in parallel at 32 and 96 rows: time = fixed (the recurrence
        # over all T) + per row
        nprobe = max(1, min(cores, nsl, 8))
        wave = members[:nprobe]
        t32 = run(wave, np.linspace(0, w.T - 1, 32).astype(np.int64), nprobe)
        t96 = run(wave, np.linspace(0, w.T - 1, 96).astype(np.int64), nprobe)
        per_row = max(t96 - t32, 1e-9) / 64
        fixed = max(t32 - 32 * per_row, 0.0)
        wave_full = fixed + per_row * w.T        # one wave of nprobe slices, all rows
        waves = budget_c / max(wave_full, 1e-9)
        rows = None
        if waves >= 1:
            nslices = min(nsl, max(nprobe, int(waves) * nprobe))
        else:
            nslices = nprobe
            n = int((budget_c - fixed) / per_row) if budget_c > fixed else 32
            rows = np.linspace(0, w.T - 1, min(w.T, max(32, n))).astype(np.int64)
        threads = max(1, min(cores, nslices))
        used = max(used, threads)
        slices = members[:nslices]
        # a sample shorter than the budget (the whole class, when it fits) is repeated until
        # about half the budget has been spent, and timed as the mean
        reps, el = 0, 0.0
        while reps == 0 or (el < 0.5 * budget_c and reps < 100):
            el += run(slices, rows, threads)
            reps += 1
        spent += el + t32 + t96
        frac_rows = 1.0 if rows is None else len(rows) / w.T
        total_s += el / reps / frac_rows * nsl / nslices
        descs.append("D=%d: %d of %d (b,h) slices, %s query rows, %d threads, mean of %d runs" % (
            D, nslices, nsl, "all" if rows is None else "%d of %d" % (len(rows), w.T), threads, reps))
    desc = "float64 oracle (recurrence + RoPE + attention); " + "; ".join(descs) + (
        "; each dilation class scaled by its slice count" if len(classes) > 1 else "")
    return w.B * w.T / total_s, used, desc, spent


def oracle_decode_sample(w: synthetic.Workload, budget_s: float = 6.0, nslices: int = 8):
    """Time the float64 decode oracle (state update, RoPE, attention over the whole history) on
    nslices (b, h) slices of the decode workload: their contexts are consumed untimed, then
    decode steps run until about the budget is spent; the per-step time is scaled to all
    B*H slices.  Returns (tokens/s, threads, description, seconds)."""
    import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    Dh = w.heads_D()
    BH = w.B * w.H
    picks = [(i * BH // nslices) for i in range(nslices)]
    bh = [(i // w.H, i % w.H) for i in picks]
    st = oracle.DecodeState([Dh[h] for _, h in bh], w.d, w.W, w.T + w.steps, rope_base=w.rope_base)
    ctx = [synthetic.decode_context_slice(w, b, h) for b, h in bh]
    st.prefill(*(torch.stack([c[i] for c in ctx]).double().numpy() for i in range(3)))
    del ctx
    tok = synthetic.decode_steps(w)
    b_idx = [b for b, _ in bh]
    h_idx = [h for _, h in bh]
    tq, tk, tv, ta = (tok[n][:, b_idx, h_idx].double().numpy() for n in ("q", "k", "v", "a"))
    threads = max(1, min(cores, nslices))
    oracle.set_threads(threads)
    n, el = 0, 0.0
    while n < w.steps and (n < 8 or el < budget_s):
        t0 = time.perf_counter()
        st.step(tq[n], tk[n], tv[n], ta[n])
        el += time.perf_counter() - t0
        n += 1
    step_full = el / n * BH / nslices
    desc = ("float64 decode oracle on %d of %d (b,h) slices (full history kept), %d of %d steps "
            "after the %d-position context, %d threads; scaled to all slices" % (
                nslices, BH, n, w.steps, w.T, threads))
    return w.B / step_full, threads, desc, el


# ----------------------------------------------------------------------------- main
OTHER_PREFILL = ("prefill_1p5b", "window_2p6b", "tiny_fp32")


def dominant_roofline(kern, peak_kind):
    """The roofline object of the step's dominant kernel (the cache append overlaps the
    attention and is left out)."""
    name = max((n for n in kern if not kern[n].get("overlapped_with")), key=lambda n: kern[n]["ms"])
    k = kern[name]
    roof = {"bound": k["bound"], "achieved": k["achieved"], "peak": k["peak"], "unit": k["unit"],
            "frac": k["frac"], "of": peak_kind, "kernel": name, "traffic": k.get("traffic")}
    if "peak_kind" in k:
        roof["peak_kind"] = k["peak_kind"]
        roof["frac_of_sustained"] = k["frac_of_sustained"]
    return roof


def attach_traffic(kern, w, variant="", window=0, n_sink=0, top_k=0):
    src_of = {"recur": "window.cu" if window else "scan.cu",
              "attn": "attn_simt.cu" if (top_k or (n_sink and w.dtype == "f32")) else "attn_sm100.cu",
              "compress": "compress.cu"}
    attn_variant = ("_top%d" % top_k if top_k else "") + ("_sinks%d" % n_sink if n_sink else "")
    for n in kern:      # DRAM bytes per launch from the committed ncu capture (null if stale)
        kern[n]["traffic"] = recorded_traffic(
            src_of[n], w.name + (variant if n == "recur" else attn_variant if n == "attn" else ""))


def workload_config(w):
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "D": w.D, "W": w.W,
            "D_per_head": list(w.D_per_head) if w.D_per_head else None,
            "rope_base": w.rope_base, "gates": [w.gate_mu, w.gate_sigma], "dtype": w.dtype}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="hybrid_7p6b",
                    help="the headline prefill workload (top-level value and roofline)")
    ap.add_argument("--only", action="store_true",
                    help="time the headline workload alone (no other workloads, no decode)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--all", action="store_true", help="(default) kept for older command lines")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--reset-every", type=int, default=0,
                    help="L > 0: the chunk-local recurrence (restart every L positions) in the "
                         "prefill step instead of the full-sequence one")
    ap.add_argument("--decode-paged", action="store_true",
                    help="also time ragged decode (context lengths T/2 .. T) on a paged cache")
    ap.add_argument("--backward", action="store_true",
                    help="also time the backward of the recurrence step on the workload (of the "
                         "chunk-local form with --reset-every, of the window form with "
                         "--window 64) and of the attention")
    ap.add_argument("--sinks", type=int, default=0,
                    help="n > 0: the first n positions join every key set (attention sinks)")
    ap.add_argument("--top-k", type=int, default=0,
                    help="k > 0: the k best chunks (by chunk-end score) are attended in full")
    ap.add_argument("--window", type=int, default=0,
                    help="Lw > 0: the fixed-window recurrence (each state over the last Lw "
                         "positions) in the prefill step")
    ap.add_argument("--min-warmup-s", type=float, default=1.0,
                    help="keep warming up at least this long (clock sampling); 0 under a profiler")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    variant_leg = bool(args.reset_every or args.window or args.sinks or args.top_k)

    w = synthetic.WORKLOADS[args.workload]
    metric = "RAT+ layer prefill tokens/s and decode tokens/s at 1 B200; % HBM / tensor roofline"
    peaks, peak_kind = load_peaks()

    if args.impl == "reference":
        # the CPU oracle runs on rank 0 only; other ranks exit at once without joining a group
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        per = []
        desc = cores = None
        for _ in range(max(1, args.steps)):
            v, cores, desc, el = oracle_sample(w, budget_s=max(2.0, 60.0 / max(args.steps, 1)))
            per.append(v)
        value = statistics.median(per)
        line = {"impl": "reference", "metric": metric, "value": value, "unit": "tokens/s",
                "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": w.B * w.T / value * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": workload_config(w),
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                 "sample": desc},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if not torch.cuda.is_available():
        print(json.dumps({"metric": metric, "error": "no CUDA device"}))
        return 1
    rank, world, local = dist_setup(args.gpus)
    import recurrence_augmented_dilated_b200 as rat
    rat.lib()       # fail loudly if the library is missing
    cpu_here = rank == 0 and world == 1 and not args.no_cpu_baseline

    pre = run_prefill(w, args.steps, args.warmup, rank, world, peaks, peak_kind,
                      with_e2e=(not args.no_e2e and not variant_leg),
                      min_warmup_s=args.min_warmup_s, reset_every=args.reset_every,
                      window=args.window, n_sink=args.sinks, top_k=args.top_k)
    kern = pre["kernels"]
    variant = ("_L%d" % args.reset_every if args.reset_every else
               "_window%d" % args.window if args.window else "")
    attach_traffic(kern, w, variant, args.window, args.sinks, args.top_k)
    cfg = workload_config(w)
    cfg.update({
        "step": "%s + %s + rat_kv_compress (on a second stream, beside the attention)" % (
            "rat_recur_prefill_window(Lw=%d)" % args.window if args.window else
            "rat_recur_prefill_local(L=%d)" % args.reset_every if args.reset_every else
            "rat_recur_prefill",
            "rat_dilated_attn_prefill_topk(n_sink=%d, top_k=%d)" % (args.sinks, args.top_k)
            if args.top_k else
            "rat_dilated_attn_prefill_sinks(n_sink=%d)" % args.sinks if args.sinks else
            "rat_dilated_attn_prefill"),
        "l2": "inputs larger than L2 (q, k, v, a = %d MB per rank)" % (
            4 * w.B * w.H * w.T * w.d * (2 if w.dtype == "bf16" else 4) // 2**20),
        "parallelism": "replicas: dp%d over (batch) with no collective" % world})
    line = {
        "metric": metric, "value": pre["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": pre["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": cfg,
        "roofline": dominant_roofline(kern, peak_kind),
        "kernels": kern,
        "clocks": pre["clocks"],
        "e2e": pre.get("e2e"),
        "gpu_launches": pre["gpu_launches_per_step"] * args.steps,
    }
    if cpu_here:
        v, cores, desc, el = oracle_sample(w)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": el}

    # every other workload, each with its own kernels, roofline, clocks and CPU baseline
    others = {}
    if not args.only and not variant_leg:
        for name in OTHER_PREFILL:
            if name == w.name:
                continue
            ow = synthetic.WORKLOADS[name]
            r = run_prefill(ow, args.steps, args.warmup, rank, world, peaks, peak_kind,
                            with_e2e=False, min_warmup_s=args.min_warmup_s)
            attach_traffic(r["kernels"], ow)
            sub = {"metric": "prefill tokens/s", "value": r["tokens_per_s"], "unit": "tokens/s",
                   "ms_per_step": r["ms_per_step"], "config": workload_config(ow),
                   "roofline": dominant_roofline(r["kernels"], peak_kind),
                   "kernels": r["kernels"], "clocks": r["clocks"],
                   "gpu_launches": r["gpu_launches_per_step"] * args.steps}
            if cpu_here:
                v, cores, desc, el = oracle_sample(ow, budget_s=6.0)
                sub["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores,
                                       "kind": "oracle", "sample": desc, "seconds": el}
            others[name] = sub
    if not args.no_decode and not args.only:
        dw = synthetic.WORKLOADS["decode_7p6b"]
        dec = run_decode(dw, max(1, min(args.steps, 10)), 3, rank, world, peaks, peak_kind,
                         window_rec=args.window if args.window == 64 else 0)
        if cpu_here:
            v, cores, desc, el = oracle_decode_sample(dw)
            dec["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                   "sample": desc, "seconds": el}
        others["decode_7p6b"] = dec
    if others:
        line["workloads"] = others
    if args.backward:
        line["backward"] = run_backward(w, args.steps, args.warmup, world, peaks, peak_kind,
                                        reset_every=args.reset_every,
                                        window=args.window if args.window == 64 else 0)
    if args.decode_paged:
        dw = synthetic.WORKLOADS["decode_7p6b"]
        line["decode_paged"] = run_decode_paged(dw, max(1, min(args.steps, 10)), 3, rank, world,
                                                peaks, peak_kind)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
