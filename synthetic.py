"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module holds no arithmetic of the method: it only draws normal random numbers with a
seeded torch generator and casts them to the run's dtype.  Both the CUDA library's callers and
the float64 oracle take their inputs from here.

Workloads (shapes of the pages' 1.5B / 2.6B / 7.6B-model layers; the pages evaluate on
FineWeb-Edu, LongBench, commonsense and NIAH suites, which these random tensors stand in for):

  tiny_fp32      B1  H2  d64  T256    D4          W0    fp32  gates N(2,1)
  prefill_1p5b   B4  H16 d128 T4096   D16         W0    bf16  gates N(2,1)   RoPE base 10000
  window_2p6b    B2  H20 d128 T16384  D64         W128  bf16  gates N(3,1)
  hybrid_7p6b    B1  H32 d128 T32768  D1 x8, D64 x24  W64  bf16  gates N(2,1.5)
  decode_7p6b    B32 H32 d128 context 65536, D64 W128, 256 one-token steps, gates N(2,1)

Recipe (prefill): one CPU ``torch.Generator`` seeded with the workload's seed draws float32
standard normals in the order q, k, v, a (a = mu + sigma * N(0,1)), each (B, H, T, d); the
results are then cast to the dtype.  Decode: the context k, v, a of slice (b, h) come from a
generator seeded with (seed, b, h, chunk) on the requested device, 8192 positions per chunk,
so one slice (or one chunk of all slices) can be regenerated alone; the per-step tokens come from one CPU generator, drawn as q, k, v, a of shape
(steps, B, H, d).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    T: int
    D: int = 1
    W: int = 0
    D_per_head: Optional[tuple] = None
    dtype: str = "bf16"
    gate_mu: float = 2.0
    gate_sigma: float = 1.0
    rope_base: float = 0.0
    seed: int = 0
    steps: int = 0          # decode steps (decode workloads only)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def heads_D(self) -> List[int]:
        if self.D_per_head is not None:
            return list(self.D_per_head)
        return [self.D] * self.H


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, H=2, d=64, T=256, D=4, W=0, dtype="f32",
                          gate_mu=2.0, gate_sigma=1.0, seed=0),
    "prefill_1p5b": Workload("prefill_1p5b", B=4, H=16, d=128, T=4096, D=16, W=0, dtype="bf16",
                             gate_mu=2.0, gate_sigma=1.0, rope_base=10000.0, seed=1),
    "window_2p6b": Workload("window_2p6b", B=2, H=20, d=128, T=16384, D=64, W=128, dtype="bf16",
                            gate_mu=3.0, gate_sigma=1.0, seed=2),
    "hybrid_7p6b": Workload("hybrid_7p6b", B=1, H=32, d=128, T=32768, W=64,
                            D_per_head=tuple([1] * 8 + [64] * 24), dtype="bf16",
                            gate_mu=2.0, gate_sigma=1.5, seed=3),
    "decode_7p6b": Workload("decode_7p6b", B=32, H=32, d=128, T=65536, D=64, W=128, dtype="bf16",
                            gate_mu=2.0, gate_sigma=1.0, seed=4, steps=256),
}


def prefill_inputs(w: Workload, B=None, H=None, T=None, seed=None):
    """q, k, v, a on the CPU in w's dtype, shape (B, H, T, d); sizes may be overridden."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    T = w.T if T is None else T
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    shape = (B, H, T, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    a = torch.randn(shape, generator=g, dtype=torch.float32) * w.gate_sigma + w.gate_mu
    dt = w.torch_dtype
    return {"q": q.to(dt), "k": k.to(dt), "v": v.to(dt), "a": a.to(dt)}


CTX_CHUNK = 8192        # context positions drawn per generator call


def decode_context_chunk(w: Workload, b: int, h: int, c: int, device="cpu", T=None):
    """Context k, v, a of slice (b, h) at positions [c*CTX_CHUNK, min((c+1)*CTX_CHUNK, T)),
    shape (3, rows, d), from a generator seeded with (seed, b, h, c) on `device`."""
    T = w.T if T is None else T
    lo, hi = c * CTX_CHUNK, min((c + 1) * CTX_CHUNK, T)
    g = torch.Generator(device=device)
    g.manual_seed(((w.seed * 1_000_003 + b) * 1009 + h) * 4099 + c + 1)
    kva = torch.randn((3, hi - lo, w.d), generator=g, dtype=torch.float32, device=device)
    kva[2].mul_(w.gate_sigma).add_(w.gate_mu)
    return kva.to(w.torch_dtype)


def decode_context_slice(w: Workload, b: int, h: int, device="cpu", T=None):
    """Whole context k, v, a of one (batch, head) slice, shape (3, T, d)."""
    T = w.T if T is None else T
    n = (T + CTX_CHUNK - 1) // CTX_CHUNK
    return torch.cat([decode_context_chunk(w, b, h, c, device, T) for c in range(n)], dim=1)


def decode_context_block(w: Workload, c: int, device="cpu", T=None, B=None, H=None):
    """Chunk c of the context of every slice: k, v, a each (B, H, rows, d), contiguous."""
    T = w.T if T is None else T
    B = w.B if B is None else B
    H = w.H if H is None else H
    lo, hi = c * CTX_CHUNK, min((c + 1) * CTX_CHUNK, T)
    out = torch.empty((3, B, H, hi - lo, w.d), dtype=w.torch_dtype, device=device)
    for b in range(B):
        for h in range(H):
            out[:, b, h] = decode_context_chunk(w, b, h, c, device, T)
    return out[0], out[1], out[2]


def ragged_lengths(w: Workload) -> List[int]:
    """Context lengths of the ragged decode batch: sequence b holds T/2 + (T/2) b / (B-1)
    positions, evenly spread from half the workload's context to all of it."""
    half = w.T // 2
    return [half + (half * b) // max(w.B - 1, 1) for b in range(w.B)]


def decode_steps(w: Workload, steps=None):
    """Per-step new tokens q, k, v, a, each (steps, B, H, d), on the CPU in w's dtype."""
    steps = w.steps if steps is None else steps
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed * 7919 + 17)
    shape = (steps, w.B, w.H, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    a = torch.randn(shape, generator=g, dtype=torch.float32) * w.gate_sigma + w.gate_mu
    dt = w.torch_dtype
    return {"q": q.to(dt), "k": k.to(dt), "v": v.to(dt), "a": a.to(dt)}
