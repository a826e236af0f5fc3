"""Helpers shared by the GPU parity tests: running the CUDA path through the binding and
comparing with the float64 oracle.

Error measure: max |x - r| / max |r| over a tensor (max-norm relative error).  Bars: 1e-4 for
float32 paths, 2e-2 for bf16 paths against the float64 oracle.
"""
import numpy as np
import torch

import recurrence_augmented_dilated_b200 as rat

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def tol_for(dtype):
    return TOL_F32 if dtype == torch.float32 else TOL_BF16


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def rel_err(x, r) -> float:
    x, r = f64(x), f64(r)
    assert x.shape == r.shape, (x.shape, r.shape)
    den = float(np.max(np.abs(r)))
    return float(np.max(np.abs(x - r))) / (den if den > 0 else 1.0)


def gpu_recur(k, v, a, rope_base=0.0, pos0=0, h0k=None, h0v=None, ws=None, reset_every=0):
    """Run rat_recur_prefill (rat_recur_prefill_local when reset_every > 0) on device copies;
    returns (k_rec, v_rec, hT_k, hT_v) on device."""
    dev = torch.device("cuda")
    k, v, a = (x.to(dev) for x in (k, v, a))
    B, H, T, d = k.shape
    kr = torch.empty_like(k)
    vr = torch.empty_like(v)
    hTk = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    hTv = torch.empty_like(hTk)
    if ws is None:
        ws = rat.Workspace(rat.rat_recur_workspace_bytes(B, H, T, d, 0 if k.dtype == torch.float32 else 1))
    if reset_every > 0:
        rat.rat_recur_prefill_local(k, v, a, kr, vr, ws, reset_every, h0_k=h0k, h0_v=h0v,
                                    hT_k=hTk, hT_v=hTv, pos0=pos0, rope_base=rope_base)
    else:
        rat.rat_recur_prefill(k, v, a, kr, vr, ws, h0_k=h0k, h0_v=h0v, hT_k=hTk, hT_v=hTv,
                              pos0=pos0, rope_base=rope_base)
    st = rat.rat_sync_status(ws)
    assert st == 0, rat.rat_status_string(st)
    return kr, vr, hTk, hTv


def gpu_attn(q, kr, vr, D=1, W=0, D_per_head=None, rope_base=0.0, pos0=0, scale=0.0):
    dev = torch.device("cuda")
    q, kr, vr = (x.to(dev) for x in (q, kr, vr))
    o = torch.empty_like(q)
    rat.rat_dilated_attn_prefill(q, kr, vr, o, D=D, W=W, D_per_head=D_per_head, pos0=pos0,
                                 rope_base=rope_base, scale=scale)
    st = rat.rat_attn_sync_status()
    assert st == 0, "attention device error %s at site %#x" % (rat.rat_status_string(st),
                                                              rat.lib().rat_attn_error_site())
    return o
