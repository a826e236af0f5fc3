"""Pins of the float64 oracle to facts other than itself (CPU only).

Each test checks the oracle against a closed form, a special case that reduces to a textbook
or library routine (torch's scaled-dot-product attention in float64), an invariant of the
method, brute force on tiny inputs, or a number the pages print.  The brute-force references
here are built by slicing and explicit products, not by calling the oracle's own predicate.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def sdpa(q, k, v, causal=False, scale=None):
    """Library attention in float64 (torch, CPU)."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)).double() for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                            scale=scale).numpy()


def closed_form_recurrence(x, a, h0):
    """h_t = sum_s (prod_{r=s+1..t} g_r)(1-g_s) x_s + (prod_{r=0..t} g_r) h0, by brute force."""
    T = x.shape[0]
    g = 1.0 / (1.0 + np.exp(-a))
    y = np.zeros_like(x)
    for t in range(T):
        acc = np.prod(g[0:t + 1], axis=0) * h0
        for s in range(t + 1):
            acc = acc + np.prod(g[s + 1:t + 1], axis=0) * (1.0 - g[s]) * x[s]
        y[t] = acc
    return y


# ----------------------------------------------------------------------------- recurrence
# "RAT+ Deep Dive" section 2.1: forget-gate recurrence over the full sequence.

def test_recurrence_matches_closed_form():
    T, d = 37, 5
    x = RNG.standard_normal((2, T, d))
    a = RNG.standard_normal((2, T, d)) * 1.5 + 1.0
    h0 = RNG.standard_normal((2, d))
    y, hT = oracle.recurrence(x, a, h0)
    for bh in range(2):
        ref = closed_form_recurrence(x[bh], a[bh], h0[bh])
        np.testing.assert_allclose(y[bh], ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(hT[bh], ref[-1], rtol=1e-12, atol=1e-12)


def test_recurrence_zero_gate_is_identity():
    # g = sigmoid(-1e4) = 0 exactly in float64, so h_t = x_t exactly.
    x = RNG.standard_normal((3, 50, 8))
    a = np.full_like(x, -1.0e4)
    h0 = RNG.standard_normal((3, 8))
    y, _ = oracle.recurrence(x, a, h0)
    assert np.array_equal(y, x)


def test_recurrence_unit_gate_holds_state():
    # g = 1 exactly: the state never changes, h_t = h0.
    x = RNG.standard_normal((2, 20, 4))
    a = np.full_like(x, 1.0e4)
    h0 = RNG.standard_normal((2, 4))
    y, hT = oracle.recurrence(x, a, h0)
    assert np.array_equal(y, np.broadcast_to(h0[:, None, :], y.shape))
    assert np.array_equal(hT, h0)


def test_recurrence_constant_gate_geometric():
    # constant g = c, x = 1, h0 = 0:  h_t = 1 - c^(t+1).
    c = 0.9
    T = 200
    a = np.full((1, T, 3), math.log(c / (1 - c)))
    x = np.ones((1, T, 3))
    y, _ = oracle.recurrence(x, a)
    ref = 1.0 - c ** (np.arange(T) + 1.0)
    np.testing.assert_allclose(y[0, :, 0], ref, rtol=1e-12, atol=1e-13)


def test_recurrence_associative_scan_any_bracketing():
    # Prefill by associative scan ("RAT+ Deep Dive" 2.1, 7.3): composing the affine maps
    # h -> A h + B with a tree of any shape gives the sequential result.
    T, d = 64, 6
    x = RNG.standard_normal((T, d))
    a = RNG.standard_normal((T, d)) + 2.0
    g = 1.0 / (1.0 + np.exp(-a))
    A, Bv = g.copy(), (1.0 - g) * x
    step = 1
    while step < T:           # Hillis-Steele inclusive scan of (A, B) pairs
        A2, B2 = A.copy(), Bv.copy()
        A2[step:] = A[step:] * A[:-step]
        B2[step:] = A[step:] * Bv[:-step] + Bv[step:]
        A, Bv = A2, B2
        step *= 2
    y, _ = oracle.recurrence(x[None], a[None])
    np.testing.assert_allclose(y[0], Bv, rtol=1e-12, atol=1e-12)


def test_recurrence_chunked_equals_whole():
    # Chunked prefill: carrying hT of a first part as h0 of the second gives the whole run.
    x = RNG.standard_normal((2, 90, 7))
    a = RNG.standard_normal((2, 90, 7)) + 2.0
    y, hT = oracle.recurrence(x, a)
    y1, h1 = oracle.recurrence(x[:, :33], a[:, :33])
    y2, h2 = oracle.recurrence(x[:, 33:], a[:, 33:], h1)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(h2, hT, rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------- RoPE

@pytest.mark.parametrize("pos0,L", [(7, 100), (3, 64)])
def test_reset_outside_the_sequence_is_the_full_recurrence(pos0, L):
    # no block boundary in pos0 .. pos0+T-1: identical operations, identical bits
    x, a = RNG.standard_normal((3, 50, 5)), RNG.standard_normal((3, 50, 5))
    h0 = RNG.standard_normal((3, 5))
    y0, hT0 = oracle.recurrence(x, a, h0)
    y1, hT1 = oracle.recurrence(x, a, h0, pos0=pos0, reset_every=L)
    assert np.array_equal(y0, y1) and np.array_equal(hT0, hT1)


def test_reset_every_position_keeps_only_the_input_term():
    # L = 1: every step starts from an empty state, h_t = (1 - g_t) x_t
    x, a = RNG.standard_normal((2, 40, 4)), 3 * RNG.standard_normal((2, 40, 4))
    y, _ = oracle.recurrence(x, a, RNG.standard_normal((2, 4)), pos0=5, reset_every=1)
    g = 1.0 / (1.0 + np.exp(-a))
    np.testing.assert_allclose(y, (1.0 - g) * x, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("pos0,L", [(0, 16), (5, 16), (13, 7), (64, 64)])
def test_reset_equals_independent_blocks(pos0, L):
    # the chunk-local recurrence is the full recurrence run separately on every block of L
    # positions, from zero at each block start (and from h0 for a block already under way)
    T = 90
    x, a = RNG.standard_normal((2, T, 3)), RNG.standard_normal((2, T, 3))
    h0 = RNG.standard_normal((2, 3))
    y, hT = oracle.recurrence(x, a, h0, pos0=pos0, reset_every=L)
    want = np.empty_like(y)
    t = 0
    h = h0
    while t < T:
        if (pos0 + t) % L == 0:
            h = np.zeros_like(h0)
        end = min(T, t + L - (pos0 + t) % L)      # up to the next block start
        ys, h = oracle.recurrence(x[:, t:end], a[:, t:end], h)
        want[:, t:end] = ys
        t = end
    assert np.array_equal(y, want) and np.array_equal(hT, h)


def test_reset_brute_force_sum():
    # y_t = sum over s in t's block (s <= t) of (prod_{r=s+1..t} g_r)(1-g_s) x_s, plus the carried
    # h0 term when t's block began before pos0
    T, L, pos0 = 23, 6, 4
    x, a = RNG.standard_normal((1, T, 2)), RNG.standard_normal((1, T, 2))
    h0 = RNG.standard_normal((1, 2))
    y, _ = oracle.recurrence(x, a, h0, pos0=pos0, reset_every=L)
    g = 1.0 / (1.0 + np.exp(-a[0]))
    for t in range(T):
        start = t - ((pos0 + t) % L)              # first position of t's block (may be < 0)
        acc = np.zeros(2)
        for s_ in range(max(start, 0), t + 1):
            acc += np.prod(g[s_ + 1:t + 1], axis=0) * (1 - g[s_]) * x[0, s_]
        if start < 0:
            acc += np.prod(g[0:t + 1], axis=0) * h0[0]
        np.testing.assert_allclose(y[0, t], acc, rtol=1e-12, atol=1e-13)


# ---- fixed-window recurrence (each state covers the last Lw positions only)
def test_window_longer_than_the_sequence_is_the_full_recurrence():
    # no position ever leaves the window: the full recurrence from a zero state
    x, a = RNG.standard_normal((2, 40, 3)), RNG.standard_normal((2, 40, 3))
    y = oracle.recurrence_window(x, a, Lw=40)
    want, _ = oracle.recurrence(x, a)
    np.testing.assert_allclose(y, want, rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(oracle.recurrence_window(x, a, Lw=1000), y)


def test_window_of_one_is_the_input_term():
    x, a = RNG.standard_normal((2, 30, 4)), 3 * RNG.standard_normal((2, 30, 4))
    y = oracle.recurrence_window(x, a, Lw=1)
    g = 1.0 / (1.0 + np.exp(-a))
    np.testing.assert_allclose(y, (1.0 - g) * x, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("Lw", [4, 7, 16])
def test_window_at_block_ends_equals_the_chunk_local_recurrence(Lw):
    # at t = m Lw + Lw - 1 the window is exactly block m of the chunk-local form
    T = 5 * Lw + 3
    x, a = RNG.standard_normal((2, T, 3)), RNG.standard_normal((2, T, 3))
    y = oracle.recurrence_window(x, a, Lw=Lw)
    loc, _ = oracle.recurrence(x, a, reset_every=Lw)
    ends = np.arange(Lw - 1, T, Lw)
    np.testing.assert_allclose(y[:, ends], loc[:, ends], rtol=1e-13, atol=1e-14)
    # before the first block ends the clipped window is the plain recurrence from row 0
    np.testing.assert_allclose(y[:, :Lw], loc[:, :Lw], rtol=1e-13, atol=1e-14)


def test_window_is_full_state_minus_the_decayed_old_state():
    # y_t = h_t - (prod_{r=t-Lw+1..t} g_r) h_{t-Lw} with h the full recurrence: a different formula
    T, Lw = 60, 9
    x, a = RNG.standard_normal((2, T, 3)), RNG.standard_normal((2, T, 3))
    y = oracle.recurrence_window(x, a, Lw=Lw)
    h, _ = oracle.recurrence(x, a)
    g = 1.0 / (1.0 + np.exp(-a))
    for t in range(Lw, T):
        want = h[:, t] - np.prod(g[:, t - Lw + 1:t + 1], axis=1) * h[:, t - Lw]
        np.testing.assert_allclose(y[:, t], want, rtol=1e-9, atol=1e-11)


def test_window_brute_force_sum_with_history():
    # explicit weighted sum over the window, the positions before row 0 taken from prev
    T, Lw = 11, 5
    x, a = RNG.standard_normal((1, T, 2)), RNG.standard_normal((1, T, 2))
    px, pa = RNG.standard_normal((1, Lw, 2)), RNG.standard_normal((1, Lw, 2))
    y = oracle.recurrence_window(x, a, Lw=Lw, prev_x=px, prev_a=pa)
    xs = np.concatenate([px[0], x[0]])
    gs = 1.0 / (1.0 + np.exp(-np.concatenate([pa[0], a[0]])))
    for t in range(T):
        u = t + Lw                                   # index into the joined sequence
        acc = np.zeros(2)
        for s_ in range(u - Lw + 1, u + 1):
            acc += np.prod(gs[s_ + 1:u + 1], axis=0) * (1 - gs[s_]) * xs[s_]
        np.testing.assert_allclose(y[0, t], acc, rtol=1e-12, atol=1e-13)


def test_window_history_equals_the_joined_sequence():
    T, Lw = 37, 8
    x, a = RNG.standard_normal((3, T, 2)), RNG.standard_normal((3, T, 2))
    px, pa = RNG.standard_normal((3, Lw, 2)), RNG.standard_normal((3, Lw, 2))
    y = oracle.recurrence_window(x, a, Lw=Lw, prev_x=px, prev_a=pa)
    joined = oracle.recurrence_window(np.concatenate([px, x], 1), np.concatenate([pa, a], 1), Lw=Lw)
    np.testing.assert_array_equal(y, joined[:, Lw:])


# ---- backward of the recurrence step
def _torch_layer(k, v, a, h0k, h0v, pos0, base):
    """The forward step written with torch float64 ops, for autograd to differentiate."""
    import torch
    T, d = k.shape[-2], k.shape[-1]
    g = torch.sigmoid(a)
    hk, hv = h0k, h0v
    yk, yv = [], []
    for t in range(T):
        hk = g[..., t, :] * hk + (1 - g[..., t, :]) * k[..., t, :]
        hv = g[..., t, :] * hv + (1 - g[..., t, :]) * v[..., t, :]
        yk.append(hk)
        yv.append(hv)
    yk, yv = torch.stack(yk, -2), torch.stack(yv, -2)
    if base > 0:
        half = d // 2
        theta = base ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
        ang = (pos0 + torch.arange(T, dtype=torch.float64))[:, None] * theta[None, :]
        c, s_ = torch.cos(ang), torch.sin(ang)
        y1, y2 = yk[..., :half], yk[..., half:]
        yk = torch.cat([y1 * c - y2 * s_, y2 * c + y1 * s_], -1)
    return yk, yv, hk, hv


@pytest.mark.parametrize("base,pos0", [(0.0, 0), (10000.0, 37)])
def test_backward_matches_autograd(base, pos0):
    import torch
    shp = (2, 9, 6)
    k, v, a = (torch.tensor(RNG.standard_normal(shp), requires_grad=True) for _ in range(3))
    h0k, h0v = (torch.tensor(RNG.standard_normal((2, 6)), requires_grad=True) for _ in range(2))
    dyk, dyv = RNG.standard_normal(shp), RNG.standard_normal(shp)
    dhk, dhv = RNG.standard_normal((2, 6)), RNG.standard_normal((2, 6))
    yk, yv, hk, hv = _torch_layer(k, v, a, h0k, h0v, pos0, base)
    loss = ((yk * torch.tensor(dyk)).sum() + (yv * torch.tensor(dyv)).sum() +
            (hk * torch.tensor(dhk)).sum() + (hv * torch.tensor(dhv)).sum())
    loss.backward()
    dk, dv, da, dh0k, dh0v = oracle.recurrence_layer_backward(
        k.detach().numpy(), v.detach().numpy(), a.detach().numpy(), dyk, dyv,
        h0k.detach().numpy(), h0v.detach().numpy(), dhk, dhv, pos0=pos0, rope_base=base)
    for mine, ref in ((dk, k.grad), (dv, v.grad), (da, a.grad), (dh0k, h0k.grad), (dh0v, h0v.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_finite_differences():
    # central differences of L = <dy, y(k, a, h0)> + <dhT, hT> on single elements
    T, d = 7, 3
    x, a = RNG.standard_normal((1, T, d)), RNG.standard_normal((1, T, d))
    h0, dy, dhT = RNG.standard_normal((1, d)), RNG.standard_normal((1, T, d)), RNG.standard_normal((1, d))

    def L(x_, a_, h0_):
        y, hT = oracle.recurrence(x_, a_, h0_)
        return float((y * dy).sum() + (hT * dhT).sum())

    dx, dg, dh0 = oracle.recurrence_backward(x, a, dy, h0, dhT)
    g = 1.0 / (1.0 + np.exp(-a))
    da = dg * g * (1 - g)
    eps = 1e-6
    for (t, c) in ((0, 0), (3, 1), (6, 2)):
        for arr, grad in ((x, dx), (a, da)):
            p_, m_ = arr.copy(), arr.copy()
            p_[0, t, c] += eps
            m_[0, t, c] -= eps
            args_p = (p_, a, h0) if arr is x else (x, p_, h0)
            args_m = (m_, a, h0) if arr is x else (x, m_, h0)
            fd = (L(*args_p) - L(*args_m)) / (2 * eps)
            assert abs(fd - grad[0, t, c]) <= 1e-7 * max(1.0, abs(fd)), (t, c, fd, grad[0, t, c])
    for c in range(d):
        p_, m_ = h0.copy(), h0.copy()
        p_[0, c] += eps
        m_[0, c] -= eps
        fd = (L(x, a, p_) - L(x, a, m_)) / (2 * eps)
        assert abs(fd - dh0[0, c]) <= 1e-7 * max(1.0, abs(fd))


def test_backward_is_the_adjoint_of_the_linear_map():
    # at fixed gates and h0 = 0, x -> y is linear: <dy, y(x)> = <dx(dy), x> exactly
    x, a, dy = (RNG.standard_normal((3, 40, 4)) for _ in range(3))
    y, _ = oracle.recurrence(x, a)
    dx, _, _ = oracle.recurrence_backward(x, a, dy)
    lhs, rhs = float((dy * y).sum()), float((dx * x).sum())
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), 1.0)


def test_backward_zero_gate_passes_the_gradient_through():
    # g = 0: y = x, so dx = dy exactly and the gate gets no gradient (g (1 - g) = 0)
    x, dy = RNG.standard_normal((2, 20, 3)), RNG.standard_normal((2, 20, 3))
    a = np.full_like(x, -1.0e4)
    dk, dv, da, dh0k, _ = oracle.recurrence_layer_backward(x, x, a, dy, dy)
    assert np.array_equal(dk, dy) and np.array_equal(dv, dy)
    assert np.all(da == 0.0) and np.all(dh0k == 0.0)


# ---- backward of the chunk-local recurrence (the state restarts at multiples of L)
def _torch_layer_reset(k, v, a, h0k, h0v, pos0, L, base):
    """The chunk-local forward step written with torch float64 ops, for autograd."""
    import torch
    T, d = k.shape[-2], k.shape[-1]
    g = torch.sigmoid(a)
    hk, hv = h0k, h0v
    yk, yv = [], []
    for t in range(T):
        if (pos0 + t) % L == 0:
            hk, hv = torch.zeros_like(hk), torch.zeros_like(hv)
        hk = g[..., t, :] * hk + (1 - g[..., t, :]) * k[..., t, :]
        hv = g[..., t, :] * hv + (1 - g[..., t, :]) * v[..., t, :]
        yk.append(hk)
        yv.append(hv)
    yk, yv = torch.stack(yk, -2), torch.stack(yv, -2)
    if base > 0:
        half = d // 2
        theta = base ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
        ang = (pos0 + torch.arange(T, dtype=torch.float64))[:, None] * theta[None, :]
        c, s_ = torch.cos(ang), torch.sin(ang)
        y1, y2 = yk[..., :half], yk[..., half:]
        yk = torch.cat([y1 * c - y2 * s_, y2 * c + y1 * s_], -1)
    return yk, yv, hk, hv


@pytest.mark.parametrize("base,pos0,L", [(0.0, 0, 4), (10000.0, 37, 5), (0.0, 3, 1), (500.0, 1, 16)])
def test_reset_backward_matches_autograd(base, pos0, L):
    import torch
    shp = (2, 11, 6)
    k, v, a = (torch.tensor(RNG.standard_normal(shp), requires_grad=True) for _ in range(3))
    h0k, h0v = (torch.tensor(RNG.standard_normal((2, 6)), requires_grad=True) for _ in range(2))
    dyk, dyv = RNG.standard_normal(shp), RNG.standard_normal(shp)
    dhk, dhv = RNG.standard_normal((2, 6)), RNG.standard_normal((2, 6))
    yk, yv, hk, hv = _torch_layer_reset(k, v, a, h0k, h0v, pos0, L, base)
    loss = ((yk * torch.tensor(dyk)).sum() + (yv * torch.tensor(dyv)).sum() +
            (hk * torch.tensor(dhk)).sum() + (hv * torch.tensor(dhv)).sum())
    loss.backward()
    dk, dv, da, dh0k, dh0v = oracle.recurrence_layer_backward(
        k.detach().numpy(), v.detach().numpy(), a.detach().numpy(), dyk, dyv,
        h0k.detach().numpy(), h0v.detach().numpy(), dhk, dhv, pos0=pos0, rope_base=base,
        reset_every=L)
    for mine, ref in ((dk, k.grad), (dv, v.grad), (da, a.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12)
    for mine, ref in ((dh0k, h0k.grad), (dh0v, h0v.grad)):
        ref = ref.numpy() if ref is not None else np.zeros_like(mine)
        np.testing.assert_allclose(mine, ref, rtol=1e-10, atol=1e-12)


def test_reset_backward_finite_differences():
    # central differences of L = <dy, y> + <dhT, hT> through the oracle's chunk-local forward
    T, d, pos0, Lb = 9, 3, 2, 4
    x, a = RNG.standard_normal((1, T, d)), RNG.standard_normal((1, T, d))
    h0, dy, dhT = RNG.standard_normal((1, d)), RNG.standard_normal((1, T, d)), RNG.standard_normal((1, d))

    def L(x_, a_, h0_):
        y, hT = oracle.recurrence(x_, a_, h0_, pos0=pos0, reset_every=Lb)
        return float((y * dy).sum() + (hT * dhT).sum())

    dx, dg, dh0 = oracle.recurrence_backward(x, a, dy, h0, dhT, pos0=pos0, reset_every=Lb)
    g = 1.0 / (1.0 + np.exp(-a))
    da = dg * g * (1 - g)
    eps = 1e-6
    for (t, c) in ((0, 0), (1, 2), (2, 1), (5, 0), (8, 2)):
        for arr, grad in ((x, dx), (a, da)):
            p_, m_ = arr.copy(), arr.copy()
            p_[0, t, c] += eps
            m_[0, t, c] -= eps
            args_p = (p_, a, h0) if arr is x else (x, p_, h0)
            args_m = (m_, a, h0) if arr is x else (x, m_, h0)
            fd = (L(*args_p) - L(*args_m)) / (2 * eps)
            assert abs(fd - grad[0, t, c]) <= 1e-7 * max(1.0, abs(fd)), (t, c, fd, grad[0, t, c])
    for c in range(d):
        p_, m_ = h0.copy(), h0.copy()
        p_[0, c] += eps
        m_[0, c] -= eps
        fd = (L(x, a, p_) - L(x, a, m_)) / (2 * eps)
        assert abs(fd - dh0[0, c]) <= 1e-7 * max(1.0, abs(fd))


def test_reset_backward_without_a_block_start_is_the_full_backward():
    # no multiple of L among pos0 .. pos0 + T - 1: the same bits as the full-sequence backward
    x, a, dy = (RNG.standard_normal((2, 30, 4)) for _ in range(3))
    h0, dhT = RNG.standard_normal((2, 4)), RNG.standard_normal((2, 4))
    full = oracle.recurrence_backward(x, a, dy, h0, dhT)
    loc = oracle.recurrence_backward(x, a, dy, h0, dhT, pos0=1, reset_every=100)
    for f, l_ in zip(full, loc):
        np.testing.assert_array_equal(f, l_)


def test_reset_backward_every_position_keeps_only_the_input_term():
    # L = 1: y_t = (1 - g_t) x_t, so dx = (1 - g) dy (+ dhT on the last row), dg = -dy x, dh0 = 0
    x, a, dy = (RNG.standard_normal((2, 12, 3)) for _ in range(3))
    dhT = RNG.standard_normal((2, 3))
    dx, dg, dh0 = oracle.recurrence_backward(x, a, dy, None, dhT, pos0=5, reset_every=1)
    mu = dy.copy()
    mu[:, -1] += dhT
    omg = 1.0 / (1.0 + np.exp(a))
    np.testing.assert_allclose(dx, omg * mu, rtol=1e-14, atol=0)
    np.testing.assert_allclose(dg, -mu * x, rtol=1e-14, atol=0)
    assert np.all(dh0 == 0.0)


# ---- backward of the fixed-window recurrence (state restarted from zero at t - Lw + 1)
def _torch_layer_window(k, v, a, pk, pv, pa, Lw, pos0, base):
    """The window forward step with torch float64 ops, for autograd: each output row runs its
    own restarted loop over the window (history rows joined in front when given)."""
    import torch
    T, d = k.shape[-2], k.shape[-1]
    if pk is not None:
        k, v, a = (torch.cat([p_, x_], -2) for p_, x_ in ((pk, k), (pv, v), (pa, a)))
        off = Lw
    else:
        off = 0
    g = torch.sigmoid(a)
    yk, yv = [], []
    for t in range(T):
        tt = t + off
        hk = torch.zeros_like(k[..., 0, :])
        hv = torch.zeros_like(v[..., 0, :])
        for s in range(max(tt - Lw + 1, 0), tt + 1):
            hk = g[..., s, :] * hk + (1 - g[..., s, :]) * k[..., s, :]
            hv = g[..., s, :] * hv + (1 - g[..., s, :]) * v[..., s, :]
        yk.append(hk)
        yv.append(hv)
    yk, yv = torch.stack(yk, -2), torch.stack(yv, -2)
    if base > 0:
        half = d // 2
        theta = base ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
        ang = (pos0 + torch.arange(T, dtype=torch.float64))[:, None] * theta[None, :]
        c, s_ = torch.cos(ang), torch.sin(ang)
        y1, y2 = yk[..., :half], yk[..., half:]
        yk = torch.cat([y1 * c - y2 * s_, y2 * c + y1 * s_], -1)
    return yk, yv


@pytest.mark.parametrize("base,pos0,Lw,hist", [(0.0, 0, 4, False), (10000.0, 37, 5, True),
                                               (0.0, 0, 1, True), (500.0, 3, 16, False),
                                               (0.0, 0, 6, True)])
def test_window_backward_matches_autograd(base, pos0, Lw, hist):
    import torch
    shp = (2, 13, 6)
    k, v, a = (torch.tensor(RNG.standard_normal(shp), requires_grad=True) for _ in range(3))
    pk = pv = pa = None
    if hist:
        pk, pv, pa = (torch.tensor(RNG.standard_normal((2, Lw, 6)), requires_grad=True)
                      for _ in range(3))
    dyk, dyv = RNG.standard_normal(shp), RNG.standard_normal(shp)
    yk, yv = _torch_layer_window(k, v, a, pk, pv, pa, Lw, pos0, base)
    ((yk * torch.tensor(dyk)).sum() + (yv * torch.tensor(dyv)).sum()).backward()
    np_ = (lambda t: None if t is None else t.detach().numpy())
    dk, dv, da, dpk, dpv, dpa = oracle.recurrence_window_layer_backward(
        np_(k), np_(v), np_(a), dyk, dyv, Lw, np_(pk), np_(pv), np_(pa), pos0=pos0, rope_base=base)
    pairs = [(dk, k.grad), (dv, v.grad), (da, a.grad)]
    if hist:
        pairs += [(dpk, pk.grad), (dpv, pv.grad), (dpa, pa.grad)]
    else:
        assert dpk is None and dpv is None and dpa is None
    for mine, ref in pairs:
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_window_backward_finite_differences():
    # central differences of L = <dy, y> through the oracle's own window forward, history included
    T, d, Lw = 11, 3, 4
    x, a = RNG.standard_normal((1, T, d)), RNG.standard_normal((1, T, d))
    px, pa = RNG.standard_normal((1, Lw, d)), RNG.standard_normal((1, Lw, d))
    dy = RNG.standard_normal((1, T, d))

    def L(x_, a_, px_, pa_):
        return float((oracle.recurrence_window(x_, a_, Lw, px_, pa_) * dy).sum())

    dx, dg, dpx, dpg = oracle.recurrence_window_backward(x, a, dy, Lw, px, pa)
    sig = lambda z: 1.0 / (1.0 + np.exp(-z))
    da, dpa = dg * sig(a) * (1 - sig(a)), dpg * sig(pa) * (1 - sig(pa))
    eps = 1e-6
    cases = [(x, dx, 0), (a, da, 1), (px, dpx, 2), (pa, dpa, 3)]
    for arr, grad, slot in cases:
        for (t, c) in ((0, 0), (1, 2), (arr.shape[1] - 1, 1), (arr.shape[1] // 2, 0)):
            p_, m_ = arr.copy(), arr.copy()
            p_[0, t, c] += eps
            m_[0, t, c] -= eps
            base_args = [x, a, px, pa]
            ap, am = list(base_args), list(base_args)
            ap[slot], am[slot] = p_, m_
            fd = (L(*ap) - L(*am)) / (2 * eps)
            assert abs(fd - grad[0, t, c]) <= 1e-7 * max(1.0, abs(fd)), (slot, t, c, fd, grad[0, t, c])
    # the oldest history row is outside every window of rows 0 .. T-1
    assert np.all(dpx[:, 0] == 0.0) and np.all(dpg[:, 0] == 0.0)


def test_window_backward_longer_than_the_sequence_is_the_full_backward():
    # Lw >= T and no history: every window starts at row 0, the full-sequence recurrence from 0
    x, a, dy = (RNG.standard_normal((2, 20, 4)) for _ in range(3))
    dx, dg, _, _ = oracle.recurrence_window_backward(x, a, dy, Lw=20)
    fx, fg, _ = oracle.recurrence_backward(x, a, dy)
    np.testing.assert_allclose(dx, fx, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dg, fg, rtol=1e-12, atol=1e-14)


def test_window_backward_of_one_keeps_only_the_input_term():
    # Lw = 1: y_t = (1 - g_t) x_t, so dx = (1 - g) dy and dg = -x dy
    x, a, dy = (RNG.standard_normal((2, 12, 3)) for _ in range(3))
    dx, dg, _, _ = oracle.recurrence_window_backward(x, a, dy, Lw=1)
    np.testing.assert_allclose(dx, dy / (1.0 + np.exp(a)), rtol=1e-14, atol=0)
    np.testing.assert_allclose(dg, -x * dy, rtol=1e-14, atol=0)


def test_window_backward_is_the_adjoint_of_the_linear_map():
    # at fixed gates the window map x -> y is linear: <dy, y(x)> = <dx(dy), x> (+ history part)
    x, a, dy = (RNG.standard_normal((3, 70, 4)) for _ in range(3))
    px, pa = RNG.standard_normal((3, 8, 4)), RNG.standard_normal((3, 8, 4))
    y = oracle.recurrence_window(x, a, 8, px, pa)
    dx, _, dpx, _ = oracle.recurrence_window_backward(x, a, dy, 8, px, pa)
    lhs, rhs = float((dy * y).sum()), float((dx * x).sum() + (dpx * px).sum())
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), 1.0)


def test_rope_transpose_inverts_rope():
    x = RNG.standard_normal((2, 11, 8))
    np.testing.assert_allclose(oracle.rope_transpose(oracle.rope(x, 123, 500.0), 123, 500.0), x,
                               rtol=1e-12, atol=1e-13)


# ---- backward of the dilated attention
def _torch_attention(q, k, v, D, W, scale):
    """Masked softmax attention in torch float64, the mask built from the key-set definition,
    for autograd to differentiate."""
    import torch
    T = q.shape[-2]
    mask = torch.tensor([[oracle.in_key_set(t, j, D, W) for j in range(T)] for t in range(T)])
    s = scale * (q @ k.transpose(-1, -2))
    s = s.masked_fill(~mask, float("-inf"))
    return torch.softmax(s, -1) @ v


@pytest.mark.parametrize("D,W,T", [(1, 0, 12), (4, 0, 19), (3, 5, 17), (8, 1, 30)])
def test_attention_backward_matches_autograd(D, W, T):
    import torch
    shp = (2, T, 8)
    q, k, v = (torch.tensor(RNG.standard_normal(shp), requires_grad=True) for _ in range(3))
    dO = RNG.standard_normal(shp)
    o = _torch_attention(q, k, v, D, W, 0.4)
    (o * torch.tensor(dO)).sum().backward()
    dq, dk, dv = oracle.dilated_attention_backward(q.detach().numpy()[None], k.detach().numpy()[None],
                                                   v.detach().numpy()[None], dO[None], D=D, W=W,
                                                   scale=0.4)
    for mine, ref in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        np.testing.assert_allclose(mine[0], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_backward_rope_and_head_dilations():
    # per-head D and the RoPE of q: autograd through rotate-half written in torch
    import torch
    B, H, T, d, base, pos0 = 1, 2, 15, 8, 100.0, 9
    q, k, v = (torch.tensor(RNG.standard_normal((B, H, T, d)), requires_grad=True) for _ in range(3))
    dO = RNG.standard_normal((B, H, T, d))
    half = d // 2
    theta = base ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
    ang = (pos0 + torch.arange(T, dtype=torch.float64))[:, None] * theta[None, :]
    c, s_ = torch.cos(ang), torch.sin(ang)
    qh = torch.cat([q[..., :half] * c - q[..., half:] * s_, q[..., half:] * c + q[..., :half] * s_], -1)
    Dh = [2, 5]
    o = torch.stack([_torch_attention(qh[:, h], k[:, h], v[:, h], Dh[h], 3, 0.5) for h in range(H)], 1)
    (o * torch.tensor(dO)).sum().backward()
    dq, dk, dv = oracle.dilated_attention_backward(q.detach().numpy(), k.detach().numpy(),
                                                   v.detach().numpy(), dO, W=3, D_per_head=Dh,
                                                   scale=0.5, rope_base=base, pos0=pos0)
    for mine, ref in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_backward_finite_differences():
    B, H, T, d, D, W = 1, 1, 10, 4, 3, 2
    q, k, v, dO = (RNG.standard_normal((B, H, T, d)) for _ in range(4))

    def L(q_, k_, v_):
        return float((oracle.dilated_attention(q_, k_, v_, D=D, W=W) * dO).sum())

    dq, dk, dv = oracle.dilated_attention_backward(q, k, v, dO, D=D, W=W)
    eps = 1e-6
    for arr, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        for (t, c) in ((0, 0), (5, 2), (9, 3)):
            p_, m_ = arr.copy(), arr.copy()
            p_[0, 0, t, c] += eps
            m_[0, 0, t, c] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = p_, m_
            fd = (L(*args_p) - L(*args_m)) / (2 * eps)
            assert abs(fd - grad[0, 0, t, c]) <= 1e-7 * max(1.0, abs(fd)), (which, t, c)


def test_attention_backward_single_key_passes_dv_only():
    # D > T, W = 0: every query sees only itself, o = v exactly: dv = dO, dq = dk = 0
    q, k, v, dO = (RNG.standard_normal((1, 2, 9, 4)) for _ in range(4))
    dq, dk, dv = oracle.dilated_attention_backward(q, k, v, dO, D=100, W=0)
    np.testing.assert_array_equal(dv, dO)
    assert np.all(dq == 0.0) and np.all(dk == 0.0)


# ---- attention sinks (StreamingLLM layers)
@pytest.mark.parametrize("D,W,n_sink", [(10**6, 8, 4), (10**6, 1, 3), (4, 0, 6), (3, 5, 7)])
def test_sink_key_count_closed_form(D, W, n_sink):
    We = max(W, 1)
    for t in range(60):
        lim = min(n_sink, max(0, t - We + 1))          # sinks older than the window
        dil = max(0, (t - We + 1) // D) if t - We + 1 >= D else 0
        want = min(We, t + 1) + dil + lim - lim // D    # sinks that are chunk ends count once
        assert oracle.key_count(t, D, W, n_sink) == want, (t, D, W, n_sink)


def test_streaming_attention_equals_masked_sdpa():
    # no chunk ends (D beyond T): the key set is the window plus the first n_sink positions
    import torch
    B, H, T, d, W, n_sink = 1, 2, 40, 8, 6, 4
    q, k, v = (RNG.standard_normal((B, H, T, d)) for _ in range(3))
    o = oracle.dilated_attention(q, k, v, D=10**6, W=W, n_sink=n_sink, scale=0.3)
    t_ = torch.arange(T)[:, None]
    j_ = torch.arange(T)[None, :]
    mask = (j_ <= t_) & ((j_ > t_ - W) | (j_ < n_sink))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v), attn_mask=mask, scale=0.3)
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_sinks_that_are_chunk_ends_change_nothing():
    # D = 1: every position is already a chunk end, so sinks add no key
    q, k, v = (RNG.standard_normal((1, 2, 30, 4)) for _ in range(3))
    a = oracle.dilated_attention(q, k, v, D=1, W=3)
    b = oracle.dilated_attention(q, k, v, D=1, W=3, n_sink=5)
    np.testing.assert_array_equal(a, b)


def test_decode_with_sinks_equals_prefill_rows():
    T0, steps, d, W, n_sink = 20, 15, 8, 3, 4
    Dh = [1, 4, 10**6]
    H = len(Dh)
    T = T0 + steps
    q, k, v, a = (RNG.standard_normal((1, H, T, d)) for _ in range(4))
    full = oracle.layer_prefill(q, k, v, a, D_per_head=Dh, W=W, rope_base=100.0, n_sink=n_sink)["o"]
    st = oracle.DecodeState(Dh, d, W, T, rope_base=100.0, n_sink=n_sink)
    st.prefill(k[0, :, :T0], v[0, :, :T0], a[0, :, :T0])
    for s_ in range(steps):
        t = T0 + s_
        o = st.step(q[0, :, t], k[0, :, t], v[0, :, t], a[0, :, t])
        np.testing.assert_allclose(o, full[0, :, t], rtol=1e-10, atol=1e-12)


# ---- top-k chunk selection combined with dilation
def test_topk_zero_is_the_dilated_attention():
    q, k, v = (RNG.standard_normal((1, 2, 50, 8)) for _ in range(3))
    a = oracle.dilated_attention(q, k, v, D=4, W=3, n_sink=2)
    b = oracle.topk_attention(q, k, v, D=4, W=3, n_sink=2, top_k=0)
    np.testing.assert_array_equal(a, b)


def test_topk_with_unit_chunks_adds_nothing():
    # D = 1: a chunk is its own chunk end, already a key
    q, k, v = (RNG.standard_normal((1, 2, 40, 8)) for _ in range(3))
    np.testing.assert_allclose(oracle.topk_attention(q, k, v, D=1, W=2, top_k=5),
                               oracle.dilated_attention(q, k, v, D=1, W=2), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("D,W,n_sink,top_k", [(4, 3, 0, 2), (5, 1, 3, 3), (8, 8, 0, 100)])
def test_topk_equals_masked_sdpa_with_argsort_selection(D, W, n_sink, top_k):
    # the selection by a library sort of the chunk scores, the mask built from it, SDPA over it
    import torch
    T, d, scale = 60, 8, 0.35
    q, k, v = (RNG.standard_normal((1, 1, T, d)) for _ in range(3))
    We = max(W, 1)
    mask = np.zeros((T, T), dtype=bool)
    for t in range(T):
        for j in range(t + 1):
            mask[t, j] = oracle.in_key_set(t, j, D, W, n_sink)
        nc = (t - We + 1) // D if t - We + 1 >= D else 0
        if nc:
            sc = np.array([scale * q[0, 0, t] @ k[0, 0, c * D + D - 1] for c in range(nc)])
            order = np.argsort(-sc, kind="stable")[:top_k]      # ties: the earlier chunk
            for c in order:
                mask[t, c * D:c * D + D] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v), attn_mask=torch.tensor(mask), scale=scale)
    got = oracle.topk_attention(q, k, v, D=D, W=W, n_sink=n_sink, top_k=top_k, scale=scale)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_attention_over_keys_equals_masked_sdpa():
    # explicit key lists (random subsets, in shuffled order) against library attention under the
    # matching boolean mask
    T, d, scale = 50, 16, 0.3
    q, k, v = (RNG.standard_normal((T, d)) for _ in range(3))
    for t in (0, 7, 31, 49):
        keys = RNG.permutation(t + 1)[:max(1, (t + 1) // 2)]
        mask = np.zeros((1, T), dtype=bool)
        mask[0, keys] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q[t:t + 1]), torch.tensor(k), torch.tensor(v),
            attn_mask=torch.tensor(mask), scale=scale).numpy()[0]
        np.testing.assert_allclose(oracle.attention_over_keys(q[t], k, v, keys, scale), ref,
                                   rtol=1e-12, atol=1e-13)


def test_attention_over_the_key_set_is_the_dilated_attention():
    T, d, D, W, n_sink = 90, 8, 6, 5, 2
    q, k, v = (RNG.standard_normal((1, 1, T, d)) for _ in range(3))
    scale = oracle.default_scale(d)
    ref = oracle.dilated_attention(q, k, v, D=D, W=W, n_sink=n_sink)
    for t in (0, 4, 5, 40, 89):
        keys = [j for j in range(t + 1) if oracle.in_key_set(t, j, D, W, n_sink)]
        np.testing.assert_allclose(oracle.attention_over_keys(q[0, 0, t], k[0, 0], v[0, 0], keys,
                                                              scale), ref[0, 0, t],
                                   rtol=1e-12, atol=1e-13)


def test_attention_lse_is_the_log_partition():
    # log2 sum_j exp(s_j) over the key set, by a library logsumexp over the masked scores
    from scipy.special import logsumexp
    T, d, D, W, scale = 33, 8, 4, 3, 0.4
    q, k, v = (RNG.standard_normal((1, 1, T, d)) for _ in range(3))
    _, lse = oracle.dilated_attention(q, k, v, D=D, W=W, n_sink=2, scale=scale, return_lse=True)
    for t in range(T):
        keys = [j for j in range(t + 1) if oracle.in_key_set(t, j, D, W, 2)]
        sc = scale * (k[0, 0, keys] @ q[0, 0, t])
        assert abs(lse[0, 0, t] - logsumexp(sc) / np.log(2.0)) <= 1e-12


def test_rope_matches_complex_rotation():
    d, T, pos0, base = 16, 9, 1000, 10000.0
    x = RNG.standard_normal((1, T, d))
    y = oracle.rope(x, pos0, base)
    half = d // 2
    z = x[0, :, :half] + 1j * x[0, :, half:]
    theta = base ** (-np.arange(half) * 2.0 / d)
    zr = z * np.exp(1j * (pos0 + np.arange(T))[:, None] * theta[None, :])
    np.testing.assert_allclose(y[0, :, :half], zr.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y[0, :, half:], zr.imag, rtol=1e-12, atol=1e-12)


def test_rope_relative_position_and_identity():
    d = 32
    q = RNG.standard_normal((1, 1, d))
    k = RNG.standard_normal((1, 1, d))
    assert np.array_equal(oracle.rope(q, 0), q)
    dots = []
    for shift in (0, 7, 5000):
        dots.append(float(np.dot(oracle.rope(q, 40 + shift)[0, 0], oracle.rope(k, 13 + shift)[0, 0])))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)


# ----------------------------------------------------------------------------- key set
# RAT+ abstract and "RAT+ Deep Dive" 3.1: dilation keeps every D-th key.

def closed_form_count(t, D, W):
    We = max(W, 1)
    return min(We, t + 1) + max(0, (t - We + 1) // D)


@pytest.mark.parametrize("D,W", [(1, 0), (4, 0), (16, 0), (64, 128), (64, 64), (3, 5), (7, 1), (300, 0)])
def test_key_count_closed_form(D, W):
    for t in list(range(0, 140)) + [511, 1000, 4095]:
        assert oracle.key_count(t, D, W) == closed_form_count(t, D, W)


def test_key_set_total_tiny_workload():
    # B1 H2 T256 D4 W0: each head attends to sum_t (1 + floor(t/4)) = 8320 keys; 16640 in all.
    total = sum(oracle.key_count(t, 4, 0) for t in range(256)) * 2
    assert total == 16640


def test_flops_table_golden():
    with open(os.path.join(GOLDEN, "flops_table.json")) as f:
        g = json.load(f)
    T = g["T"]
    for row in g["rows"]:
        assert oracle.key_count(T - 1, row["D"], 0) == row["keys"] == T // row["D"]
    cap = oracle.cache_capacity(T, [64])
    assert T // int(cap[0]) == g["kv_reduction_at_D64"]


# ----------------------------------------------------------------------------- attention

def rand_qkv(B, H, T, d):
    return (RNG.standard_normal((B, H, T, d)), RNG.standard_normal((B, H, T, d)),
            RNG.standard_normal((B, H, T, d)))


def test_dense_when_D_is_1():
    q, k, v = rand_qkv(1, 2, 70, 16)
    for W in (0, 1, 9, 200):
        o = oracle.dilated_attention(q, k, v, D=1, W=W)
        np.testing.assert_allclose(o, sdpa(q, k, v, causal=True), rtol=1e-11, atol=1e-12)


def test_dense_when_window_covers_sequence():
    q, k, v = rand_qkv(2, 1, 50, 8)
    o = oracle.dilated_attention(q, k, v, D=16, W=50)
    np.testing.assert_allclose(o, sdpa(q, k, v, causal=True), rtol=1e-11, atol=1e-12)


def test_self_only_when_D_exceeds_T():
    q, k, v = rand_qkv(1, 2, 40, 8)
    o = oracle.dilated_attention(q, k, v, D=41, W=0)
    assert np.array_equal(o, v)


def test_chunk_end_queries_equal_causal_attention_on_subsampled_sequence():
    # With W = 0 a query at a chunk end t = mD + D - 1 sees exactly the chunk ends 0..m:
    # dense causal attention over the stride-D subsequence starting at D - 1.
    D, T = 8, 96
    q, k, v = rand_qkv(1, 2, T, 16)
    rows = np.arange(D - 1, T, D)
    o = oracle.dilated_attention(q, k, v, D=D, W=0, rows=rows)
    ref = sdpa(q[:, :, D - 1::D], k[:, :, D - 1::D], v[:, :, D - 1::D], causal=True)
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("D,W,T", [(4, 0, 64), (8, 5, 77), (16, 16, 130), (3, 1, 40), (64, 10, 200)])
def test_general_key_set_by_slicing(D, W, T):
    # Reference built by slicing: chunk ends k[D-1 :: D] older than the window, then the window.
    d = 8
    q, k, v = rand_qkv(1, 1, T, d)
    o = oracle.dilated_attention(q, k, v, D=D, W=W)
    We = max(W, 1)
    for t in range(T):
        lo = max(0, t - We + 1)     # first window position; chunk ends stop before it
        kk = np.concatenate([k[0, 0, D - 1:lo:D], k[0, 0, lo:t + 1]])
        vv = np.concatenate([v[0, 0, D - 1:lo:D], v[0, 0, lo:t + 1]])
        ref = sdpa(q[0, 0, t:t + 1][None], kk[None], vv[None])[0, 0]
        np.testing.assert_allclose(o[0, 0, t], ref, rtol=1e-11, atol=1e-12)


def test_head_hybrid_equals_uniform_runs():
    # "RAT+ Deep Dive" 6, head-wise hybrid: each head behaves as a uniform-D run of that head.
    q, k, v = rand_qkv(2, 4, 60, 8)
    Dh = [1, 1, 4, 16]
    o = oracle.dilated_attention(q, k, v, W=3, D_per_head=Dh)
    for h, D in enumerate(Dh):
        oh = oracle.dilated_attention(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], D=D, W=3)
        np.testing.assert_array_equal(o[:, h:h + 1], oh)


def test_row_subset_equals_full():
    q, k, v = rand_qkv(1, 2, 90, 8)
    full = oracle.dilated_attention(q, k, v, D=4, W=6)
    rows = [0, 5, 44, 89]
    np.testing.assert_array_equal(oracle.dilated_attention(q, k, v, D=4, W=6, rows=rows),
                                  full[:, :, rows])


# ----------------------------------------------------------------------------- cache build

def tagged(B, H, T, d, dtype=np.float32):
    x = np.zeros((B, H, T, d), dtype=dtype)
    x[..., 0] = np.arange(T)[None, None, :]
    x[..., 1] = (np.arange(B)[:, None] * H + np.arange(H)[None, :])[:, :, None]
    x[..., 2:] = np.arange(2, d)
    return x


def test_kv_compress_index_layout():
    B, H, T, d, W = 2, 3, 100, 8, 6
    Dh = [1, 4, 7]
    Tcap = 120
    x = tagged(B, H, T, d)
    dil, ring = oracle.kv_compress(x, Dh, W, Tcap)
    caps = [Tcap // D for D in Dh]
    off = np.concatenate([[0], np.cumsum(caps)])
    for h, D in enumerate(Dh):
        n = T // D          # entries present after T positions: floor(T / D)
        np.testing.assert_array_equal(dil[:, off[h]:off[h] + n], x[:, h, D - 1::D][:, :n])
        assert np.all(dil[:, off[h] + n:off[h + 1]] == 0)
        # ring slots read from slot T % W onwards give the last W positions in order
        order = [(T - W + i) % W for i in range(W)]
        np.testing.assert_array_equal(ring[:, h, order], x[:, h, T - W:])


def test_kv_compress_chunked_equals_whole():
    B, H, T, d, W, Tcap = 1, 2, 64, 4, 5, 64
    Dh = [2, 8]
    x = tagged(B, H, T, d)
    dil, ring = oracle.kv_compress(x, Dh, W, Tcap)
    d1, r1 = oracle.kv_compress(x[:, :, :27], Dh, W, Tcap, pos0=0)
    d2, r2 = oracle.kv_compress(x[:, :, 27:], Dh, W, Tcap, pos0=27, dil=d1, ring=r1)
    np.testing.assert_array_equal(d2, dil)
    np.testing.assert_array_equal(r2, ring)


# ----------------------------------------------------------------------------- decode

@pytest.mark.parametrize("rope_base,reset", [(0.0, 0), (10000.0, 0), (10000.0, 8)])
def test_decode_equals_prefill_rows(rope_base, reset):
    B, H, T0, steps, d, W = 1, 3, 40, 12, 8, 4
    Dh = [1, 4, 16]
    T = T0 + steps
    q, k, v = rand_qkv(B, H, T, d)
    a = RNG.standard_normal((B, H, T, d)) + 2.0
    ref = oracle.layer_prefill(q, k, v, a, D_per_head=Dh, W=W, rope_base=rope_base, reset_every=reset)
    st = oracle.DecodeState(np.tile(Dh, B), d, W, Tcap=T, rope_base=rope_base, reset_every=reset)
    st.prefill(k[:, :, :T0].reshape(B * H, T0, d), v[:, :, :T0].reshape(B * H, T0, d),
               a[:, :, :T0].reshape(B * H, T0, d))
    for s in range(steps):
        t = T0 + s
        o = st.step(q[:, :, t].reshape(B * H, d), k[:, :, t].reshape(B * H, d),
                    v[:, :, t].reshape(B * H, d), a[:, :, t].reshape(B * H, d))
        np.testing.assert_allclose(o.reshape(B, H, d), ref["o"][:, :, t], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(st.hk.reshape(B, H, d), ref["hT_k"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st.hv.reshape(B, H, d), ref["hT_v"], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("rope_base,T0,Lw", [(0.0, 100, 64), (10000.0, 30, 64), (10000.0, 70, 8)])
def test_window_decode_equals_prefill_rows(rope_base, T0, Lw):
    # the fixed-window form: decoding token by token gives the attention rows of the joined
    # sequence over the window recurrence's outputs (before and after the window fills)
    B, H, steps, d, W = 1, 3, 50, 8, 3
    Dh = [1, 4, 16]
    T = T0 + steps
    q, k, v = rand_qkv(B, H, T, d)
    a = RNG.standard_normal((B, H, T, d)) + 2.0
    yk = oracle.recurrence_window(k, a, Lw)
    yv = oracle.recurrence_window(v, a, Lw)
    qr = q
    if rope_base > 0:
        yk = oracle.rope(yk, 0, rope_base)
        qr = oracle.rope(q, 0, rope_base)
    ref = oracle.dilated_attention(qr, yk, yv, D_per_head=Dh, W=W)
    st = oracle.DecodeState(np.tile(Dh, B), d, W, Tcap=T, rope_base=rope_base, window_rec=Lw)
    st.prefill(k[:, :, :T0].reshape(B * H, T0, d), v[:, :, :T0].reshape(B * H, T0, d),
               a[:, :, :T0].reshape(B * H, T0, d))
    for s in range(steps):
        t = T0 + s
        o = st.step(q[:, :, t].reshape(B * H, d), k[:, :, t].reshape(B * H, d),
                    v[:, :, t].reshape(B * H, d), a[:, :, t].reshape(B * H, d))
        np.testing.assert_allclose(o.reshape(B, H, d), ref[:, :, t], rtol=1e-11, atol=1e-12)


def test_window_decode_longer_than_the_sequence_is_the_full_recurrence():
    # a window at least as long as every position's history: the full-recurrence decode
    B, H, T0, steps, d, W = 1, 2, 20, 10, 8, 2
    Dh = [1, 4]
    q, k, v = rand_qkv(B, H, T0 + steps, d)
    a = RNG.standard_normal((B, H, T0 + steps, d)) + 2.0
    outs = []
    for Lw in (0, 64):
        st = oracle.DecodeState(np.tile(Dh, B), d, W, Tcap=T0 + steps, window_rec=Lw)
        st.prefill(k[0, :, :T0], v[0, :, :T0], a[0, :, :T0])
        outs.append([st.step(q[0, :, t], k[0, :, t], v[0, :, t], a[0, :, t]) for t in range(T0, T0 + steps)])
    np.testing.assert_allclose(np.array(outs[1]), np.array(outs[0]), rtol=1e-12, atol=1e-13)
