"""Pins of the backward oracle (``oracle.attn_bwd``): gradients of L = sum(dO * O) through the
attention definition, recomputing the probabilities ("FlashAttention on Ascend NPUs",
recomputation section).  Checked against central finite differences of the forward oracle,
against float64 autograd through an explicit masked softmax, and against closed forms."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic


def _inputs(B, Hq, Hkv, Sq, Skv, D, seed):
    return (synthetic.normal_bf16(seed, (B, Sq, Hq, D)),
            synthetic.normal_bf16(seed + 1, (B, Skv, Hkv, D)),
            synthetic.normal_bf16(seed + 2, (B, Skv, Hkv, D)),
            synthetic.normal_bf16(seed + 3, (B, Sq, Hq, D)))


def _f64(bits):
    return synthetic.bf16_bits_to_f32(bits).astype(np.float64)


@pytest.mark.parametrize("causal,window", [(0, 0), (1, 0), (1, 3)])
def test_finite_differences(causal, window):
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 5, 7, 64
    q, k, v, do = _inputs(B, Hq, Hkv, Sq, Skv, D, 100 + causal + window)
    s = 0.125
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, s, causal, window)
    qf, kf, vf, dof = _f64(q), _f64(k), _f64(v), _f64(do)

    def loss(qx, kx, vx):
        o, _ = oracle.attn(qx, kx, vx, s, causal, window)
        return float(np.sum(o * dof))

    rng = np.random.default_rng(7)
    h = 1e-5
    for name, x, g in (("q", qf, dq), ("k", kf, dk), ("v", vf, dv)):
        for _ in range(25):
            idx = tuple(rng.integers(0, n) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, kf, vf), "k": (qf, xp, vf), "v": (qf, kf, xp)}[name]
            args_m = {"q": (xm, kf, vf), "k": (qf, xm, vf), "v": (qf, kf, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-7 + 1e-6 * abs(fd), (name, idx, fd, g[idx])


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Skv,D,causal,window", [
    (2, 4, 2, 9, 13, 64, 1, 0),     # GQA, Sq != Skv (bottom-right causal)
    (1, 2, 2, 16, 16, 128, 1, 5),   # window
    (1, 3, 1, 8, 8, 64, 0, 0),      # MQA, non-causal
    (1, 2, 1, 6, 3, 64, 1, 0),      # Sq > Skv: rows with no key get zero gradients
])
def test_matches_float64_autograd(B, Hq, Hkv, Sq, Skv, D, causal, window):
    q, k, v, do = _inputs(B, Hq, Hkv, Sq, Skv, D, 200 + Sq)
    s = 0.1
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, s, causal, window)
    G = Hq // Hkv
    qt = torch.tensor(_f64(q), requires_grad=True)
    kt = torch.tensor(_f64(k), requires_grad=True)
    vt = torch.tensor(_f64(v), requires_grad=True)
    kr = kt.repeat_interleave(G, dim=2)
    vr = vt.repeat_interleave(G, dim=2)
    scores = torch.einsum("bihd,bjhd->bhij", qt, kr) * s
    i = torch.arange(Sq)[:, None] + (Skv - Sq)
    j = torch.arange(Skv)[None, :]
    keep = torch.ones(Sq, Skv, dtype=torch.bool)
    if causal:
        keep &= j <= i
    if window:
        keep &= j > i - window
    scores = scores.masked_fill(~keep, float("-inf"))
    p = torch.softmax(scores, dim=-1)
    p = torch.nan_to_num(p, nan=0.0)  # rows with no visible key
    o = torch.einsum("bhij,bjhd->bihd", p, vr)
    (o * torch.tensor(_f64(do))).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-11, rtol=0)


def test_closed_forms():
    B, Hq, Hkv, S, D = 1, 2, 1, 12, 64
    q, k, v, do = _inputs(B, Hq, Hkv, S, S, D, 300)
    # sum over keys of dV equals the sum over queries and heads of dO (each row of P sums to 1)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.125, 1, 0)
    np.testing.assert_allclose(dv.sum(axis=1)[0, 0], _f64(do).sum(axis=(1, 2))[0], atol=1e-12)
    # identical keys: every row of P is uniform over its visible keys and dQ vanishes
    k_same = np.broadcast_to(k[:, :1], k.shape).copy()
    dq2, dk2, dv2 = oracle.attn_bwd(q, k_same, v, do, 0.125, 1, 0)
    assert np.max(np.abs(dq2)) < 1e-12
    # the keys' gradient sums to zero over keys (row sums of dS vanish)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
