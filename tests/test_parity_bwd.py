"""GPU parity of the backward pass (fa_bwd, after fa_fwd on the same inputs) against the fp64
gradients of the oracle.

The bar, per gradient tensor T (dQ, dK, dV), relative to its largest reference magnitude:
max|err| <= 2e-2 * max|T_ref| and mean|err| <= 2e-3 * max|T_ref|.  The kernel works from the
bf16 O and fp32 LSE of the forward pass and rounds P and dS to bf16 before the tensor-core
products (relative 2^-9 each) with fp32 accumulation, then rounds the gradients to bf16."""
import math

import numpy as np
import pytest

import oracle
import synthetic
from parity_util import to_dev_bf16

pytestmark = pytest.mark.gpu

REL_MAX = 2e-2
REL_MEAN = 2e-3


@pytest.fixture(scope="module")
def fa():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tiled_attention_26_b200 as m
    m.lib()
    return m


def _grads(fa, q, k, v, do, s, causal, window):
    import torch
    qd, kd, vd, dod = (to_dev_bf16(x) for x in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, causal=causal, window=window, scale=s)
    dq, dk, dv = fa.fa_bwd(qd, kd, vd, o, dod, lse, causal=causal, window=window, scale=s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    return tuple(t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv))


def _check(name, got, ref, what):
    top = np.max(np.abs(ref))
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what} {name}: non-finite"
    print(f"{what} {name}: max|ref| {top:.3e} max|err| {err.max():.3e} "
          f"({err.max() / top:.2e}) mean|err| {err.mean():.3e} ({err.mean() / top:.2e})")
    assert err.max() <= REL_MAX * top, f"{what} {name}: max|err| {err.max():.3e} vs {top:.3e}"
    assert err.mean() <= REL_MEAN * top, f"{what} {name}: mean|err| {err.mean():.3e}"


CASES = [
    # B, Hq, Hkv, Sq, Skv, D, causal, window
    (1, 2, 2, 128, 128, 128, 0, 0),
    (1, 2, 2, 256, 256, 128, 1, 0),
    (2, 4, 2, 300, 300, 128, 1, 0),       # GQA, ragged tail
    (1, 8, 1, 200, 333, 128, 1, 0),       # MQA, Sq != Skv (bottom-right causal)
    (1, 4, 4, 384, 384, 64, 1, 96),       # window, D=64
    (2, 16, 2, 160, 160, 128, 0, 0),      # G=8 packed rows, non-causal
    (1, 2, 1, 100, 40, 128, 1, 0),        # Sq > Skv: rows without keys
    (1, 16, 1, 130, 257, 64, 1, 0),       # G = 16, D = 64, Sq != Skv, ragged key tail
    (2, 4, 2, 129, 129, 128, 1, 64),      # window, one row past a tile, two batches
    (1, 2, 2, 1000, 1000, 128, 0, 0),     # non-causal, eight key tiles per query tile
]


@pytest.mark.parametrize("case", CASES)
def test_backward_full_oracle(fa, case):
    B, Hq, Hkv, Sq, Skv, D, causal, window = case
    seed = 5000 + Sq + Skv
    q = synthetic.normal_bf16(seed, (B, Sq, Hq, D))
    k = synthetic.normal_bf16(seed + 1, (B, Skv, Hkv, D))
    v = synthetic.normal_bf16(seed + 2, (B, Skv, Hkv, D))
    do = synthetic.normal_bf16(seed + 3, (B, Sq, Hq, D))
    s = float(np.float32(1 / math.sqrt(D)))
    dq, dk, dv = _grads(fa, q, k, v, do, s, causal, window)
    rq, rk, rv = oracle.attn_bwd(q, k, v, do, s, causal, window)
    what = f"bwd B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Skv{Skv} D{D} c{causal} w{window}"
    _check("dq", dq, rq, what)
    _check("dk", dk, rk, what)
    _check("dv", dv, rv, what)


def test_backward_dk_dv_repeat_bitwise_dq_within_rounding(fa):
    # dK and dV are deterministic; dQ adds per-key-tile fp32 shares in the order the reductions
    # land, so two runs agree to within a few fp32 roundings before the bf16 rounding
    import torch
    B, Hq, Hkv, S, D = 1, 4, 2, 700, 128
    q = to_dev_bf16(synthetic.normal_bf16(71, (B, S, Hq, D)))
    k = to_dev_bf16(synthetic.normal_bf16(72, (B, S, Hkv, D)))
    v = to_dev_bf16(synthetic.normal_bf16(73, (B, S, Hkv, D)))
    do = to_dev_bf16(synthetic.normal_bf16(74, (B, S, Hq, D)))
    s = float(np.float32(1 / math.sqrt(D)))
    o, lse = fa.fa_fwd(q, k, v, causal=True, scale=s)
    g1 = fa.fa_bwd(q, k, v, o, do, lse, causal=True, scale=s)
    g2 = fa.fa_bwd(q, k, v, o, do, lse, causal=True, scale=s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    d = (g1[0].float() - g2[0].float()).abs()
    assert d.max().item() <= 2 ** -7 * max(g1[0].float().abs().max().item(), 1e-3)


def test_backward_invariants(fa):
    # sum over keys of dV equals the sum over queries of dO (rows of P sum to 1), and dK sums to
    # zero over keys (rows of dS sum to zero); both per (batch, KV head) for MHA
    B, H, S, D = 1, 2, 512, 128
    q = synthetic.normal_bf16(61, (B, S, H, D))
    k = synthetic.normal_bf16(62, (B, S, H, D))
    v = synthetic.normal_bf16(63, (B, S, H, D))
    do = synthetic.normal_bf16(64, (B, S, H, D))
    s = float(np.float32(1 / math.sqrt(D)))
    dq, dk, dv = _grads(fa, q, k, v, do, s, 1, 0)
    dof = synthetic.bf16_bits_to_f32(do).astype(np.float64)
    np.testing.assert_allclose(dv.sum(axis=1), dof.sum(axis=1), atol=0.05 * np.abs(dof.sum(axis=1)).max())
    assert np.abs(dk.sum(axis=1)).max() <= 0.02 * np.abs(dk).max() * math.sqrt(S)


def test_backward_full_size_one_head(fa):
    # the MHA causal workload (B=2, H=32, S=4096, D=128) through the kernels; the oracle checks
    # head (b=1, h=31) in full (an MHA head's gradients depend on that head's inputs only)
    import torch
    w = synthetic.WORKLOADS["mha_causal"]
    q, k, v = synthetic.make_qkv_torch(w, "cuda")
    do = synthetic.normal_bf16_torch(w.seed(3), w.q_shape(), "cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=True, scale=w.scale)
    dq, dk, dv = fa.fa_bwd(q, k, v, o, do, lse, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    from parity_util import to_host_bits
    b, h = 1, 31
    sl = lambda t: np.ascontiguousarray(to_host_bits(t[b:b + 1, :, h:h + 1]))
    rq, rk, rv = oracle.attn_bwd(sl(q), sl(k), sl(v), sl(do), w.scale, 1, 0)
    g = lambda t: t[b:b + 1, :, h:h + 1].float().cpu().numpy().astype(np.float64)
    _check("dq", g(dq), rq, "mha_causal full b1 h31")
    _check("dk", g(dk), rk, "mha_causal full b1 h31")
    _check("dv", g(dv), rv, "mha_causal full b1 h31")
