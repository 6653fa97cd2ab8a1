"""GPU parity at large sizes, where 32-bit index arithmetic would overflow first: a 65536-token
causal prefill, a decode over 1,048,576 INT8 keys, and the backward pass of one 6144-token head.
Sampled rows against the fp64 oracle (the full oracle would take minutes)."""
import math

import numpy as np
import pytest

import oracle
import synthetic
from parity_util import check_lse, check_o, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tiled_attention_26_b200 as m
    m.lib()
    return m


def test_prefill_64k_tokens(fa):
    import torch
    w = synthetic.Workload("long", 40, 1, 2, 1, 65536, 65536, 128, 1)
    q, k, v = synthetic.make_qkv_torch(w, "cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    rows = synthetic.sample_rows(w.B, w.Hq, w.Sq, w.seed(5), 120)
    o_ref, l_ref = oracle.attn_rows(to_host_bits(q), to_host_bits(k), to_host_bits(v), w.scale, 1, 0,
                                    rows)
    og = o.float().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]].astype(np.float64)
    lg = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
    check_o(og, o_ref, "prefill S=65536")
    check_lse(lg, l_ref, "prefill S=65536")


def test_decode_one_million_keys(fa):
    import torch
    w = synthetic.Workload("longdec", 41, 1, 8, 1, 1, 1 << 20, 128, 1, int8_kv=True)
    q, kq, vq, ks, vs = synthetic.make_decode_inputs_torch(w, "cuda")
    o, lse = fa.fa_decode_int8(q, kq, vq, ks, vs, num_splits=64, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    rows = np.array([(0, h) for h in range(8)], dtype=np.int64)
    o_ref, l_ref = oracle.decode_int8_rows(to_host_bits(q), kq.cpu().numpy(), vq.cpu().numpy(),
                                           ks.cpu().numpy(), vs.cpu().numpy(), w.scale, 1, rows)
    check_o(o.float().cpu().numpy()[0, 0].astype(np.float64), o_ref, "decode Skv=2^20")
    check_lse(lse.cpu().numpy()[0].astype(np.float64), l_ref, "decode Skv=2^20")


def test_backward_6k_head(fa):
    import torch
    w = synthetic.Workload("longbwd", 42, 1, 1, 1, 6144, 6144, 128, 1)
    q, k, v = synthetic.make_qkv_torch(w, "cuda")
    do = synthetic.normal_bf16_torch(w.seed(3), w.q_shape(), "cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=True, scale=w.scale)
    dq, dk, dv = fa.fa_bwd(q, k, v, o, do, lse, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    ref = oracle.attn_bwd(to_host_bits(q), to_host_bits(k), to_host_bits(v), to_host_bits(do),
                          w.scale, 1, 0)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        g = got.float().cpu().numpy().astype(np.float64)
        top = np.abs(r).max()
        err = np.abs(g - r)
        assert err.max() <= 2e-2 * top, (name, err.max(), top)
        assert err.mean() <= 2e-3 * top, (name, err.mean(), top)
