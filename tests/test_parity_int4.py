"""GPU parity of the INT4 KV-cache decode (fa_decode_int4, fa_decode_int4_paged) against the
fp64 oracle: ragged shapes through the full oracle, the full INT4 workload on sampled rows, the
paged variant, and bitwise equality of identity paging with the contiguous kernel."""
import math

import numpy as np
import pytest

import oracle
import synthetic
from parity_util import check_lse, check_o, o_to_f64, to_dev_bf16, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import tiled_attention_26_b200 as m
    m.lib()
    return m


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


CASES = [
    # B, Hq, Hkv, Skv, D, splits
    (2, 8, 2, 1000, 128, 1),
    (2, 8, 2, 1000, 128, 16),
    (1, 4, 4, 777, 64, 5),          # MHA, D=64 (32-byte rows)
    (2, 16, 2, 513, 128, 4),        # G=8
    (1, 16, 1, 300, 128, 2),        # G=16: two blocks of 8 heads
    (3, 6, 2, 129, 64, 7),          # G=3
    (1, 2, 1, 1, 128, 1),           # one cached key
    (1, 8, 2, 5, 128, 16),          # empty splits
]


@pytest.mark.parametrize("case", CASES)
def test_int4_decode_full_oracle(fa, case):
    B, Hq, Hkv, Skv, D, splits = case
    w = synthetic.Workload("i4", 0, B, Hq, Hkv, 1, Skv, D, 1)
    q = synthetic.normal_bf16(4100 + Skv, (B, 1, Hq, D))
    k4, ks = synthetic.quantize_int4_per_token(synthetic.normal_bf16(5100 + Skv, w.kv_shape()))
    v4, vs = synthetic.quantize_int4_per_token(synthetic.normal_bf16(6100 + Skv, w.kv_shape()))
    o, lse = fa.fa_decode_int4(to_dev_bf16(q), _dev(k4), _dev(v4), _dev(ks), _dev(vs),
                               num_splits=splits, scale=w.scale)
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.decode_int4(q, k4, v4, ks, vs, w.scale)
    what = f"int4 B{B} Hq{Hq} Hkv{Hkv} Skv{Skv} D{D} splits{splits}"
    check_o(o_to_f64(o), o_ref, what)
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, what)


def test_int4_full_workload_sampled(fa):
    import torch
    w = synthetic.WORKLOADS["decode_int4"]
    q, k4, v4, ks, vs = synthetic.make_decode_int4_inputs_torch(w, "cuda")
    o, lse = fa.fa_decode_int4(q, k4, v4, ks, vs, num_splits=w.num_splits, scale=w.scale)
    o1, l1 = fa.fa_decode_int4(q, k4, v4, ks, vs, num_splits=1, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    raw = synthetic.splitmix64(w.seed(9), 0, 48)
    pairs = sorted({(int(r % np.uint64(w.B)), int((r >> np.uint64(20)) % np.uint64(w.Hq)))
                    for r in raw} | {(0, 0), (w.B - 1, w.Hq - 1)})
    rows = np.array(pairs, dtype=np.int64)
    o_ref, l_ref = oracle.decode_int4_rows(to_host_bits(q), k4.cpu().numpy(), v4.cpu().numpy(),
                                           ks.cpu().numpy(), vs.cpu().numpy(), w.scale, 1, rows)
    og = o.float().cpu().numpy()[rows[:, 0], 0, rows[:, 1], :].astype(np.float64)
    lg = lse.cpu().numpy()[rows[:, 0], rows[:, 1]].astype(np.float64)
    check_o(og, o_ref, "decode_int4 full")
    check_lse(lg, l_ref, "decode_int4 full")
    assert (o.float() - o1.float()).abs().max().item() <= 1e-2
    assert (lse - l1).abs().max().item() <= 1e-4


PAGED = [
    # B, Hq, Hkv, D, P, seqlens, splits
    (3, 8, 2, 128, 64, [1000, 37, 640], 4),
    (4, 8, 2, 128, 16, [1, 15, 16, 17], 3),
    (3, 6, 2, 64, 32, [129, 64, 0], 7),
    (2, 16, 1, 128, 256, [300, 700], 2),
]


@pytest.mark.parametrize("case", PAGED)
def test_int4_paged_full_oracle(fa, case):
    B, Hq, Hkv, D, P, seqlens, splits = case
    w = synthetic.PagedDecodeWorkload("p4", 3, B, Hq, Hkv, D, P, 0, max(seqlens))
    q, kp, vp, ksp, vsp, bt, sl = synthetic.make_paged_decode_inputs(w, seqlens=seqlens, bits=4)
    o, lse = fa.fa_decode_int4_paged(to_dev_bf16(q), _dev(kp), _dev(vp), _dev(ksp), _dev(vsp),
                                     _dev(bt), _dev(sl), num_splits=splits, scale=w.scale)
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.decode_int4_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale)
    what = f"int4 paged P{P} lens{seqlens}"
    check_o(o_to_f64(o), o_ref, what)
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, what)


def test_int4_identity_pages_match_contiguous_bitwise(fa):
    import torch
    B, Hq, Hkv, S, D, P = 2, 16, 2, 1024, 128, 64
    wc = synthetic.Workload("i4p", 0, B, Hq, Hkv, 1, S, D, 1)
    q = synthetic.normal_bf16(81, wc.q_shape())
    k4, ks = synthetic.quantize_int4_per_token(synthetic.normal_bf16(82, wc.kv_shape()))
    v4, vs = synthetic.quantize_int4_per_token(synthetic.normal_bf16(83, wc.kv_shape()))
    npg = S // P
    kp = k4.reshape(B * npg, P, Hkv, D // 2)
    vp = v4.reshape(B * npg, P, Hkv, D // 2)
    ksp = ks.reshape(B, Hkv, npg, P).transpose(0, 2, 1, 3).reshape(B * npg, Hkv, P)
    vsp = vs.reshape(B, Hkv, npg, P).transpose(0, 2, 1, 3).reshape(B * npg, Hkv, P)
    bt = np.arange(B * npg, dtype=np.int32).reshape(B, npg)
    sl = np.full(B, S, dtype=np.int32)
    qd = to_dev_bf16(q)
    for splits in (1, 4):
        oc, lc = fa.fa_decode_int4(qd, _dev(k4), _dev(v4), _dev(ks), _dev(vs), num_splits=splits,
                                   scale=wc.scale)
        op, lp = fa.fa_decode_int4_paged(qd, _dev(kp), _dev(vp), _dev(ksp), _dev(vsp), _dev(bt),
                                         _dev(sl), num_splits=splits, scale=wc.scale)
        torch.cuda.synchronize()
        assert torch.equal(oc, op) and torch.equal(lc, lp), splits
    assert fa.fa_device_status() == 0
