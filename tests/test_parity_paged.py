"""GPU parity of the paged, variable-length INT8 decode (fa_decode_int8_paged) against the fp64
oracle, plus device invariants: identity paging reproduces the contiguous kernel bit for bit,
lengths changed in device memory take effect in a captured CUDA graph, and out-of-range page ids
or lengths are reported through the device status word without any access outside the pool."""
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


def _inputs(B, Hq, Hkv, D, P, seqlens, index=1):
    max_len = max(max(seqlens), 1)
    w = synthetic.PagedDecodeWorkload("paged", index, B, Hq, Hkv, D, P, 0, max_len)
    return w, synthetic.make_paged_decode_inputs(w, seqlens=seqlens)


def _run(fa, w, host, splits):
    q, kp, vp, ksp, vsp, bt, sl = host
    return fa.fa_decode_int8_paged(to_dev_bf16(q), _dev(kp), _dev(vp), _dev(ksp), _dev(vsp),
                                   _dev(bt), _dev(sl), num_splits=splits, scale=w.scale)


PAGED = [
    # B, Hq, Hkv, D, P, seqlens, splits
    (3, 8, 2, 128, 64, [1000, 37, 640], 4),
    (3, 8, 2, 128, 64, [1000, 37, 640], 1),
    (4, 8, 2, 128, 16, [1, 15, 16, 17], 3),        # tails around one 16-token group
    (2, 16, 2, 128, 32, [513, 96], 16),            # G = 8, many splits
    (2, 16, 1, 128, 128, [300, 129], 2),           # G = 16: two blocks of 8 heads
    (3, 6, 2, 64, 64, [129, 64, 63], 7),           # D = 64, G = 3
    (2, 4, 4, 64, 256, [777, 256], 5),             # MHA, large pages
    (4, 8, 2, 128, 64, [0, 5, 0, 70], 4),          # empty sequences: O = 0, LSE = -inf
    (1, 8, 2, 128, 16, [5], 16),                   # more splits than groups
    # lengths ranked on the device: equal lengths (ties by index), ascending order
    (6, 8, 2, 128, 16, [48, 200, 48, 7, 200, 48], 3),
    (5, 4, 1, 64, 16, [10, 20, 30, 40, 50], 2),
    # more sequences than the kernel ranks (one per thread): grid order is kept
    (130, 4, 1, 64, 16, [(7 * x) % 50 for x in range(130)], 2),
]


@pytest.mark.parametrize("case", PAGED)
def test_paged_decode_full_oracle(fa, case):
    B, Hq, Hkv, D, P, seqlens, splits = case
    w, host = _inputs(B, Hq, Hkv, D, P, seqlens)
    o, lse = _run(fa, w, host, splits)
    assert fa.fa_device_status() == 0
    q, kp, vp, ksp, vsp, bt, sl = host
    o_ref, l_ref = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale, 1)
    what = f"paged B{B} Hq{Hq} Hkv{Hkv} D{D} P{P} lens{seqlens} splits{splits}"
    og = o_to_f64(o)
    check_o(og, o_ref, what)
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, what)
    for b, n in enumerate(seqlens):
        if n == 0:
            assert np.all(og[b] == 0)


def test_identity_pages_match_contiguous_kernel_bitwise(fa):
    # a contiguous cache viewed as pages, one split (and splits whose chunks are multiples of 16):
    # the paged kernel runs exactly the contiguous kernel's arithmetic
    import torch
    B, Hq, Hkv, S, D, P = 2, 16, 2, 1024, 128, 64
    wc = synthetic.Workload("idp", 0, B, Hq, Hkv, 1, S, D, 1)
    q = synthetic.normal_bf16(71, wc.q_shape())
    kq, ks = synthetic.quantize_int8_per_token(synthetic.normal_bf16(72, wc.kv_shape()))
    vq, vs = synthetic.quantize_int8_per_token(synthetic.normal_bf16(73, wc.kv_shape()))
    npg = S // P
    kp = kq.reshape(B * npg, P, Hkv, D)
    vp = vq.reshape(B * npg, P, Hkv, D)
    ksp = ks.reshape(B, Hkv, npg, P).transpose(0, 2, 1, 3).reshape(B * npg, Hkv, P)
    vsp = vs.reshape(B, Hkv, npg, P).transpose(0, 2, 1, 3).reshape(B * npg, Hkv, P)
    bt = np.arange(B * npg, dtype=np.int32).reshape(B, npg)
    sl = np.full(B, S, dtype=np.int32)
    qd = to_dev_bf16(q)
    for splits in (1, 4, 16):
        oc, lc = fa.fa_decode_int8(qd, _dev(kq), _dev(vq), _dev(ks), _dev(vs), num_splits=splits,
                                   scale=wc.scale)
        op, lp = fa.fa_decode_int8_paged(qd, _dev(kp), _dev(vp), _dev(ksp), _dev(vsp), _dev(bt),
                                         _dev(sl), num_splits=splits, scale=wc.scale)
        torch.cuda.synchronize()
        assert torch.equal(oc, op), splits
        assert torch.equal(lc, lp), splits
    assert fa.fa_device_status() == 0


def test_full_paged_workload_all_rows(fa):
    import torch
    w = synthetic.PAGED_WORKLOADS["decode_int8_paged"]
    q, kp, vp, ksp, vsp, bt, sl = synthetic.make_paged_decode_inputs_torch(w, "cuda")
    o, lse = fa.fa_decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, num_splits=w.num_splits,
                                     scale=w.scale)
    o1, l1 = fa.fa_decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, num_splits=1, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.decode_int8_paged(to_host_bits(q), kp.cpu().numpy(), vp.cpu().numpy(),
                                            ksp.cpu().numpy(), vsp.cpu().numpy(),
                                            bt.cpu().numpy(), sl.cpu().numpy(), w.scale, 1)
    check_o(o_to_f64(o), o_ref, "decode_int8_paged full")
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, "decode_int8_paged full")
    assert (o.float() - o1.float()).abs().max().item() <= 1e-2
    assert (lse - l1).abs().max().item() <= 1e-4


def test_lengths_in_device_memory_drive_a_captured_graph(fa):
    # the lengths are read on the device, so one captured graph serves every step of a
    # generation loop: rewrite them in place and replay
    import torch
    B, Hq, Hkv, D, P = 3, 8, 2, 128, 64
    w, host = _inputs(B, Hq, Hkv, D, P, [640, 640, 640], index=2)
    q, kp, vp, ksp, vsp, bt, sl = host
    dq, dk, dv, dks, dvs, dbt = (to_dev_bf16(q), _dev(kp), _dev(vp), _dev(ksp), _dev(vsp),
                                 _dev(bt))
    dsl = _dev(np.array([10, 20, 30], dtype=np.int32))
    o = torch.empty_like(dq)
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_decode_int8_workspace_bytes(B, Hq, D, 4), dtype=torch.uint8,
                     device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fa.fa_decode_int8_paged(dq, dk, dv, dks, dvs, dbt, dsl, num_splits=4, scale=w.scale,
                                o=o, lse=lse, workspace=ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fa.fa_decode_int8_paged(dq, dk, dv, dks, dvs, dbt, dsl, num_splits=4, scale=w.scale,
                                o=o, lse=lse, workspace=ws, stream=torch.cuda.current_stream())
    for lens in ([10, 20, 30], [1, 639, 64], [640, 0, 333]):
        dsl.copy_(torch.tensor(lens, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        o_ref, l_ref = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt,
                                                np.array(lens, np.int32), w.scale, 1)
        check_o(o_to_f64(o), o_ref, f"graph lens {lens}")
        check_lse(lse.cpu().numpy().astype(np.float64), l_ref, f"graph lens {lens}")
    del g
    assert fa.fa_device_status() == 0


def test_out_of_range_page_or_length_is_reported(fa):
    # the kernel range-checks every page id and length it reads; a bad one is replaced by a
    # valid one (no access leaves the pool) and reported by fa_device_status
    import torch
    B, Hq, Hkv, D, P = 2, 8, 2, 128, 64
    w, host = _inputs(B, Hq, Hkv, D, P, [200, 100], index=3)
    q, kp, vp, ksp, vsp, bt, sl = host
    args = [to_dev_bf16(q), _dev(kp), _dev(vp), _dev(ksp), _dev(vsp)]
    assert fa.fa_device_status() == 0
    bad_bt = bt.copy()
    bad_bt[0, 1] = kp.shape[0] + 5
    fa.fa_decode_int8_paged(*args, _dev(bad_bt), _dev(sl), num_splits=2, scale=w.scale)
    assert fa.fa_device_status() == fa.STATUS["FA_ERR_DEVICE_INDEX"]
    bad_bt[0, 1] = -3
    fa.fa_decode_int8_paged(*args, _dev(bad_bt), _dev(sl), num_splits=2, scale=w.scale)
    assert fa.fa_device_status() == fa.STATUS["FA_ERR_DEVICE_INDEX"]
    too_long = np.array([bt.shape[1] * P + 1, 100], dtype=np.int32)
    fa.fa_decode_int8_paged(*args, _dev(bt), _dev(too_long), num_splits=2, scale=w.scale)
    assert fa.fa_device_status() == fa.STATUS["FA_ERR_DEVICE_INDEX"]
    negative = np.array([-7, 100], dtype=np.int32)
    fa.fa_decode_int8_paged(*args, _dev(bt), _dev(negative), num_splits=2, scale=w.scale)
    assert fa.fa_device_status() == fa.STATUS["FA_ERR_DEVICE_INDEX"]
    # the context is intact and a good call is clean again
    o, lse = fa.fa_decode_int8_paged(*args, _dev(bt), _dev(sl), num_splits=2, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale, 1)
    check_o(o_to_f64(o), o_ref, "after bad indices")
