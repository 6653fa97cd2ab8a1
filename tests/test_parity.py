"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on identical seeded
inputs, plus invariants that must hold on the device."""
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


def run_and_check(fa, B, Hq, Hkv, Sq, Skv, D, causal, window, seed=0, scale=None):
    q = synthetic.normal_bf16(1000 + seed, (B, Sq, Hq, D))
    k = synthetic.normal_bf16(2000 + seed, (B, Skv, Hkv, D))
    v = synthetic.normal_bf16(3000 + seed, (B, Skv, Hkv, D))
    s = float(np.float32(1 / math.sqrt(D))) if scale is None else scale
    o, lse = fa.fa_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), causal=causal,
                       window=window, scale=s)
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.attn(q, k, v, s, causal, window)
    what = f"B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Skv{Skv} D{D} c{causal} w{window}"
    check_o(o_to_f64(o), o_ref, what)
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, what)


SMALL = [
    # B, Hq, Hkv, Sq, Skv, D, causal, window
    (1, 2, 2, 128, 128, 64, 0, 0),      # the tiny workload's shape
    (1, 2, 2, 300, 300, 128, 1, 0),     # several tiles, ragged tail
    (2, 4, 4, 300, 300, 128, 0, 0),
    (1, 4, 1, 517, 517, 64, 1, 0),      # G=4: 4 heads packed per tile
    (1, 8, 1, 260, 260, 128, 1, 0),     # G=8
    (1, 12, 2, 200, 200, 64, 1, 0),     # G=6: 2 heads packed, 3 packs per group
    (1, 32, 2, 150, 150, 128, 1, 0),    # G=16: 8 packed, 2 packs
    (1, 4, 2, 700, 700, 128, 1, 100),   # sliding window
    (1, 4, 2, 600, 600, 64, 1, 129),    # window edge across a key tile
    (1, 2, 2, 200, 450, 128, 1, 0),     # Sq < Skv (bottom-right causal)
    (1, 2, 2, 450, 200, 128, 1, 0),     # Sq > Skv: leading rows see nothing
    (1, 2, 1, 1, 1, 64, 0, 0),          # one token
    (2, 2, 2, 1, 300, 128, 1, 0),       # one query over many keys
    (1, 2, 2, 64, 1000, 128, 0, 0),     # non-causal, ragged keys
    (3, 3, 3, 257, 129, 64, 0, 0),
]


@pytest.mark.parametrize("case", SMALL)
def test_prefill_small_full_oracle(fa, case):
    run_and_check(fa, *case)


def test_prefill_tiny_workload(fa):
    w = synthetic.WORKLOADS["tiny"]
    q, k, v = synthetic.make_qkv(w)
    o, lse = fa.fa_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), causal=w.causal,
                       scale=w.scale)
    o_ref, l_ref = oracle.attn(q, k, v, w.scale, w.causal, w.window)
    check_o(o_to_f64(o), o_ref, "tiny")
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, "tiny")


@pytest.mark.parametrize("name", ["mha_causal", "gqa_causal", "gqa_sw512", "mqa_causal"])
def test_prefill_full_workload_sampled_rows(fa, name):
    import torch
    w = synthetic.WORKLOADS[name]
    q, k, v = synthetic.make_qkv_torch(w, "cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=w.causal, window=w.window, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    rows = synthetic.sample_rows(w.B, w.Hq, w.Sq, seed=w.seed(9), n_random=1500, window=w.window)
    qh, kh, vh = to_host_bits(q), to_host_bits(k), to_host_bits(v)
    o_ref, l_ref = oracle.attn_rows(qh, kh, vh, w.scale, w.causal, w.window, rows)
    og = o.float().cpu().numpy()
    lg = lse.cpu().numpy()
    o_got = og[rows[:, 0], rows[:, 2], rows[:, 1], :].astype(np.float64)
    l_got = lg[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
    check_o(o_got, o_ref, name)
    check_lse(l_got, l_ref, name)
    # properties that hold at any size: finite everywhere, LSE >= the row's max score bound
    assert torch.isfinite(o.float()).all()
    assert torch.isfinite(lse).all()


def test_constant_v_and_causal_row_zero(fa):
    import torch
    B, H, S, D = 1, 4, 300, 128
    q = to_dev_bf16(synthetic.normal_bf16(11, (B, S, H, D)))
    k = to_dev_bf16(synthetic.normal_bf16(12, (B, S, H, D)))
    v = torch.full((B, S, H, D), 0.8125, dtype=torch.bfloat16, device="cuda")
    o, _ = fa.fa_fwd(q, k, v, causal=True)
    assert (o.float() - 0.8125).abs().max().item() <= 2e-3
    v = to_dev_bf16(synthetic.normal_bf16(13, (B, S, H, D)))
    o, _ = fa.fa_fwd(q, k, v, causal=True)
    # row 0 sees only key 0: p = 1, so O[0] is V[0] exactly
    assert torch.equal(o[:, 0], v[:, 0])


def test_gqa_equals_mha_after_repeat(fa):
    import torch
    B, Hq, Hkv, S, D = 1, 16, 4, 333, 128
    q = to_dev_bf16(synthetic.normal_bf16(21, (B, S, Hq, D)))
    k = to_dev_bf16(synthetic.normal_bf16(22, (B, S, Hkv, D)))
    v = to_dev_bf16(synthetic.normal_bf16(23, (B, S, Hkv, D)))
    o1, l1 = fa.fa_fwd(q, k, v, causal=True, window=77)
    kr = k.repeat_interleave(Hq // Hkv, dim=2).contiguous()
    vr = v.repeat_interleave(Hq // Hkv, dim=2).contiguous()
    o2, l2 = fa.fa_fwd(q, kr, vr, causal=True, window=77)
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-5


def test_zero_query_lse_counts_visible_keys(fa):
    import torch
    B, H, S, D, W = 1, 2, 700, 64, 200
    q = torch.zeros((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    k = to_dev_bf16(synthetic.normal_bf16(31, (B, S, H, D)))
    v = to_dev_bf16(synthetic.normal_bf16(32, (B, S, H, D)))
    _, lse = fa.fa_fwd(q, k, v, causal=True, window=W)
    n = torch.minimum(torch.arange(S, device="cuda") + 1, torch.tensor(W, device="cuda"))
    assert (lse - torch.log(n.double()).float()).abs().max().item() <= 1e-5


# ------------------------------------------------------------------ decode (INT8 KV) ---------
def decode_case(fa, B, Hq, Hkv, Skv, D, splits, seed=0):
    import torch
    q = synthetic.normal_bf16(4000 + seed, (B, 1, Hq, D))
    kq, ks = synthetic.quantize_int8_per_token(synthetic.normal_bf16(5000 + seed, (B, Skv, Hkv, D)))
    vq, vs = synthetic.quantize_int8_per_token(synthetic.normal_bf16(6000 + seed, (B, Skv, Hkv, D)))
    s = float(np.float32(1 / math.sqrt(D)))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    o, lse = fa.fa_decode_int8(to_dev_bf16(q), dev(kq), dev(vq), dev(ks), dev(vs),
                               num_splits=splits, scale=s)
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.decode_int8(q, kq, vq, ks, vs, s, 1)
    what = f"decode B{B} Hq{Hq} Hkv{Hkv} Skv{Skv} D{D} splits{splits}"
    check_o(o_to_f64(o), o_ref, what)
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, what)


DECODE = [
    # B, Hq, Hkv, Skv, D, splits
    (2, 8, 2, 1000, 128, 1),
    (2, 8, 2, 1000, 128, 3),
    (2, 8, 2, 1000, 128, 16),
    (1, 4, 4, 777, 64, 5),          # MHA decode, D=64
    (2, 16, 2, 513, 128, 4),        # G=8
    (1, 16, 1, 300, 128, 2),        # G=16: two blocks of 8 heads
    (3, 6, 2, 129, 64, 7),          # G=3
    (1, 2, 1, 1, 128, 1),           # a single cached token
    (1, 8, 2, 5, 128, 16),          # more splits than keys: empty splits
]


@pytest.mark.parametrize("case", DECODE)
def test_decode_small_full_oracle(fa, case):
    decode_case(fa, *case)


def test_decode_full_workload_sampled(fa):
    import torch
    w = synthetic.WORKLOADS["decode_int8"]
    q, kq, vq, ks, vs = synthetic.make_decode_inputs_torch(w, "cuda")
    o, lse = fa.fa_decode_int8(q, kq, vq, ks, vs, num_splits=w.num_splits, scale=w.scale)
    o1, l1 = fa.fa_decode_int8(q, kq, vq, ks, vs, num_splits=1, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    raw = synthetic.splitmix64(w.seed(9), 0, 48)
    pairs = sorted({(int(r % np.uint64(w.B)), int((r >> np.uint64(20)) % np.uint64(w.Hq))) for r in raw}
                   | {(0, 0), (w.B - 1, w.Hq - 1)})
    rows = np.array(pairs, dtype=np.int64)
    qh = to_host_bits(q)
    o_ref, l_ref = oracle.decode_int8_rows(qh, kq.cpu().numpy(), vq.cpu().numpy(), ks.cpu().numpy(),
                                           vs.cpu().numpy(), w.scale, 1, rows)
    og = o.float().cpu().numpy()[rows[:, 0], 0, rows[:, 1], :].astype(np.float64)
    lg = lse.cpu().numpy()[rows[:, 0], rows[:, 1]].astype(np.float64)
    check_o(og, o_ref, "decode_int8 full")
    check_lse(lg, l_ref, "decode_int8 full")
    # split-invariance on the device: 16 splits vs 1 split over all (b, h)
    assert (o.float() - o1.float()).abs().max().item() <= 1e-2
    assert (lse - l1).abs().max().item() <= 1e-4


# ------------------------------------------------------------------ failure detection --------
def test_bounded_wait_reports_timeout(fa):
    import torch
    assert fa.fa_device_status() == 0
    assert fa.fa_selftest_bounded_wait(2000) == 0
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.STATUS["FA_ERR_TIMEOUT"]
    assert fa.fa_device_status() == 0  # cleared
    # the context is still usable
    run_and_check(fa, 1, 2, 2, 130, 130, 64, 1, 0)


def test_binding_raises_on_bad_arguments(fa):
    import torch
    q = torch.zeros((1, 8, 2, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd(q, q, q)
    assert e.value.status == fa.STATUS["FA_ERR_UNSUPPORTED"]
    q = torch.zeros((1, 8, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd(q, q, q, causal=False, window=4)
    assert e.value.status == fa.STATUS["FA_ERR_INVALID_ARG"]


def test_decode_equals_prefill_on_representable_kv(fa):
    # With power-of-two scales, code * scale is exact in bf16, so the INT8 decode of one query
    # must match the bf16 prefill kernel on the dequantised cache (Sq = 1, bottom-right causal).
    import torch
    B, Hq, Hkv, Skv, D = 2, 8, 2, 700, 128
    rng = np.random.default_rng(12)
    q = synthetic.normal_bf16(90, (B, 1, Hq, D))
    codes_k = rng.integers(-127, 128, size=(B, Skv, Hkv, D)).astype(np.int8)
    codes_v = rng.integers(-127, 128, size=(B, Skv, Hkv, D)).astype(np.int8)
    ks = (2.0 ** rng.integers(-9, -5, size=(B, Hkv, Skv))).astype(np.float32)
    vs = (2.0 ** rng.integers(-9, -5, size=(B, Hkv, Skv))).astype(np.float32)
    kf = codes_k.astype(np.float32) * np.transpose(ks, (0, 2, 1))[..., None]
    vf = codes_v.astype(np.float32) * np.transpose(vs, (0, 2, 1))[..., None]
    kb, vb = synthetic.f32_to_bf16_bits(kf), synthetic.f32_to_bf16_bits(vf)
    assert np.array_equal(synthetic.bf16_bits_to_f32(kb), kf)  # exact
    s = float(np.float32(1 / math.sqrt(D)))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    od, ld = fa.fa_decode_int8(to_dev_bf16(q), dev(codes_k), dev(codes_v), dev(ks), dev(vs),
                               num_splits=4, scale=s)
    op, lp = fa.fa_fwd(to_dev_bf16(q), to_dev_bf16(kb), to_dev_bf16(vb), causal=True, scale=s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    assert (od.float() - op.float()).abs().max().item() <= 2e-2
    assert (ld - lp[:, :, 0]).abs().max().item() <= 1e-3
