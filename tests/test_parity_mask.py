"""GPU parity of the forward pass with an additive mask tensor and with global tokens
(fa_fwd_ext through the binding's ``mask`` / ``n_global``) against the fp64 oracle."""
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


def _qkv(B, Hq, Hkv, Sq, Skv, D, seed):
    return (synthetic.normal_bf16(seed, (B, Sq, Hq, D)),
            synthetic.normal_bf16(seed + 1, (B, Skv, Hkv, D)),
            synthetic.normal_bf16(seed + 2, (B, Skv, Hkv, D)))


def _mask(kind, B, Hq, Sq, Skv, seed):
    rng = np.random.default_rng(seed)
    if kind == "bias11":
        return rng.normal(0, 1.5, size=(1, 1, Sq, Skv)).astype(np.float32)
    if kind == "bias1h":
        return rng.normal(0, 1.5, size=(1, Hq, Sq, Skv)).astype(np.float32)
    if kind == "biasb1":
        return rng.normal(0, 1.5, size=(B, 1, Sq, Skv)).astype(np.float32)
    if kind == "holes":
        m = rng.normal(0, 1.0, size=(1, Hq, Sq, Skv)).astype(np.float32)
        m[rng.random(m.shape) < 0.3] = -np.inf
        m[0, 0, 1, :] = -np.inf          # a row with no key
        return m
    if kind == "band":                   # the page's sliding window as a dense -inf mask
        i = np.arange(Sq)[:, None] + (Skv - Sq)
        j = np.arange(Skv)[None, :]
        keep = (j <= i) & (j > i - 64)
        return np.where(keep, 0.0, -np.inf).astype(np.float32)[None, None]
    raise ValueError(kind)


MASKED = [
    # B, Hq, Hkv, Sq, Skv, D, causal, window, mask kind
    (1, 2, 2, 200, 300, 128, 0, 0, "bias11"),
    (2, 4, 2, 130, 257, 128, 0, 0, "bias1h"),     # Skv % 4 != 0: scalar mask loads
    (2, 8, 2, 300, 300, 128, 1, 0, "biasb1"),     # causal + mask, GQA rows packed 4 per token
    (1, 4, 1, 256, 256, 64, 0, 0, "holes"),       # -inf holes and an empty row, D=64
    (1, 2, 1, 384, 384, 128, 0, 0, "band"),
    (1, 16, 1, 100, 100, 128, 1, 32, "bias1h"),   # window + mask, G=16
]


@pytest.mark.parametrize("case", MASKED)
def test_masked_forward_full_oracle(fa, case):
    import torch
    B, Hq, Hkv, Sq, Skv, D, causal, window, kind = case
    q, k, v = _qkv(B, Hq, Hkv, Sq, Skv, D, 700 + Sq)
    mask = _mask(kind, B, Hq, Sq, Skv, 7)
    s = float(np.float32(1 / math.sqrt(D)))
    o, lse = fa.fa_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), causal=causal,
                       window=window, scale=s, mask=torch.from_numpy(mask).cuda())
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.attn_ext(q, k, v, s, causal, window, 0, mask)
    what = f"mask {kind} B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Skv{Skv} D{D} c{causal} w{window}"
    check_o(o_to_f64(o), o_ref, what)
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, what)


def test_zero_mask_matches_unmasked_kernel(fa):
    import torch
    q, k, v = _qkv(2, 8, 2, 300, 300, 128, 901)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    o0, l0 = fa.fa_fwd(qd, kd, vd, causal=True)
    o1, l1 = fa.fa_fwd(qd, kd, vd, causal=True,
                       mask=torch.zeros((1, 1, 300, 300), dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert (o0.float() - o1.float()).abs().max().item() <= 2e-2
    assert (l0 - l1).abs().max().item() <= 1e-5


GLOBAL = [
    # B, Hq, Hkv, S, D, G, W
    (1, 2, 2, 512, 128, 16, 64),
    (2, 8, 2, 700, 128, 200, 100),     # global tiles and the band overlap; allq tiles
    (1, 4, 1, 1000, 64, 3, 32),        # D=64, a gap of skipped tiles
    (1, 16, 1, 640, 128, 130, 1),      # GQA 16:1, window of one key
    (2, 4, 4, 300, 128, 400, 50),      # every token global
]


@pytest.mark.parametrize("case", GLOBAL)
def test_global_local_full_oracle(fa, case):
    B, Hq, Hkv, S, D, G, W = case
    q, k, v = _qkv(B, Hq, Hkv, S, S, D, 800 + S)
    s = float(np.float32(1 / math.sqrt(D)))
    o, lse = fa.fa_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), causal=True, window=W,
                       scale=s, n_global=G)
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.attn_ext(q, k, v, s, 1, W, G)
    what = f"global G{G} W{W} B{B} Hq{Hq} Hkv{Hkv} S{S} D{D}"
    check_o(o_to_f64(o), o_ref, what)
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, what)


MASKED_GLOBAL = [
    # B, Hq, Hkv, S, D, global tokens, W, mask kind: the mask tensor and global + local
    # attention together (the key tiles between the global ones and the band are skipped, so the
    # mask staging follows the same gaps)
    (1, 4, 2, 700, 128, 150, 64, "bias1h"),
    (2, 2, 1, 1000, 64, 3, 32, "holes"),
]


@pytest.mark.parametrize("case", MASKED_GLOBAL)
def test_masked_global_local_full_oracle(fa, case):
    import torch
    B, Hq, Hkv, S, D, G, W, kind = case
    q, k, v = _qkv(B, Hq, Hkv, S, S, D, 850 + S)
    mask = _mask(kind, B, Hq, S, S, 11)
    s = float(np.float32(1 / math.sqrt(D)))
    o, lse = fa.fa_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), causal=True, window=W,
                       scale=s, n_global=G, mask=torch.from_numpy(mask).cuda())
    assert fa.fa_device_status() == 0
    o_ref, l_ref = oracle.attn_ext(q, k, v, s, 1, W, G, mask)
    what = f"mask {kind} + global G{G} W{W} B{B} Hq{Hq} Hkv{Hkv} S{S} D{D}"
    check_o(o_to_f64(o), o_ref, what)
    check_lse(lse.cpu().numpy().astype(np.float64), l_ref, what)


def test_global_local_full_size_sampled(fa):
    # the GQA sliding-window workload (B=3, Hq=32, Hkv=8, S=4096, W=512) with 64 global tokens
    import torch
    w = synthetic.WORKLOADS["gqa_sw512"]
    G = 64
    q, k, v = synthetic.make_qkv_torch(w, "cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=True, window=w.window, scale=w.scale, n_global=G)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    rows = synthetic.sample_rows(w.B, w.Hq, w.Sq, w.seed(31), 600, window=w.window)
    extra = np.array([(b, h, i) for b in range(w.B) for h in (0, 31) for i in (0, 63, 64, 65)],
                     dtype=np.int64)
    rows = np.unique(np.concatenate([rows, extra]), axis=0)
    o_ref, l_ref = oracle.attn_ext_rows(to_host_bits(q), to_host_bits(k), to_host_bits(v),
                                        w.scale, 1, w.window, G, None, rows)
    og = o.float().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]].astype(np.float64)
    lg = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
    check_o(og, o_ref, "gqa_sw512 + 64 global")
    check_lse(lg, l_ref, "gqa_sw512 + 64 global")


def test_masked_full_size_sampled(fa):
    # the MHA causal workload (B=2, H=32, S=4096) with a per-head additive bias (ALiBi-like
    # slopes, built on the host) on top of the causal rule
    import torch
    w = synthetic.WORKLOADS["mha_causal"]
    q, k, v = synthetic.make_qkv_torch(w, "cuda")
    slopes = 2.0 ** (-8.0 * np.arange(1, w.Hq + 1) / w.Hq)
    dist = (np.arange(w.Skv)[None, :] - np.arange(w.Sq)[:, None]).astype(np.float64)
    mask = (slopes[:, None, None] * np.minimum(dist, 0.0)[None]).astype(np.float32)[None]
    md = torch.from_numpy(mask).cuda()
    o, lse = fa.fa_fwd(q, k, v, causal=True, scale=w.scale, mask=md)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    rows = synthetic.sample_rows(w.B, w.Hq, w.Sq, w.seed(32), 400)
    o_ref, l_ref = oracle.attn_ext_rows(to_host_bits(q), to_host_bits(k), to_host_bits(v),
                                        w.scale, 1, 0, 0, mask, rows)
    og = o.float().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]].astype(np.float64)
    lg = lse.cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
    check_o(og, o_ref, "mha_causal + per-head bias")
    check_lse(lg, l_ref, "mha_causal + per-head bias")
