"""Pins of the INT4 KV-cache pieces: the nibble unpacking (``oracle.unpack_int4``), the INT4
quantisation recipe, and the INT4 decode oracle.

The pages name INT4 next to INT8 as a KV-cache format used without decompression ("Flash
Attention on Ascend: three techniques", KV-compression section) and give no packing.  This
project's format: two 4-bit two's-complement codes per byte, dim 2i in the low nibble and dim
2i+1 in the high nibble, one fp32 scale per (token, KV head), codes in [-7, 7]."""
import numpy as np
import pytest
import torch

import oracle
import synthetic


def test_unpack_worked_bytes():
    packed = np.array([0x00, 0x7F, 0x80, 0x18, 0xF1, 0x99], dtype=np.uint8)
    want = [0, 0, -1, 7, 0, -8, -8, 1, 1, -1, -7, -7]
    assert oracle.unpack_int4(packed).tolist() == want


def test_unpack_matches_independent_packing():
    rng = np.random.default_rng(5)
    codes = rng.integers(-8, 8, size=(3, 7, 64), dtype=np.int64)
    # pack by arithmetic on the code values (no bit masks): v mod 16 is the nibble
    lo, hi = codes[..., 0::2] % 16, codes[..., 1::2] % 16
    packed = (lo + 16 * hi).astype(np.uint8)
    assert np.array_equal(oracle.unpack_int4(packed), codes.astype(np.int8))


def test_int4_recipe_bounds_and_round_trip():
    x = synthetic.normal_bf16(91, (2, 33, 3, 64))
    x[0, 5, 1, :] = 0  # an all-zero row: scale 0, codes 0
    packed, sc = synthetic.quantize_int4_per_token(x)
    assert packed.shape == (2, 33, 3, 32) and sc.shape == (2, 3, 33)
    codes = oracle.unpack_int4(packed)
    assert codes.min() >= -7 and codes.max() <= 7
    assert np.all(codes[0, 5, 1] == 0) and sc[0, 1, 5] == 0
    xf = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    deq = codes.astype(np.float64) * np.transpose(sc, (0, 2, 1))[..., None].astype(np.float64)
    err = np.abs(deq - xf)
    half = 0.5 * np.transpose(sc, (0, 2, 1))[..., None].astype(np.float64)
    assert np.all(err <= half * (1 + 1e-6) + 1e-12)
    # the largest magnitude of each row maps to +-7
    assert np.all(np.abs(codes).max(axis=-1)[sc.transpose(0, 2, 1) > 0] == 7)


def test_int4_recipe_torch_matches_numpy():
    x = synthetic.normal_bf16(92, (2, 40, 2, 128))
    p_np, s_np = synthetic.quantize_int4_per_token(x)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    p_t, s_t = synthetic.quantize_int4_per_token_torch(xt)
    assert np.array_equal(p_t.numpy(), p_np)
    assert np.array_equal(s_t.numpy(), s_np)


def test_int4_decode_one_key_closed_form():
    w = synthetic.Workload("i4", 0, 2, 4, 2, 1, 1, 64, 1)
    q, k4, v4, ks, vs = synthetic.make_decode_int4_inputs(w)
    o, lse = oracle.decode_int4(q, k4, v4, ks, vs, w.scale)
    vcodes = oracle.unpack_int4(v4)
    for b in range(2):
        for h in range(4):
            g = h // 2
            want = vcodes[b, 0, g].astype(np.float64) * np.float64(vs[b, g, 0])
            np.testing.assert_allclose(o[b, 0, h], want, rtol=1e-15, atol=1e-15)


def test_int4_decode_brute_force():
    w = synthetic.Workload("i4", 0, 2, 6, 3, 1, 77, 64, 1)
    q, k4, v4, ks, vs = synthetic.make_decode_int4_inputs(w)
    o, lse = oracle.decode_int4(q, k4, v4, ks, vs, w.scale, num_splits=3)
    # independent unpacking: nibble value n -> n - 16 * (n >= 8)
    def unpack(p):
        lo = (p % 16).astype(np.int64)
        hi = (p // 16).astype(np.int64)
        out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int64)
        out[..., 0::2] = lo - 16 * (lo >= 8)
        out[..., 1::2] = hi - 16 * (hi >= 8)
        return out
    K = unpack(k4) * np.transpose(ks, (0, 2, 1))[..., None].astype(np.float64)
    V = unpack(v4) * np.transpose(vs, (0, 2, 1))[..., None].astype(np.float64)
    qf = synthetic.bf16_bits_to_f32(q).astype(np.float64)
    for b in range(w.B):
        for h in range(w.Hq):
            g = h // 2
            s = (K[b, :, g] @ qf[b, 0, h]) * w.scale
            m = s.max()
            e = np.exp(s - m)
            np.testing.assert_allclose(o[b, 0, h], (e / e.sum()) @ V[b, :, g], atol=1e-12, rtol=0)
            np.testing.assert_allclose(lse[b, h], m + np.log(e.sum()), atol=1e-12, rtol=0)
