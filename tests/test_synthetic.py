"""Pins of the seeded input recipe shared by both sides."""
import numpy as np

import synthetic


def test_splitmix64_published_vectors():
    # Reference outputs of splitmix64 (Vigna's reference implementation) for state 1234567,
    # and the first output for state 0.
    got = [int(x) for x in synthetic.splitmix64(1234567, 0, 5)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]
    assert int(synthetic.splitmix64(0, 0, 1)[0]) == 0xE220A8397B1DCDAF
    # counter-based: any window of the stream equals the same slice of a longer draw
    assert np.array_equal(synthetic.splitmix64(7, 10, 5), synthetic.splitmix64(7, 0, 15)[10:])


def test_normal_moments_and_determinism():
    x = synthetic.normal_f64(99, 1_000_001)
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1) < 5e-3
    assert np.array_equal(x[:1001], synthetic.normal_f64(99, 1001))


def test_bf16_rounding_ties_to_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38], dtype=np.float32)
    bits = synthetic.f32_to_bf16_bits(vals)
    back = synthetic.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins;
    # 1 + 3*2^-8 ties between 1 + 2^-7 and 1 + 2^-6: even (1 + 2^-6) wins.
    assert back.tolist()[:4] == [1.0, 1.0, 1.0 + 2 ** -6, -2.5]


def test_int8_quantisation_recipe():
    x = np.zeros((1, 3, 2, 8), dtype=np.float32)
    x[0, 0, 0] = [127.0, -63.5, 0.5, 1.5, 2.5, -0.5, 0, 64.0]    # scale exactly 1
    x[0, 1, 1] = [-4.0, 2.0, 1.0, 0, 0, 0, 0, 0]                  # max at a negative value
    # x[0, 2, *] and x[0, 0, 1] are all zero -> scale 0, codes 0
    bits = synthetic.f32_to_bf16_bits(x)
    q, s = synthetic.quantize_int8_per_token(bits)
    assert q.dtype == np.int8 and s.dtype == np.float32 and s.shape == (1, 2, 3)
    assert s[0, 0, 0] == 1.0
    # round half to even: -63.5 -> -64, 0.5 -> 0, 1.5 -> 2, 2.5 -> 2, -0.5 -> -0
    assert q[0, 0, 0].tolist() == [127, -64, 0, 2, 2, 0, 0, 64]
    assert s[0, 1, 1] == np.float32(4.0) / np.float32(127.0)
    assert q[0, 1, 1, 0] == -127
    assert s[0, 0, 1] == 0 and np.all(q[0, 0, 1] == 0) and np.all(q[0, 2] == 0)


def test_workload_table():
    w = synthetic.WORKLOADS
    assert (w["mha_causal"].B, w["mha_causal"].Hq, w["mha_causal"].Sq, w["mha_causal"].D) == (2, 32, 4096, 128)
    assert w["gqa_causal"].Hq // w["gqa_causal"].Hkv == 4
    assert w["gqa_sw512"].window == 512
    assert (w["mqa_causal"].Hq, w["mqa_causal"].Hkv, w["mqa_causal"].D) == (232, 1, 64)
    d = w["decode_int8"]
    assert (d.B, d.Hq, d.Hkv, d.Sq, d.Skv, d.num_splits) == (16, 32, 8, 1, 32768, 16)
    assert w["tiny"].scale == 0.125


def test_torch_generator_matches_numpy_stream():
    import torch
    ints = synthetic.splitmix64_torch(1234567, 0, 5)
    assert [int(x) & 0xFFFFFFFFFFFFFFFF for x in ints] == [int(x) for x in synthetic.splitmix64(1234567, 0, 5)]
    a = synthetic.normal_bf16(777, (3, 1001))
    b = synthetic.normal_bf16_torch(777, (3, 1001), chunk=257).view(torch.int16).numpy().view(np.uint16)
    # same integer stream; fp64 transcendental functions may differ in the last bit
    assert np.mean(a != b) < 1e-3
    q1, s1 = synthetic.quantize_int8_per_token(a.reshape(1, 3, 7, 143))
    tq, ts = synthetic.quantize_int8_per_token_torch(
        torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).reshape(1, 3, 7, 143))
    assert np.array_equal(q1, tq.numpy()) and np.array_equal(s1, ts.numpy())
