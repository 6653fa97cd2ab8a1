"""Pins of the paged / variable-length decode oracle (``oracle.decode_int8_paged``).

Paging only changes where key j of a sequence is stored ("Sparse attention and MLA operators in
ops-transformer", section 2.2: the KV cache stored in pages addressed through a block_table), and
a per-sequence length only changes how many keys a sequence has ("Flash Attention on Ascend: three
techniques", version section: sequences of different lengths in one batch).
So the paged oracle must reduce to the contiguous decode oracle (itself pinned against the
definition in test_oracle.py) when the pages are a plain reshape of a contiguous cache, must not
depend on where the pages sit in the pool, and must ignore everything past each length.
"""
import numpy as np
import pytest

import oracle
import synthetic


def _contiguous_case(B, Hq, Hkv, S, D, seed):
    w = synthetic.Workload("pg", 0, B, Hq, Hkv, 1, S, D, 1)
    q = synthetic.normal_bf16(seed, w.q_shape())
    kq, ks = synthetic.quantize_int8_per_token(synthetic.normal_bf16(seed + 1, w.kv_shape()))
    vq, vs = synthetic.quantize_int8_per_token(synthetic.normal_bf16(seed + 2, w.kv_shape()))
    return w, q, kq, vq, ks, vs


def _as_pages(kq, vq, ks, vs, P):
    """A contiguous cache [B, S, Hkv, D] viewed as pages: sequence b owns pages b*npg .. ."""
    B, S, Hkv, D = kq.shape
    npg = S // P
    kp = kq.reshape(B * npg, P, Hkv, D)
    vp = vq.reshape(B * npg, P, Hkv, D)
    ksp = ks.reshape(B, Hkv, npg, P).transpose(0, 2, 1, 3).reshape(B * npg, Hkv, P)
    vsp = vs.reshape(B, Hkv, npg, P).transpose(0, 2, 1, 3).reshape(B * npg, Hkv, P)
    bt = np.arange(B * npg, dtype=np.int32).reshape(B, npg)
    return (np.ascontiguousarray(kp), np.ascontiguousarray(vp), np.ascontiguousarray(ksp),
            np.ascontiguousarray(vsp), bt)


@pytest.mark.parametrize("B,Hq,Hkv,S,D,P", [(2, 4, 2, 64, 64, 16), (3, 8, 1, 96, 128, 32),
                                            (1, 6, 3, 128, 64, 64)])
def test_identity_pages_equal_contiguous_decode(B, Hq, Hkv, S, D, P):
    w, q, kq, vq, ks, vs = _contiguous_case(B, Hq, Hkv, S, D, 777 + S)
    kp, vp, ksp, vsp, bt = _as_pages(kq, vq, ks, vs, P)
    sl = np.full(B, S, dtype=np.int32)
    o_ref, l_ref = oracle.decode_int8(q, kq, vq, ks, vs, w.scale)
    o, l = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, l_ref, rtol=0, atol=1e-12)


def test_page_placement_does_not_matter():
    B, Hq, Hkv, S, D, P = 3, 8, 2, 128, 64, 16
    w, q, kq, vq, ks, vs = _contiguous_case(B, Hq, Hkv, S, D, 4242)
    kp, vp, ksp, vsp, bt = _as_pages(kq, vq, ks, vs, P)
    sl = np.array([128, 77, 5], dtype=np.int32)
    o0, l0 = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale)
    # move physical page i to slot perm[i] and rewrite the table accordingly
    n = kp.shape[0]
    perm = np.random.default_rng(3).permutation(n)
    kp2, vp2, ksp2, vsp2 = (np.empty_like(t) for t in (kp, vp, ksp, vsp))
    for src, dst in enumerate(perm):
        kp2[dst], vp2[dst], ksp2[dst], vsp2[dst] = kp[src], vp[src], ksp[src], vsp[src]
    bt2 = perm[bt].astype(np.int32)
    o1, l1 = oracle.decode_int8_paged(q, kp2, vp2, ksp2, vsp2, bt2, sl, w.scale)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


@pytest.mark.parametrize("L", [1, 15, 16, 17, 63, 100])
def test_length_truncates_to_the_first_keys(L):
    B, Hq, Hkv, S, D, P = 2, 4, 2, 128, 64, 16
    w, q, kq, vq, ks, vs = _contiguous_case(B, Hq, Hkv, S, D, 99)
    kp, vp, ksp, vsp, bt = _as_pages(kq, vq, ks, vs, P)
    sl = np.array([L, S], dtype=np.int32)
    o, l = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale)
    # sequence 0 alone, contiguous, with only its first L keys
    o_ref, l_ref = oracle.decode_int8(q[:1], kq[:1, :L].copy(), vq[:1, :L].copy(),
                                      ks[:1, :, :L].copy(), vs[:1, :, :L].copy(), w.scale)
    np.testing.assert_allclose(o[:1], o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l[:1], l_ref, rtol=0, atol=1e-12)
    # rows past the length, and table entries past the last page, are never read
    kp2, vp2, ksp2, vsp2 = kp.copy(), vp.copy(), ksp.copy(), vsp.copy()
    first_unused = L  # sequence 0 owns pages 0 .. S/P-1 of the identity table
    for j in range(first_unused, S):
        pg, r = j // P, j % P
        kp2[pg, r] = 127 - kp2[pg, r]
        vp2[pg, r] = -vp2[pg, r]
        ksp2[pg, :, r] *= 3.0
        vsp2[pg, :, r] *= 5.0
    bt2 = bt.copy()
    bt2[0, -(-L // P):] = -1
    o2, l2 = oracle.decode_int8_paged(q, kp2, vp2, ksp2, vsp2, bt2, sl, w.scale)
    assert np.array_equal(o2[:1], o[:1]) and np.array_equal(l2[:1], l[:1])


def test_empty_sequence_and_split_invariance():
    w = synthetic.PagedDecodeWorkload("pg", 0, 4, 8, 2, 64, 16, 0, 200)
    q, kp, vp, ksp, vsp, bt, sl = synthetic.make_paged_decode_inputs(
        w, seqlens=[0, 1, 37, 200])
    o1, l1 = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale, 1)
    assert np.all(o1[0] == 0) and np.all(np.isneginf(l1[0]))
    assert np.all(np.isfinite(l1[1:]))
    for ns in (2, 3, 16, 64, 300):
        o, l = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale, ns)
        np.testing.assert_allclose(o, o1, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l[1:], l1[1:], rtol=0, atol=1e-12)
        assert np.all(np.isneginf(l[0]))


def test_one_key_returns_its_value_row():
    # softmax over a single key is 1: O equals that key's dequantised V row exactly
    w = synthetic.PagedDecodeWorkload("pg", 0, 2, 4, 2, 64, 16, 1, 64)
    q, kp, vp, ksp, vsp, bt, sl = synthetic.make_paged_decode_inputs(w, seqlens=[1, 1])
    o, l = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale)
    for b in range(2):
        for h in range(4):
            g = h // 2
            pg = bt[b, 0]
            want = vp[pg, 0, g].astype(np.float64) * np.float64(vsp[pg, g, 0])
            np.testing.assert_allclose(o[b, 0, h], want, rtol=1e-15, atol=1e-15)


def test_brute_force_tiny_scattered():
    # scattered pages, GQA, ragged lengths: explicit gather + dequantise + softmax in numpy
    w = synthetic.PagedDecodeWorkload("pg", 0, 3, 6, 3, 64, 16, 1, 80)
    q, kp, vp, ksp, vsp, bt, sl = synthetic.make_paged_decode_inputs(w)
    o, l = oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, w.scale)
    qf = synthetic.bf16_bits_to_f32(q).astype(np.float64)
    G = w.Hq // w.Hkv
    for b in range(w.B):
        n = int(sl[b])
        for h in range(w.Hq):
            g = h // G
            K = np.stack([kp[bt[b, j // 16], j % 16, g].astype(np.float64)
                          * np.float64(ksp[bt[b, j // 16], g, j % 16]) for j in range(n)])
            V = np.stack([vp[bt[b, j // 16], j % 16, g].astype(np.float64)
                          * np.float64(vsp[bt[b, j // 16], g, j % 16]) for j in range(n)])
            s = (K @ qf[b, 0, h]) * w.scale
            m = s.max()
            e = np.exp(s - m)
            np.testing.assert_allclose(o[b, 0, h], (e / e.sum()) @ V, rtol=0, atol=1e-12)
            np.testing.assert_allclose(l[b, h], m + np.log(e.sum()), rtol=0, atol=1e-12)


def test_rejects_bad_tables():
    w = synthetic.PagedDecodeWorkload("pg", 0, 2, 4, 2, 64, 16, 1, 64)
    q, kp, vp, ksp, vsp, bt, sl = synthetic.make_paged_decode_inputs(w, seqlens=[40, 64])
    bad = bt.copy()
    bad[0, 1] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bad, sl, w.scale)
    with pytest.raises(ValueError):
        oracle.decode_int8_paged(q, kp, vp, ksp, vsp, bt, np.array([65, 1], np.int32), w.scale)


def test_paged_layout_recipe():
    w = synthetic.PAGED_WORKLOADS["decode_int8_paged"]
    sl, bt, num_pages = synthetic.paged_layout(w)
    assert sl.dtype == np.int32 and sl.min() >= 1 and sl.max() <= w.max_len
    npg = -(-sl.astype(np.int64) // w.page_size)
    assert num_pages == npg.sum()
    used = np.concatenate([bt[b, :npg[b]] for b in range(w.B)])
    # every physical page is owned by exactly one (sequence, slot)
    assert np.array_equal(np.sort(used), np.arange(num_pages))
    for b in range(w.B):
        assert np.all(bt[b, npg[b]:] == -1)
    # the pages are scattered, not handed out in order
    assert not np.array_equal(used, np.arange(num_pages))
