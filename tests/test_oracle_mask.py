"""Pins of the oracle's additive-mask and global+local evaluation (``oracle.attn_ext``).

"FlashAttention variants: GQA, MQA, sparse attention" passes the sliding window as an additive
mask (-inf where a key is dropped) and describes global+local attention: a few global tokens
attend to, and are attended by, every token, the rest see their local window.  Its printed code
runs one attention over the global keys and one over the local keys and concatenates the outputs
along the sequence, which has the wrong number of rows; the two partial results of a query are
instead merged through their log-sum-exp.  Here that merge, built from the basic (separately
pinned) oracle, pins the fused global+local evaluation."""
import math

import numpy as np
import pytest

import oracle
import synthetic


def _qkv(B, Hq, Hkv, Sq, Skv, D, seed):
    return (synthetic.normal_bf16(seed, (B, Sq, Hq, D)),
            synthetic.normal_bf16(seed + 1, (B, Skv, Hkv, D)),
            synthetic.normal_bf16(seed + 2, (B, Skv, Hkv, D)))


def _f64(bits):
    return synthetic.bf16_bits_to_f32(bits).astype(np.float64)


def test_zero_mask_is_no_mask():
    q, k, v = _qkv(2, 4, 2, 70, 90, 64, 11)
    s = 0.125
    o0, l0 = oracle.attn(q, k, v, s, 1, 0)
    o1, l1 = oracle.attn_ext(q, k, v, s, 1, 0, 0, np.zeros((1, 1, 70, 90), np.float32))
    np.testing.assert_allclose(o1, o0, atol=1e-15, rtol=0)
    np.testing.assert_allclose(l1, l0, atol=1e-15, rtol=0)


@pytest.mark.parametrize("W", [1, 17, 64])
def test_band_mask_equals_window_rule(W):
    # the sliding window written as the page does: an additive -inf mask on a plain attention
    Sq = Skv = 100
    q, k, v = _qkv(1, 4, 1, Sq, Skv, 64, 21)
    i = np.arange(Sq)[:, None]
    j = np.arange(Skv)[None, :]
    keep = (j <= i) & (j > i - W)
    mask = np.where(keep, 0.0, -np.inf).astype(np.float32)[None, None]
    o0, l0 = oracle.attn(q, k, v, 0.125, 1, W)
    o1, l1 = oracle.attn_ext(q, k, v, 0.125, 0, 0, 0, mask)
    np.testing.assert_allclose(o1, o0, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l1, l0, atol=1e-13, rtol=0)


def test_constant_bias_shifts_lse_only():
    q, k, v = _qkv(2, 2, 2, 33, 47, 64, 31)
    o0, l0 = oracle.attn(q, k, v, 0.1, 0, 0)
    o1, l1 = oracle.attn_ext(q, k, v, 0.1, 0, 0, 0, np.full((1, 1, 33, 47), 2.5, np.float32))
    np.testing.assert_allclose(o1, o0, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l1, l0 + 2.5, atol=1e-12, rtol=0)


def test_per_head_bias_brute_force():
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 21, 37, 64
    q, k, v = _qkv(B, Hq, Hkv, Sq, Skv, D, 41)
    rng = np.random.default_rng(0)
    mask = rng.normal(0, 2, size=(1, Hq, Sq, Skv)).astype(np.float32)
    mask[0, 1, 3, :] = -np.inf           # a row with no key: O = 0, LSE = -inf
    mask[0, 2, :, 5:9] = -np.inf
    o, l = oracle.attn_ext(q, k, v, 0.2, 0, 0, 0, mask)
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    for b in range(B):
        for h in range(Hq):
            g = h // 2
            S = 0.2 * qf[b, :, h] @ kf[b, :, g].T + mask[0, h].astype(np.float64)
            for i in range(Sq):
                if np.all(np.isneginf(S[i])):
                    assert np.all(o[b, i, h] == 0) and np.isneginf(l[b, h, i])
                    continue
                m = S[i].max()
                e = np.exp(S[i] - m)
                np.testing.assert_allclose(o[b, i, h], (e / e.sum()) @ vf[b, :, g], atol=1e-12)
                np.testing.assert_allclose(l[b, h, i], m + np.log(e.sum()), atol=1e-12)


def test_batch_broadcast_of_mask():
    q, k, v = _qkv(3, 2, 1, 16, 16, 64, 51)
    rng = np.random.default_rng(1)
    m1 = rng.normal(size=(1, 1, 16, 16)).astype(np.float32)
    o1, l1 = oracle.attn_ext(q, k, v, 0.125, 0, 0, 0, m1)
    o3, l3 = oracle.attn_ext(q, k, v, 0.125, 0, 0, 0, np.repeat(np.repeat(m1, 3, 0), 2, 1))
    np.testing.assert_array_equal(o1, o3)
    np.testing.assert_array_equal(l1, l3)


def _merge(parts):
    """Merge partial (O, LSE) results of disjoint key sets through their log-sum-exp."""
    L = np.logaddexp.reduce([lp for _, lp in parts], axis=0)
    O = 0
    for op, lp in parts:
        w = np.where(np.isneginf(lp), 0.0, np.exp(lp - np.where(np.isneginf(L), 0.0, L)))
        O = O + w.transpose(0, 2, 1)[..., None] * op
    return O, L


@pytest.mark.parametrize("G,W", [(4, 16), (1, 1), (40, 8), (7, 100)])
def test_global_local_equals_lse_merge_of_two_passes(G, W):
    B, Hq, Hkv, S, D = 2, 4, 2, 96, 64
    q, k, v = _qkv(B, Hq, Hkv, S, S, D, 61)
    s = 0.125
    o, l = oracle.attn_ext(q, k, v, s, 1, W, G)
    # pass A: every query over the global keys [0, G), no mask
    oa, la = oracle.attn(q, np.ascontiguousarray(k[:, :G]), np.ascontiguousarray(v[:, :G]), s, 0, 0)
    # pass B: the local window over the other keys [G, S) (bottom-right alignment keeps key
    # positions: query i sees j in (i - W, i] with j >= G)
    ob, lb = oracle.attn(q, np.ascontiguousarray(k[:, G:]), np.ascontiguousarray(v[:, G:]), s, 1, W)
    om, lm = _merge([(oa, la), (ob, lb)])
    # global queries i < G see every key
    oc, lc = oracle.attn(np.ascontiguousarray(q[:, :G]), k, v, s, 0, 0)
    om[:, :G] = oc
    lm[:, :, :G] = lc
    np.testing.assert_allclose(o, om, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l, lm, atol=1e-12, rtol=0)


def test_global_local_brute_force_and_reductions():
    B, Hq, Hkv, S, D, G, W = 1, 2, 1, 40, 64, 3, 5
    q, k, v = _qkv(B, Hq, Hkv, S, S, D, 71)
    o, l = oracle.attn_ext(q, k, v, 0.125, 1, W, G)
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    vis = ((j <= i) & (j > i - W)) | (j < G) | (i < G)
    mask = np.where(vis, 0.0, -np.inf).astype(np.float32)[None, None]
    o2, l2 = oracle.attn_ext(q, k, v, 0.125, 0, 0, 0, mask)
    np.testing.assert_allclose(o, o2, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l, l2, atol=1e-13, rtol=0)
    # no global tokens: the plain window rule
    o3, l3 = oracle.attn_ext(q, k, v, 0.125, 1, W, 0)
    o4, l4 = oracle.attn(q, k, v, 0.125, 1, W)
    np.testing.assert_allclose(o3, o4, atol=1e-15, rtol=0)
    np.testing.assert_allclose(l3, l4, atol=1e-15, rtol=0)


@pytest.mark.parametrize("W", [1, 8, 50])
def test_printed_mask_code_is_window_w_plus_one(W):
    # the page builds tril(ones, 0) * triu(ones, -W): it keeps i - W <= j <= i, i.e. W + 1 keys,
    # which this project's rule reaches as window = W + 1 (its own reading keeps W keys)
    S = 64
    q, k, v = _qkv(1, 2, 1, S, S, 64, 81 + W)
    ones = np.ones((S, S))
    keep = np.tril(ones, 0) * np.triu(ones, -W)
    mask = np.where(keep > 0, 0.0, -np.inf).astype(np.float32)[None, None]
    o_page, l_page = oracle.attn_ext(q, k, v, 0.125, 0, 0, 0, mask)
    o_w1, l_w1 = oracle.attn(q, k, v, 0.125, 1, W + 1)
    np.testing.assert_allclose(o_page, o_w1, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l_page, l_w1, atol=1e-13, rtol=0)
    assert int(keep.sum()) == sum(min(i + 1, W + 1) for i in range(S))
