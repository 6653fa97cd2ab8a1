"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

* closed forms (Q = 0 gives LSE = ln(number of visible keys) and O = mean of those V rows;
  constant V returns that constant; causal row 0 returns V[0]);
* invariants (probability rows sum to 1 and vanish on masked keys; the tiled online softmax
  agrees with the full score matrix for every block size; GQA equals MHA after an explicit
  repeat of the KV heads);
* a library routine (torch's scaled_dot_product_attention in float64 on the CPU, masks built
  here from the readings of the pages);
* a worked 2x2 example computed by hand;
* the pages' own connection counts (tests/golden/page_counts.json).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def visible_range(i, Sq, Skv, causal, window):
    """Visible keys of row i written out from the readings: bottom-right causal alignment,
    a window of W keys that includes the query's own position."""
    ip = i + Skv - Sq
    hi = min(ip, Skv - 1) if causal else Skv - 1
    lo = max(0, ip - window + 1) if window > 0 else 0
    return lo, hi  # inclusive; empty if hi < lo


CASES = [
    # B, Hq, Hkv, Sq, Skv, D, causal, window
    (1, 2, 2, 1, 1, 4, 0, 0),
    (2, 4, 2, 17, 17, 8, 1, 0),
    (1, 4, 1, 33, 33, 8, 1, 5),
    (2, 6, 3, 20, 45, 8, 1, 0),
    (1, 2, 2, 45, 20, 8, 1, 0),   # Sq > Skv: leading rows see nothing
    (1, 3, 1, 64, 64, 16, 0, 0),
    (1, 2, 1, 50, 70, 8, 1, 9),
]


@pytest.mark.parametrize("case", CASES)
def test_brute_tiled_rows_agree(case):
    B, Hq, Hkv, Sq, Skv, D, causal, window = case
    q, k, v = rand((B, Sq, Hq, D), 1), rand((B, Skv, Hkv, D), 2), rand((B, Skv, Hkv, D), 3)
    s = 1 / math.sqrt(D)
    ob, lb = oracle.attn_brute(q, k, v, s, causal, window)
    orow, lrow = oracle.attn(q, k, v, s, causal, window)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lrow))
    assert np.max(np.abs(ob - orow)) <= 1e-12
    assert np.max(np.abs(lb[fin] - lrow[fin])) <= 1e-12
    for tile in sorted({1, 7, 128, max(Sq, Skv)}):
        ot, lt = oracle.attn_tiled(q, k, v, s, causal, window, tile)
        assert np.array_equal(fin, np.isfinite(lt))
        assert np.max(np.abs(ob - ot)) <= 1e-12, tile
        assert np.max(np.abs(lb[fin] - lt[fin])) <= 1e-12, tile
    # rows that see no key: O = 0, LSE = -inf
    for b in range(B):
        for h in range(Hq):
            for i in range(Sq):
                lo, hi = visible_range(i, Sq, Skv, causal, window)
                if hi < lo:
                    assert lb[b, h, i] == -np.inf
                    assert np.all(ob[b, i, h] == 0)


@pytest.mark.parametrize("case", CASES)
def test_zero_query_closed_form(case):
    """Q = 0: every visible score is 0, so LSE = ln(n_i) and O_i = mean of the visible V rows."""
    B, Hq, Hkv, Sq, Skv, D, causal, window = case
    q = np.zeros((B, Sq, Hq, D))
    k, v = rand((B, Skv, Hkv, D), 4), rand((B, Skv, Hkv, D), 5)
    o, lse = oracle.attn(q, k, v, 0.3, causal, window)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            for i in range(Sq):
                lo, hi = visible_range(i, Sq, Skv, causal, window)
                if hi < lo:
                    assert lse[b, h, i] == -np.inf
                    continue
                n = hi - lo + 1
                assert abs(lse[b, h, i] - math.log(n)) <= 1e-13
                mean = v[b, lo:hi + 1, h // G, :].mean(axis=0)
                assert np.max(np.abs(o[b, i, h] - mean)) <= 1e-13


def test_probability_rows():
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 40, 40, 8
    q, k, v = rand((B, Sq, Hq, D), 6), rand((B, Skv, Hkv, D), 7), rand((B, Skv, Hkv, D), 8)
    for causal, window in [(0, 0), (1, 0), (1, 7)]:
        _, _, p = oracle.attn_brute(q, k, v, 0.5, causal, window, want_probs=True)
        assert np.max(np.abs(p.sum(-1) - 1)) <= 1e-12
        for i in range(Sq):
            lo, hi = visible_range(i, Sq, Skv, causal, window)
            assert np.all(p[:, :, i, :lo] == 0) and np.all(p[:, :, i, hi + 1:] == 0)
            assert np.all(p[:, :, i, lo:hi + 1] > 0)


def test_constant_v_and_causal_row_zero():
    B, Hq, Hkv, S, D = 2, 4, 2, 50, 16
    q, k = rand((B, S, Hq, D), 9), rand((B, S, Hkv, D), 10)
    v = np.full((B, S, Hkv, D), 0.8125)
    o, _ = oracle.attn(q, k, v, 0.25, 1, 0)
    assert np.max(np.abs(o - 0.8125)) <= 1e-14
    v = rand((B, S, Hkv, D), 11)
    o, lse = oracle.attn(q, k, v, 0.25, 1, 0)
    for h in range(Hq):
        assert np.array_equal(o[:, 0, h], v[:, 0, h // (Hq // Hkv)])
    # row 0 sees one key: LSE is that single scaled score
    s0 = 0.25 * np.einsum("bhd,bhd->bh", q[:, 0], np.repeat(k[:, 0], Hq // Hkv, axis=1))
    assert np.max(np.abs(lse[:, :, 0] - s0)) <= 1e-13


def test_gqa_equals_mha_after_repeat():
    B, Hq, Hkv, S, D = 2, 8, 2, 30, 8
    q, k, v = rand((B, S, Hq, D), 12), rand((B, S, Hkv, D), 13), rand((B, S, Hkv, D), 14)
    G = Hq // Hkv
    o1, l1 = oracle.attn(q, k, v, 0.3, 1, 6)
    o2, l2 = oracle.attn(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), 0.3, 1, 6)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def sdpa_reference(q, k, v, scale, causal, window):
    """torch SDPA in float64 on the CPU with an explicit boolean mask (True = visible)."""
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    mask = torch.zeros(Sq, Skv, dtype=torch.bool)
    for i in range(Sq):
        lo, hi = visible_range(i, Sq, Skv, causal, window)
        if hi >= lo:
            mask[i, lo:hi + 1] = True
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(np.repeat(k, G, axis=2)).permute(0, 2, 1, 3)
    tv = torch.from_numpy(np.repeat(v, G, axis=2)).permute(0, 2, 1, 3)
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    return out.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("case", [c for c in CASES if c[3] <= c[4]])
def test_matches_torch_sdpa_float64(case):
    B, Hq, Hkv, Sq, Skv, D, causal, window = case
    q, k, v = rand((B, Sq, Hq, D), 15), rand((B, Skv, Hkv, D), 16), rand((B, Skv, Hkv, D), 17)
    s = 0.37
    o, _ = oracle.attn(q, k, v, s, causal, window)
    ref = sdpa_reference(q, k, v, s, causal, window)
    assert np.max(np.abs(o - ref)) <= 1e-12


def test_worked_two_by_two():
    """q = k = I (D=2), v = [[1,2],[3,4]], scale 1, no mask.
    Row 0 scores (1, 0): p = (e, 1)/(e+1); row 1 scores (0, 1): p = (1, e)/(e+1)."""
    e = math.e
    q = np.eye(2).reshape(1, 2, 1, 2)
    k = np.eye(2).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 2, 1, 2)
    o, lse = oracle.attn(q, k, v, 1.0, 0, 0)
    want = np.array([[(e + 3) / (e + 1), (2 * e + 4) / (e + 1)],
                     [(1 + 3 * e) / (e + 1), (2 + 4 * e) / (e + 1)]])
    assert np.max(np.abs(o[0, :, 0, :] - want)) <= 1e-15
    assert np.max(np.abs(lse[0, 0] - math.log(e + 1))) <= 1e-15
    # causal: row 0 sees only key 0 -> v[0]; row 1 unchanged
    o, lse = oracle.attn(q, k, v, 1.0, 1, 0)
    assert np.array_equal(o[0, 0, 0], [1.0, 2.0])
    assert abs(lse[0, 0, 0] - 1.0) <= 1e-15


def test_bf16_path_matches_widened_f64():
    B, Hq, Hkv, S, D = 1, 4, 2, 40, 64
    qb = synthetic.normal_bf16(101, (B, S, Hq, D))
    kb = synthetic.normal_bf16(102, (B, S, Hkv, D))
    vb = synthetic.normal_bf16(103, (B, S, Hkv, D))
    w = lambda a: synthetic.bf16_bits_to_f32(a).astype(np.float64)
    o1, l1 = oracle.attn(qb, kb, vb, 0.125, 1, 9)
    o2, l2 = oracle.attn(w(qb), w(kb), w(vb), 0.125, 1, 9)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_page_connection_counts():
    """The pages count N^2 = 16,777,216 connections for full attention and N*W = 2,097,152 for
    a W=512 window at N=4096.  With Q = 0 the oracle's LSE is ln(visible keys), so
    sum(exp(LSE)) counts the visible pairs of its masks."""
    g = json.load(open(os.path.join(GOLDEN, "page_counts.json")))
    N = g["full_attention_connections"]["N"]
    W = g["window_connections_prose"]["W"]
    q = np.zeros((1, N, 1, 1))
    k = np.zeros((1, N, 1, 1))
    v = np.zeros((1, N, 1, 1))
    _, l_full = oracle.attn(q, k, v, 1.0, 0, 0)
    assert round(float(np.exp(l_full).sum())) == g["full_attention_connections"]["value"]
    _, l_win = oracle.attn(q, k, v, 1.0, 1, W)
    n = np.rint(np.exp(l_win[0, 0])).astype(np.int64)
    # every row past the first W-1 sees exactly its nearest W tokens (itself included)
    assert np.all(n[W - 1:] == W)
    # the page's N*W count ignores that the first W-1 rows have fewer predecessors
    assert int(n.sum()) == g["window_connections_prose"]["value"] - W * (W - 1) // 2
    saving = 100 * (1 - g["window_connections_prose"]["value"] / g["full_attention_connections"]["value"])
    assert saving == g["window_saving_percent"]["value"]
    assert N * N * 4 == g["score_matrix_bytes_fp32_4096"]["value_mib"] * 2 ** 20


def _dequant(codes, scales):
    # codes [B,S,H,D] int8, scales [B,H,S] fp32 -> fp64 [B,S,H,D]
    return codes.astype(np.float64) * np.transpose(scales, (0, 2, 1))[..., None].astype(np.float64)


def test_decode_split_merge_and_definition():
    B, Hq, Hkv, Skv, D = 2, 8, 2, 300, 32
    qb = synthetic.normal_bf16(201, (B, 1, Hq, D))
    kq, ks = synthetic.quantize_int8_per_token(synthetic.normal_bf16(202, (B, Skv, Hkv, D)))
    vq, vs = synthetic.quantize_int8_per_token(synthetic.normal_bf16(203, (B, Skv, Hkv, D)))
    s = 1 / math.sqrt(D)
    o1, l1 = oracle.decode_int8(qb, kq, vq, ks, vs, s, 1)
    for splits in (2, 7, 16, 300, 512):  # 512 > Skv: trailing splits are empty
        o2, l2 = oracle.decode_int8(qb, kq, vq, ks, vs, s, splits)
        assert np.max(np.abs(o1 - o2)) <= 1e-12 and np.max(np.abs(l1 - l2)) <= 1e-12
    qd = synthetic.bf16_bits_to_f32(qb).astype(np.float64)
    o3, l3 = oracle.attn(qd, _dequant(kq, ks), _dequant(vq, vs), s, 1, 0)
    assert np.max(np.abs(o1 - o3)) <= 1e-13 and np.max(np.abs(l1 - l3[:, :, 0])) <= 1e-13
