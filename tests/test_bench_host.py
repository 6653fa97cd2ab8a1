"""Host logic of bench.py: the algorithmic work figures that every throughput and roofline
fraction divides by, checked against closed forms and brute-force counts written here
independently, plus the whole-job throughput rule."""
import numpy as np

import bench
import synthetic


def _pairs_brute(Sq, Skv, causal, window, n_global=0):
    """Visible (query, key) pairs counted one by one: bottom-right causal alignment, a window of
    W keys ending at the query's own position, and tokens below n_global seen by and seeing
    everyone ("FlashAttention variants: GQA, MQA, sparse attention", sliding-window and
    global+local sections)."""
    n = 0
    for i in range(Sq):
        ip = i + (Skv - Sq)
        for j in range(Skv):
            ok = (not causal or j <= ip) and (window <= 0 or j > ip - window)
            if n_global and (j < n_global or i < n_global):
                ok = True
            n += ok
    return n


def test_prefill_flops_closed_forms():
    # causal, Sq = Skv = S: S (S + 1) / 2 visible pairs per (b, h); 4 D flops per pair
    for name in ("mha_causal", "gqa_causal", "mqa_causal"):
        w = synthetic.WORKLOADS[name]
        S = w.Sq
        assert bench.prefill_flops(w) == S * (S + 1) // 2 * 4 * w.D * w.B * w.Hq
    assert bench.prefill_flops(synthetic.WORKLOADS["mha_causal"]) == 274_945_015_808
    assert bench.prefill_flops(synthetic.WORKLOADS["gqa_causal"]) == 137_472_507_904
    assert bench.prefill_flops(synthetic.WORKLOADS["mqa_causal"]) == 124_614_868_992
    # window of W keys including self: N W - W (W - 1) / 2 pairs per (b, h)
    w = synthetic.WORKLOADS["gqa_sw512"]
    W, N = w.window, w.Sq
    assert bench.prefill_flops(w) == (N * W - W * (W - 1) // 2) * 4 * w.D * w.B * w.Hq
    assert bench.prefill_flops(w) == 32_216_449_024


def test_prefill_flops_match_brute_force_on_small_shapes():
    for Sq, Skv, causal, window in [(37, 37, 1, 0), (20, 50, 1, 0), (50, 20, 1, 0),
                                    (64, 64, 1, 9), (33, 70, 1, 16), (17, 40, 0, 0)]:
        w = synthetic.Workload("t", 0, 2, 3, 1, Sq, Skv, 64, causal, window)
        assert bench.prefill_flops(w) == _pairs_brute(Sq, Skv, causal, window) * 4 * 64 * 2 * 3


def test_global_local_flops_match_brute_force():
    for S, window, G in [(64, 9, 5), (100, 16, 0), (100, 16, 40), (128, 128, 7), (50, 1, 3)]:
        w = synthetic.Workload("t", 0, 1, 2, 1, S, S, 64, 1, window)
        want = _pairs_brute(S, S, 1, window, G) * 4 * 64 * 1 * 2
        assert bench.global_local_flops(w, G) == want, (S, window, G)


def test_decode_bytes():
    w = synthetic.WORKLOADS["decode_int8"]
    assert bench.decode_bytes(w) == 1_107_560_448
    # INT4: half the code bytes of INT8 for the same keys, the same scales, q, o and LSE
    w4 = synthetic.WORKLOADS["decode_int4"]
    codes8 = 2 * w4.B * w4.Skv * w4.Hkv * w4.D
    assert bench.int4_decode_bytes(w4) == bench.decode_bytes(w4) - codes8 // 2


def test_paged_decode_bytes_brute_force():
    w = synthetic.PagedDecodeWorkload("t", 0, 3, 8, 2, 128, 16, 1, 100)
    sl = np.array([1, 16, 37], dtype=np.int32)
    n = 0
    for L in sl:
        n += int(L) * w.Hkv * (2 * w.D + 2 * 4)  # K and V code rows, their two fp32 scales
        n += 4 * (-(-int(L) // w.page_size))       # one table entry per page in use
        n += 4                                     # the length
    n += w.B * w.Hq * (2 * w.D * 2 + 4)            # q in, o out (bf16), LSE (fp32)
    assert bench.paged_decode_bytes(w, sl) == n


def test_weak_scaling_throughput():
    # 4 ranks, 10 steps of 3e9 units each, slowest rank 20 ms: 4 * 10 * 3e9 / 0.02 s
    assert bench.weak_scaling_throughput(4, 10, 3e9, 20.0) == 4 * 10 * 3e9 / 0.02
    assert bench.weak_scaling_throughput(1, 1, 1.0, 1.0) == 1000.0


def test_tile_ceiling_against_a_tile_by_tile_count():
    """The useful fraction of the computed score-tile area: for the sliding window of 512 keys
    the page's workload gives 5 key tiles of 128 per 128-row Q tile against 512 x 128 useful
    pairs (80 %, up to the first rows); a non-causal square problem wastes nothing."""
    w = synthetic.WORKLOADS["gqa_sw512"]
    assert abs(bench.tile_ceiling(w) - 0.8) < 2e-3
    assert bench.tile_ceiling(synthetic.WORKLOADS["tiny"]) == 1.0
    # brute force on a small causal MQA-like shape: 8 heads packed per tile (16 tokens)
    small = synthetic.Workload("t", 0, 1, 8, 1, 100, 100, 64, 1)
    tiles = 0
    for t0 in range(0, 100, 16):
        hi = min(t0 + 15, 99)
        tiles += hi // 128 + 1
    useful = _pairs_brute(100, 100, 1, 0) * 8
    assert abs(bench.tile_ceiling(small) - useful / (tiles * 128 * 128)) < 1e-12


def test_tensor_peak_follows_the_power_cap_samples():
    peaks = {"bf16_tflops": 1629.0, "bf16_tflops_sustained": 1374.6, "hbm_gbs": 6557.4}
    assert bench.tensor_peak(peaks, {"reasons": []})[0] == 1629.0
    assert bench.tensor_peak(peaks, {"reasons": ["sw_power_cap"]})[0] == 1374.6
    assert bench.tensor_peak(peaks, None)[0] == 1629.0
