#!/usr/bin/env python
"""Benchmark of the fused attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  * prefill  (fa_fwd): MHA, B=2, Hq=Hkv=32, S=4096, D=128, causal, bf16 -- the workload the
    headline metric is quoted on (attention forward TFLOP/s);
  * decode   (fa_decode_int8, split kernel + combine kernel): B=16, Hq=32, Hkv=8, Skv=32768,
    D=128, INT8 KV cache with per-token scales, 16 splits (KV-read GB/s).
After the timed steps, short loops of their own time the paged, variable-length decode
(fa_decode_int8_paged, "paged_decode"), the INT4 decode (fa_decode_int4, "int4_decode"), the
masked and global+local forward passes, the backward pass, and the GQA causal, GQA
sliding-window and MQA causal forward workloads ("gqa_causal", "gqa_sw512", "mqa_causal"); they
are not part of the step.  Tensor-core fractions divide by the measured burst bf16 peak unless
the clock samples of the timed region saw the power cap.
Inputs are seeded synthetic N(0,1) draws (see synthetic.py) resident in HBM; both inputs are
larger than the 126 MB L2 (prefill 268 MB, decode 1.1 GB), so no flush is needed between steps.

Prints ONE JSON line (rank 0).  Under torchrun every rank runs the same workload on its own
GPU with its own seeds (independent problems, weak scaling, no data-path collective); times are
CUDA-event times, max over ranks.

On rank 0 of a one-GPU run the fp64 CPU oracle is also timed on bounded samples of the
prefill and decode workloads ("cpu_baseline", "cpu_baseline_decode"), and the INT8 / INT4 decode
results of the first two sequences are compared with the oracle over the unquantised bf16 K and
V ("kv_quant_error", informational).

``--impl reference`` times the fp64 CPU oracle on a bounded row sample of the same prefill
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn fwd TFLOP/s & % bf16 TC peak; decode KV-read GB/s & % HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# dram__bytes_read.sum + dram__bytes_write.sum per launch from ncu, keyed by the sha256 of the
# kernel sources they were taken on; a kernel edited since then reports traffic = null.
NCU_TRAFFIC = {
    # profiles/fa_prefill_kernel_mha_causal.md: 536,197,888 B read + 48,389,376 B written
    "prefill": {"9a69e24198021cef": 584_587_264},
    # profiles/fa_decode_split_kernel_decode_int8.md: 1,108,619,776 B read + 4,625,664 B written
    "decode": {"fdcac03dd1d0d86e": 1_113_245_440},
    # profiles/fa_decode_split_kernel_decode_int8_paged.md: 424,227,840 B read + 3,291,904 B
    # written
    "paged_decode": {"fdcac03dd1d0d86e": 427_519_744},
}


# the kernel that runs the plain prefill (causal / window / full) and its sources
KERNEL_PREFILL = "fa_prefill_kernel<{D}>"
PREFILL_SOURCES = ("prefill.cuh", "sm100.cuh")


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "tiled_attention_26_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def prefill_flops(w) -> int:
    """Algorithmic flops: 4*D per visible (query, key) pair (QK^T and PV, 2 flops per MAC)."""
    pairs = 0
    off = w.Skv - w.Sq
    for i in range(w.Sq):
        hi = min(i + off, w.Skv - 1) if w.causal else w.Skv - 1
        lo = max(0, i + off - w.window + 1) if w.window > 0 else 0
        pairs += max(0, hi - lo + 1)
    return pairs * 4 * w.D * w.B * w.Hq


def decode_bytes(w) -> int:
    """Algorithmic bytes: int8 K and V, fp32 scales, bf16 q in and o out, fp32 LSE."""
    kv = 2 * w.B * w.Skv * w.Hkv * w.D
    scales = 2 * w.B * w.Hkv * w.Skv * 4
    qo = 2 * w.B * w.Hq * w.D * 2
    return kv + scales + qo + w.B * w.Hq * 4


def paged_decode_bytes(w, seqlens) -> int:
    """Algorithmic bytes of one paged decode call: the int8 K and V rows and fp32 scales of every
    cached key, the block-table entries of the pages in use, the lengths, q in, o out, LSE."""
    import numpy as np
    sl = np.asarray(seqlens, dtype=np.int64)
    keys = int(sl.sum())
    pages = int((-(-sl // w.page_size)).sum())
    kv = 2 * keys * w.Hkv * w.D + 2 * keys * w.Hkv * 4
    return kv + 4 * pages + 4 * w.B + 2 * w.B * w.Hq * w.D * 2 + w.B * w.Hq * 4


def time_calls(torch, stream, call, steps: int, warmup: int) -> float:
    """Average ms per call of ``call`` over ``steps`` back-to-back launches (CUDA events)."""
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def global_local_flops(w, n_global: int) -> int:
    """4*D flops per visible (query, key) pair under the causal window rule plus global tokens."""
    import numpy as np
    i = np.arange(w.Sq, dtype=np.int64)
    ip = i + (w.Skv - w.Sq)
    hi = np.minimum(ip, w.Skv - 1)
    lo = np.maximum(0, ip - w.window + 1) if w.window > 0 else np.zeros_like(ip)
    band = np.maximum(0, hi - lo + 1)
    # keys below G outside the band, for rows that are not global themselves
    extra = np.maximum(0, np.minimum(n_global, lo) - 0)
    pairs = np.where(i < n_global, w.Skv, band + extra)
    return int(pairs.sum()) * 4 * w.D * w.B * w.Hq


def tile_ceiling(w) -> float:
    """Useful fraction of the score-tile area the prefill kernel computes for workload w: visible
    (query, key) pairs over (tiles computed x 128 x 128).  A Q tile holds 128 rows = 128 / Gp
    tokens x Gp query heads of one KV group (Gp the largest power of two <= 8 dividing Hq/Hkv);
    it computes every 128-key tile that holds a key one of its rows sees."""
    G = w.Hq // w.Hkv
    gp = 1
    while gp < 8 and G % (2 * gp) == 0:
        gp *= 2
    tpt = 128 // gp
    off = w.Skv - w.Sq
    tiles = 0
    for t0 in range(0, w.Sq, tpt):
        t1 = min(t0 + tpt, w.Sq) - 1
        hi = min(t1 + off, w.Skv - 1) if w.causal else w.Skv - 1
        lo = max(0, t0 + off - w.window + 1) if w.window > 0 else 0
        if hi >= lo and hi >= 0:
            tiles += hi // 128 - lo // 128 + 1
    computed = tiles * (w.Hq // gp) * w.B * 128 * 128
    return prefill_flops(w) / (4 * w.D) / computed


def tensor_peak(peaks, clk):
    """The dense bf16 peak a prefill kernel is held against: the burst figure, unless the clock
    samples of the timed region saw the power cap, then the sustained one."""
    if "sw_power_cap" in (clk or {}).get("reasons", []):
        return peaks["bf16_tflops_sustained"], "sustained (sw_power_cap seen in the timed region)"
    return peaks["bf16_tflops"], "burst (no power cap seen in the timed region)"


def measure_prefill_configs(fa, synthetic, torch, dev, stream, steps: int, warmup: int,
                            seed_off: int = 0):
    """fa_fwd on the GQA causal, GQA sliding-window and MQA causal workloads, each in its own
    loop.  Returns {name: (ms per call, algorithmic flops)}."""
    out = {}
    for name in ("gqa_causal", "gqa_sw512", "mqa_causal"):
        w = synthetic.WORKLOADS[name]
        q = synthetic.normal_bf16_torch(w.seed(0) + seed_off, w.q_shape(), dev)
        k = synthetic.normal_bf16_torch(w.seed(1) + seed_off, w.kv_shape(), dev)
        v = synthetic.normal_bf16_torch(w.seed(2) + seed_off, w.kv_shape(), dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=dev)
        ms = time_calls(torch, stream, lambda: fa.fa_fwd(q, k, v, causal=w.causal, window=w.window,
                                                          scale=w.scale, o=o, lse=lse,
                                                          stream=stream), steps, warmup)
        out[name] = (ms, prefill_flops(w))
        del q, k, v, o, lse
    if fa.fa_device_status() != 0:
        raise RuntimeError("a prefill kernel reported a device-side error")
    return out


def measure_mask_variants(fa, synthetic, torch, dev, stream, steps: int, warmup: int):
    """The forward pass with a per-head additive bias mask on the MHA causal workload, and with
    64 global tokens on the GQA sliding-window workload.  Returns {name: (ms, flops)}."""
    import numpy as np
    out = {}
    w = synthetic.WORKLOADS["mha_causal"]
    q, k, v = synthetic.make_qkv_torch(w, dev)
    slopes = 2.0 ** (-8.0 * np.arange(1, w.Hq + 1) / w.Hq)
    dist = (np.arange(w.Skv)[None, :] - np.arange(w.Sq)[:, None]).astype(np.float64)
    mask = torch.from_numpy(
        (slopes[:, None, None] * np.minimum(dist, 0.0)[None]).astype(np.float32)[None]).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=dev)
    ms = time_calls(torch, stream, lambda: fa.fa_fwd(q, k, v, causal=True, scale=w.scale, o=o,
                                                      lse=lse, mask=mask, stream=stream),
                    steps, warmup)
    out["masked"] = (ms, prefill_flops(w))
    del q, k, v, mask, o, lse
    w = synthetic.WORKLOADS["gqa_sw512"]
    q, k, v = synthetic.make_qkv_torch(w, dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=dev)
    ms = time_calls(torch, stream, lambda: fa.fa_fwd(q, k, v, causal=True, window=w.window,
                                                      scale=w.scale, o=o, lse=lse, n_global=64,
                                                      stream=stream), steps, warmup)
    out["global_local"] = (ms, global_local_flops(w, 64))
    if fa.fa_device_status() != 0:
        raise RuntimeError("a masked forward reported a device-side error")
    return out


def measure_backward(fa, synthetic, torch, dev, stream, steps: int, warmup: int):
    """fa_bwd on the MHA causal workload (its own loop; the forward pass runs once, outside the
    timing).  Returns (ms per call, algorithmic flops = 10*D per visible pair: the five products
    S, dP, dV, dK, dQ)."""
    w = synthetic.WORKLOADS["mha_causal"]
    q, k, v = synthetic.make_qkv_torch(w, dev)
    do = synthetic.normal_bf16_torch(w.seed(3), w.q_shape(), dev)
    o, lse = fa.fa_fwd(q, k, v, causal=True, scale=w.scale, stream=stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.Hq, w.Sq), dtype=torch.uint8, device=dev)
    ms = time_calls(torch, stream,
                    lambda: fa.fa_bwd(q, k, v, o, do, lse, causal=True, scale=w.scale, dq=dq,
                                      dk=dk, dv=dv, workspace=ws, stream=stream), steps, warmup)
    if fa.fa_device_status() != 0:
        raise RuntimeError("the backward pass reported a device-side error")
    return ms, prefill_flops(w) // 4 * 10


def measure_paged_decode(fa, synthetic, torch, dev, stream, steps: int, warmup: int):
    """Time fa_decode_int8_paged on the paged workload (its own short loop after the step loop).
    Returns (ms per call averaged over ``steps`` launches, algorithmic bytes per call)."""
    w = synthetic.PAGED_WORKLOADS["decode_int8_paged"]
    q, kp, vp, ksp, vsp, bt, sl = synthetic.make_paged_decode_inputs_torch(w, dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_int8_workspace_bytes(w.B, w.Hq, w.D, w.num_splits),
                     dtype=torch.uint8, device=dev)

    def call():
        fa.fa_decode_int8_paged(q, kp, vp, ksp, vsp, bt, sl, num_splits=w.num_splits,
                                scale=w.scale, o=o, lse=lse, workspace=ws, stream=stream)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    if fa.fa_device_status() != 0:
        raise RuntimeError("the paged decode reported a device-side error")
    return a.elapsed_time(b) / steps, paged_decode_bytes(w, sl.cpu().numpy())


def int4_decode_bytes(w) -> int:
    """Algorithmic bytes of one INT4 decode call: packed K and V codes (D/2 bytes per key and
    head), fp32 scales, bf16 q in and o out, fp32 LSE."""
    kv = 2 * w.B * w.Skv * w.Hkv * (w.D // 2)
    scales = 2 * w.B * w.Hkv * w.Skv * 4
    return kv + scales + 2 * w.B * w.Hq * w.D * 2 + w.B * w.Hq * 4


def measure_int4_decode(fa, synthetic, torch, dev, stream, steps: int, warmup: int):
    """Time fa_decode_int4 on the INT4 workload (its own short loop after the step loop).
    Returns (ms per call averaged over ``steps`` launches, algorithmic bytes per call)."""
    w = synthetic.WORKLOADS["decode_int4"]
    q, k4, v4, ks, vs = synthetic.make_decode_int4_inputs_torch(w, dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_int8_workspace_bytes(w.B, w.Hq, w.D, w.num_splits),
                     dtype=torch.uint8, device=dev)

    def call():
        fa.fa_decode_int4(q, k4, v4, ks, vs, num_splits=w.num_splits, scale=w.scale, o=o,
                          lse=lse, workspace=ws, stream=stream)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    if fa.fa_device_status() != 0:
        raise RuntimeError("the INT4 decode reported a device-side error")
    return a.elapsed_time(b) / steps, int4_decode_bytes(w)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"samples": 0, "sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"samples": len(sm), "sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


class OracleTimer:
    """Times the fp64 oracle, as it stands, on bounded row samples of the prefill workload."""

    def __init__(self, w):
        import numpy as np

        import oracle
        import synthetic

        self.w, self.oracle, self.np, self.synthetic = w, oracle, np, synthetic
        self.q, self.k, self.v = synthetic.make_qkv(w)
        self.cores = oracle.max_threads()
        t0 = time.perf_counter()
        self.run(self.rows(w.seed(39), 64))
        self.rows_per_s = 64 / max(time.perf_counter() - t0, 1e-3)

    def rows(self, seed, n):
        np, w = self.np, self.w
        raw = self.synthetic.splitmix64(seed, 0, 3 * n).reshape(-1, 3)
        return np.stack([raw[:, 0] % np.uint64(w.B), raw[:, 1] % np.uint64(w.Hq),
                         raw[:, 2] % np.uint64(w.Sq)], axis=1).astype(np.int64)

    def flops(self, rows):
        w = self.w
        off = w.Skv - w.Sq
        n = 0
        for _, _, i in rows:
            hi = min(i + off, w.Skv - 1) if w.causal else w.Skv - 1
            lo = max(0, i + off - w.window + 1) if w.window > 0 else 0
            n += 4 * w.D * max(0, hi - lo + 1)
        return n

    def run(self, rows):
        w = self.w
        self.oracle.attn_rows(self.q, self.k, self.v, w.scale, w.causal, w.window, rows)

    def sample(self, seed, budget_s):
        """Returns (flops, seconds, n_rows) for a sample sized to take about budget_s."""
        n = max(8, int(self.rows_per_s * budget_s))
        rows = self.rows(seed, n)
        t0 = time.perf_counter()
        self.run(rows)
        return self.flops(rows), time.perf_counter() - t0, n


def cpu_baseline(w, budget_s: float, seed: int):
    t = OracleTimer(w)
    fl, dt, n = t.sample(seed, budget_s)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": t.cores, "kind": "oracle",
            "sample": f"{n} seeded (b, h, i) rows of the prefill workload, every visible key, "
                      f"fp64, {dt:.1f} s"}, dt


def cpu_baseline_decode(dev_inputs, w, budget_s: float, seed: int):
    """The fp64 oracle's INT8 decode (as it stands) on a bounded sample of (b, h) rows of the
    decode workload, on the host cores: algorithmic bytes of the sampled rows per second."""
    import numpy as np

    import oracle
    import torch
    q = dev_inputs[0].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    kq, vq, ks, vs = (t.cpu().numpy() for t in dev_inputs[1:])
    G = w.Hq // w.Hkv

    def rows(n, s):
        import synthetic
        raw = synthetic.splitmix64(s, 0, 2 * n).reshape(-1, 2)
        return np.stack([raw[:, 0] % np.uint64(w.B), raw[:, 1] % np.uint64(w.Hq)],
                        axis=1).astype(np.int64)

    def bytes_of(r):
        # each row reads its KV head's codes and scales once (the kernel reads them once per
        # group of G rows), plus its q, o and LSE
        per_kv = 2 * w.Skv * w.D + 2 * w.Skv * 4
        return len(r) * (per_kv / G + 2 * w.D * 2 + 4)

    t0 = time.perf_counter()
    oracle.decode_int8_rows(q, kq, vq, ks, vs, w.scale, 1, rows(8, seed))
    per_row = max((time.perf_counter() - t0) / 8, 1e-4)
    r = rows(max(8, int(budget_s / per_row)), seed + 1)
    t0 = time.perf_counter()
    oracle.decode_int8_rows(q, kq, vq, ks, vs, w.scale, 1, r)
    dt = time.perf_counter() - t0
    return {"value": bytes_of(r) / dt / 1e9, "unit": "GB/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{len(r)} seeded (b, h) rows of the INT8 decode workload, all "
                      f"{w.Skv} keys each, fp64, {dt:.1f} s (bytes counted as the kernel reads "
                      f"them: each KV head's codes and scales once per {G} query heads)"}


def kv_quant_error(fa, synthetic, torch, dev, w, n_batch: int = 2):
    """Informational: how far INT8 and INT4 KV-cache decode land from attention over the
    unquantised bf16 K and V, on the first n_batch sequences of the decode workload (the same
    seeded bf16 values the INT8 cache was quantised from).  The reference is the fp64 oracle
    over the bf16 values; the quantised results are this library's decode kernels."""
    import numpy as np

    import oracle
    shp = (n_batch, w.Skv, w.Hkv, w.D)
    q = synthetic.normal_bf16_torch(w.seed(0), (n_batch, 1, w.Hq, w.D), dev)
    k = synthetic.normal_bf16_torch(w.seed(1), shp, dev)
    v = synthetic.normal_bf16_torch(w.seed(2), shp, dev)
    host = [t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16) for t in (q, k, v)]
    o_ref, _ = oracle.attn(host[0], host[1], host[2], w.scale, 0, 0)
    o_ref = o_ref.reshape(n_batch, w.Hq, w.D)
    out = {}
    for name, quant, call in (("int8", synthetic.quantize_int8_per_token_torch, fa.fa_decode_int8),
                              ("int4", synthetic.quantize_int4_per_token_torch, fa.fa_decode_int4)):
        kq, ks = quant(k)
        vq, vs = quant(v)
        o, _ = call(q, kq, vq, ks, vs, num_splits=w.num_splits, scale=w.scale)
        got = o.float().cpu().numpy().astype(np.float64).reshape(n_batch, w.Hq, w.D)
        d = np.abs(got - o_ref)
        out[name] = {"max_abs": float(d.max()), "mean_abs": float(d.mean()),
                     "rel_l2": float(np.linalg.norm(d) / np.linalg.norm(o_ref)),
                     "max_abs_over_max_ref": float(d.max() / np.abs(o_ref).max())}
    if fa.fa_device_status() != 0:
        raise RuntimeError("a decode kernel reported a device-side error")
    return {"rows": f"{n_batch} x {w.Hq} (b, h) rows of the INT8 decode workload, {w.Skv} keys",
            "reference": "fp64 oracle over the unquantised bf16 K and V",
            "pages_claim": "precision loss < 0.5 % with the INT8 KV cache (no metric stated); "
                           "rel_l2 is the closest figure here",
            **out}


def run_reference(args):
    import synthetic

    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    w = synthetic.WORKLOADS["mha_causal"]
    timer = OracleTimer(w)
    per_step = min(4.0, 120.0 / max(1, args.steps + args.warmup))
    tot_f, tot_t, n_rows = 0, 0.0, 0
    for step in range(args.warmup + args.steps):
        fl, dt, n = timer.sample(w.seed(50 + step), per_step)
        if step >= args.warmup:
            tot_f, tot_t, n_rows = tot_f + fl, tot_t + dt, n_rows + n
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * tot_t / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "mha_causal prefill B=2 Hq=Hkv=32 S=4096 D=128 causal "
                               "(bounded row sample per step)", "parallelism": "rank 0 only"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": timer.cores, "kind": "oracle",
                         "sample": f"{n_rows} seeded (b, h, i) rows over {args.steps} steps, every "
                                   f"visible key, fp64, {tot_t:.1f} s"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class Ranks:
    """One process per GPU: rank / world from the torchrun environment, a process group when
    world > 1 (nccl on GPUs; the tests use gloo), a barrier, and the max over ranks that every
    reported time goes through.  Every rank runs its own independent workload, so no data-path
    collective exists: the only collectives are the barrier and these max-reductions."""

    def __init__(self, world: int, rank: int, local: int, backend: str | None):
        import torch
        self.world, self.rank, self.local = world, rank, local
        self.dist = None
        self.device = "cpu"
        if backend == "nccl":
            torch.cuda.set_device(local)
            self.device = torch.device("cuda", local)
        if world > 1:
            import datetime

            import torch.distributed as dist
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.dist = dist

    @classmethod
    def from_env(cls, backend: str):
        return cls(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                   int(os.environ.get("LOCAL_RANK", "0")), backend)

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, x: float) -> float:
        if self.dist is None:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()
            self.dist = None


def rank_seed_offset(rank: int) -> int:
    """Rank r draws its inputs from seeds shifted by 1000 r: independent problems per GPU."""
    return 1000 * rank


def weak_scaling_throughput(world: int, steps: int, work_per_step: float, max_ms: float) -> float:
    """Whole-job throughput (work units per second): every rank did `steps` steps of
    `work_per_step` units; the job took the slowest rank's time."""
    return world * steps * work_per_step / (max_ms * 1e-3)


def run_only_prefill(args):
    """fa_fwd on one prefill workload alone (--workload, default the MHA causal one), one JSON
    line (used to profile the prefill kernel without the other workloads resident)."""
    import torch

    import synthetic
    import tiled_attention_26_b200 as fa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    w = synthetic.WORKLOADS[args.workload]
    q, k, v = synthetic.make_qkv_torch(w, dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=dev)
    ms = time_calls(torch, stream, lambda: fa.fa_fwd(q, k, v, causal=w.causal, window=w.window,
                                                      scale=w.scale, o=o, lse=lse, stream=stream),
                    args.steps, args.warmup)
    if fa.fa_device_status() != 0:
        raise RuntimeError("the prefill kernel reported a device-side error")
    flops = prefill_flops(w)
    peaks, _ = load_peaks()
    print(json.dumps({"metric": "attention forward TFLOP/s (4*D flops per visible pair)",
                      "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "ms_per_call": ms, "steps": args.steps, "warmup": args.warmup,
                      "frac_of_burst": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                      "config": {"workload": args.workload}}), flush=True)
    return 0


def run_only_masked(args):
    """fa_fwd with the per-head additive bias mask on the MHA causal workload alone, one JSON
    line (used to profile the masked prefill kernel)."""
    import torch

    import synthetic
    import tiled_attention_26_b200 as fa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    mv = measure_mask_variants(fa, synthetic, torch, dev, stream, steps=args.steps,
                               warmup=args.warmup)
    ms, flops = mv["masked"]
    peaks, _ = load_peaks()
    print(json.dumps({"metric": "masked attention forward TFLOP/s (4*D flops per visible pair)",
                      "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_call": ms,
                      "steps": args.steps, "warmup": args.warmup,
                      "frac_of_burst": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                      "config": {"workload": "mha_causal + per-head fp32 bias [1, 32, 4096, 4096]"}}),
          flush=True)
    return 0


def run_only_backward(args):
    """fa_bwd on the MHA causal workload alone, one JSON line (used to profile the backward
    kernels without the other workloads resident on the device)."""
    import torch

    import synthetic
    import tiled_attention_26_b200 as fa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    ms, flops = measure_backward(fa, synthetic, torch, dev, stream, steps=args.steps,
                                 warmup=args.warmup)
    peaks, _ = load_peaks()
    print(json.dumps({"metric": "attention backward TFLOP/s (10*D flops per visible pair)",
                      "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "ms_per_call": ms, "steps": args.steps, "warmup": args.warmup,
                      "frac_of_burst": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                      "config": {"workload": "mha_causal (B=2, H=32, S=4096, D=128, causal)"}}),
          flush=True)
    return 0


def run_only_decode(args):
    """fa_decode_int8 on the contiguous decode workload alone, one JSON line (used to profile
    the decode kernels without the other workloads resident on the device)."""
    import torch

    import synthetic
    import tiled_attention_26_b200 as fa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    w = synthetic.WORKLOADS["decode_int8"]
    q, k, v, ks, vs = synthetic.make_decode_inputs_torch(w, dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_int8_workspace_bytes(w.B, w.Hq, w.D, w.num_splits),
                     dtype=torch.uint8, device=dev)
    ms = time_calls(torch, stream, lambda: fa.fa_decode_int8(q, k, v, ks, vs,
                                                             num_splits=w.num_splits,
                                                             scale=w.scale, o=o, lse=lse,
                                                             workspace=ws, stream=stream),
                    args.steps, args.warmup)
    if fa.fa_device_status() != 0:
        raise RuntimeError("the decode kernels reported a device-side error")
    nbytes = decode_bytes(w)
    peaks, _ = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({"metric": "INT8 decode GB/s (algorithmic bytes)", "value": gbs,
                      "unit": "GB/s", "ms_per_call": ms, "bytes_per_call": nbytes,
                      "steps": args.steps, "warmup": args.warmup,
                      "frac_of_hbm": gbs / peaks["hbm_gbs"],
                      "config": {"workload": "decode_int8"}}), flush=True)
    return 0


def run_only_int4(args):
    """fa_decode_int4 on the INT4 decode workload alone, one JSON line (used to profile the
    4-bit decode kernels without the other workloads resident on the device)."""
    import torch

    import synthetic
    import tiled_attention_26_b200 as fa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    ms, nbytes = measure_int4_decode(fa, synthetic, torch, dev, stream, steps=args.steps,
                                     warmup=args.warmup)
    peaks, _ = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({"metric": "INT4 decode GB/s (algorithmic bytes)", "value": gbs,
                      "unit": "GB/s", "ms_per_call": ms, "bytes_per_call": nbytes,
                      "steps": args.steps, "warmup": args.warmup,
                      "frac_of_hbm": gbs / peaks["hbm_gbs"],
                      "config": {"workload": "decode_int4"}}), flush=True)
    return 0


def run_only_paged(args):
    """fa_decode_int8_paged on the paged workload alone, one JSON line (used to profile the
    paged decode kernels without the other workloads resident on the device)."""
    import torch

    import synthetic
    import tiled_attention_26_b200 as fa
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    ms, nbytes = measure_paged_decode(fa, synthetic, torch, dev, stream, steps=args.steps,
                                      warmup=args.warmup)
    peaks, _ = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({"metric": "paged INT8 decode GB/s (algorithmic bytes)", "value": gbs,
                      "unit": "GB/s", "ms_per_call": ms, "bytes_per_call": nbytes,
                      "steps": args.steps, "warmup": args.warmup,
                      "frac_of_hbm": gbs / peaks["hbm_gbs"],
                      "config": {"workload": "decode_int8_paged"}}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mha_causal",
                    choices=["mha_causal", "gqa_causal", "gqa_sw512", "mqa_causal"],
                    help="prefill workload of --only prefill")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["backward", "prefill", "paged", "decode", "int4", "masked"],
                    default=None,
                    help="time one further row on its own (for profiling); prints its own line")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.only == "backward":
        return run_only_backward(args)
    if args.only == "prefill":
        return run_only_prefill(args)
    if args.only == "paged":
        return run_only_paged(args)
    if args.only == "decode":
        return run_only_decode(args)
    if args.only == "int4":
        return run_only_int4(args)
    if args.only == "masked":
        return run_only_masked(args)

    import torch

    import synthetic
    import tiled_attention_26_b200 as fa

    ranks = Ranks.from_env("nccl")
    world, rank, local = ranks.world, ranks.rank, ranks.local
    barrier, max_over_ranks = ranks.barrier, ranks.max

    wp = synthetic.WORKLOADS["mha_causal"]
    wd = synthetic.WORKLOADS["decode_int8"]
    dev = torch.device("cuda", local)
    seed_off = rank_seed_offset(rank)
    q = synthetic.normal_bf16_torch(wp.seed(0) + seed_off, wp.q_shape(), dev)
    k = synthetic.normal_bf16_torch(wp.seed(1) + seed_off, wp.kv_shape(), dev)
    v = synthetic.normal_bf16_torch(wp.seed(2) + seed_off, wp.kv_shape(), dev)
    o = torch.empty_like(q)
    lse = torch.empty((wp.B, wp.Hq, wp.Sq), dtype=torch.float32, device=dev)
    dq = synthetic.normal_bf16_torch(wd.seed(0) + seed_off, wd.q_shape(), dev)
    dk, dks = synthetic.quantize_int8_per_token_torch(
        synthetic.normal_bf16_torch(wd.seed(1) + seed_off, wd.kv_shape(), dev))
    dv, dvs = synthetic.quantize_int8_per_token_torch(
        synthetic.normal_bf16_torch(wd.seed(2) + seed_off, wd.kv_shape(), dev))
    do = torch.empty_like(dq)
    dlse = torch.empty((wd.B, wd.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_int8_workspace_bytes(wd.B, wd.Hq, wd.D, wd.num_splits),
                     dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def prefill():
        fa.fa_fwd(q, k, v, causal=True, scale=wp.scale, o=o, lse=lse, stream=stream)

    def decode():
        fa.fa_decode_int8(dq, dk, dv, dks, dvs, num_splits=wd.num_splits, scale=wd.scale, o=do,
                          lse=dlse, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        prefill()
        decode()
    torch.cuda.synchronize()
    if fa.fa_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side timeout during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    phys = int(visible[local]) if local < len(visible) and visible[local].strip().isdigit() else local
    clocks = ClockSampler(phys)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)  # let the sampler start before the timed region
    start.record(stream)
    for s in range(K):
        ev[s][0].record(stream)
        prefill()
        ev[s][1].record(stream)
        decode()
        ev[s][2].record(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    if fa.fa_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side timeout in the timed region")

    total_ms = max_over_ranks(start.elapsed_time(stop))
    pre_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(K)]
    dec_ms = [ev[s][1].elapsed_time(ev[s][2]) for s in range(K)]
    pre_sum = max_over_ranks(sum(pre_ms))
    dec_sum = max_over_ranks(sum(dec_ms))

    flops = prefill_flops(wp)
    dbytes = decode_bytes(wd)
    peaks, peak_src = load_peaks()
    pre_tflops = weak_scaling_throughput(world, K, flops, pre_sum) / 1e12
    dec_gbs = weak_scaling_throughput(world, K, dbytes, dec_sum) / 1e9
    pre_avg_s = sum(pre_ms) / K * 1e-3
    dec_avg_s = sum(dec_ms) / K * 1e-3
    achieved = flops / pre_avg_s / 1e12
    d_achieved = dbytes / dec_avg_s / 1e9

    # ---- the paged, variable-length decode (a further row of the path), its own short loop ----
    pg_ms, pg_bytes = measure_paged_decode(fa, synthetic, torch, dev, stream,
                                           steps=min(K, 200), warmup=max(3, args.warmup // 4))
    pg_ms = max_over_ranks(pg_ms)
    i4_ms, i4_bytes = measure_int4_decode(fa, synthetic, torch, dev, stream,
                                          steps=min(K, 200), warmup=max(3, args.warmup // 4))
    i4_ms = max_over_ranks(i4_ms)
    mv = measure_mask_variants(fa, synthetic, torch, dev, stream, steps=min(K, 100),
                               warmup=max(3, args.warmup // 4))
    mv = {kk: (max_over_ranks(ms), fl) for kk, (ms, fl) in mv.items()}
    bw_ms, bw_flops = measure_backward(fa, synthetic, torch, dev, stream, steps=min(K, 50),
                                       warmup=max(3, args.warmup // 4))
    bw_ms = max_over_ranks(bw_ms)
    pc = measure_prefill_configs(fa, synthetic, torch, dev, stream, steps=min(K, 100),
                                 warmup=max(3, args.warmup // 4), seed_off=seed_off)
    pc = {kk: (max_over_ranks(ms), fl) for kk, (ms, fl) in pc.items()}

    # ---- end to end through the public API, host buffers, copies inside the timed region ----
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho, hl = torch.empty_like(hq).pin_memory(), lse.cpu().pin_memory()
        hdq, hdk, hdv, hdks, hdvs = (t.cpu().pin_memory() for t in (dq, dk, dv, dks, dvs))
        hdo, hdl = torch.empty_like(hdq).pin_memory(), dlse.cpu().pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdq, hdk, hdv, hdks, hdvs))
        d2h = sum(t.numel() * t.element_size() for t in (ho, hl, hdo, hdl))
        E = args.e2e_steps
        e3 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(E)]
        barrier()
        torch.cuda.synchronize()
        for s in range(E):
            e3[s][0].record(stream)
            for d_, h_ in ((q, hq), (k, hk), (v, hv)):
                d_.copy_(h_, non_blocking=True)
            prefill()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            e3[s][1].record(stream)
            for d_, h_ in ((dq, hdq), (dk, hdk), (dv, hdv), (dks, hdks), (dvs, hdvs)):
                d_.copy_(h_, non_blocking=True)
            decode()
            hdo.copy_(do, non_blocking=True)
            hdl.copy_(dlse, non_blocking=True)
            e3[s][2].record(stream)
        torch.cuda.synchronize()
        barrier()
        p_ms = max_over_ranks(sum(e3[s][0].elapsed_time(e3[s][1]) for s in range(E)))
        d_ms = max_over_ranks(sum(e3[s][1].elapsed_time(e3[s][2]) for s in range(E)))
        e2e = {"value": weak_scaling_throughput(world, E, flops, p_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": E,
               "decode": {"value": weak_scaling_throughput(world, E, dbytes, d_ms) / 1e9,
                          "unit": "GB/s"},
               "ms_per_step": (p_ms + d_ms) / E}

    cpu = cpu_dec = qerr = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, _ = cpu_baseline(wp, args.cpu_budget, seed=wp.seed(40))
        cpu_dec = cpu_baseline_decode((dq, dk, dv, dks, dvs), wd, args.cpu_budget,
                                      seed=wd.seed(40))
        qerr = kv_quant_error(fa, synthetic, torch, dev, wd)

    tpeak, tpeak_src = tensor_peak(peaks, clk)

    def prefill_row(name, desc):
        ms, fl = pc[name]
        w = synthetic.WORKLOADS[name]
        tf = fl / (ms * 1e-3) / 1e12
        return {"workload": desc, "kernel": KERNEL_PREFILL.format(D=w.D), "ms_per_call": ms,
                "flops_per_call": fl, "achieved": tf, "unit": "TFLOP/s", "peak": tpeak,
                "frac": tf / tpeak, "tile_ceiling": tile_ceiling(w)}

    if rank == 0:
        tp = NCU_TRAFFIC["prefill"].get(source_hash(*PREFILL_SOURCES))
        td = NCU_TRAFFIC["decode"].get(source_hash("decode.cuh", "sm100.cuh"))
        line = {
            "metric": METRIC,
            "value": pre_tflops,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": total_ms / K,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {
                "workload": "one step = mha_causal prefill (B=2, Hq=Hkv=32, S=4096, D=128, causal, "
                            "bf16) + decode_int8 (B=16, Hq=32, Hkv=8, Skv=32768, D=128, INT8 KV, "
                            "16 splits)",
                "prefill_flops_per_step": flops,
                "decode_bytes_per_step": dbytes,
                "l2": "no flush: every step reads inputs larger than L2 (prefill 268 MB, decode 1.1 GB)",
                "parallelism": f"{world} independent GPU(s), no data-path collective",
            },
            "decode": {"value": dec_gbs, "unit": "GB/s", "frac_of_hbm": dec_gbs / world / peaks["hbm_gbs"],
                       "ms_per_call": dec_sum / K},
            # The denominator is the burst dense bf16 figure unless the clock samples of the
            # timed region saw the power cap (then the sustained one); the fraction of the
            # other figure is reported beside it.
            "roofline": {"bound": "tensor", "achieved": achieved,
                         "peak": tpeak, "unit": "TFLOP/s",
                         "frac": achieved / tpeak,
                         "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
                         "frac_of_sustained_peak": achieved / peaks["bf16_tflops_sustained"],
                         "traffic": tp, "kernel": KERNEL_PREFILL.format(D=wp.D),
                         "peak_source": f"{peak_src} bf16 dense, {tpeak_src}",
                         "ms_per_launch": pre_avg_s * 1e3},
            "roofline_decode": {"bound": "hbm", "achieved": d_achieved, "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": d_achieved / peaks["hbm_gbs"],
                                "traffic": td,
                                "kernel": "fa_decode_split_kernel<128> + fa_decode_combine_kernel<128>",
                                "peak_source": f"{peak_src} copy bandwidth",
                                "ms_per_call": dec_avg_s * 1e3},
            "paged_decode": {
                "workload": "decode_int8_paged: B=16, Hq=32, Hkv=8, D=128, INT8 KV in 64-token "
                            "pages scattered over the pool, lengths uniform in [1, 32768] "
                            f"({pg_bytes / 1e6:.1f} MB per call), 8 splits",
                "kernel": "fa_decode_split_kernel<128, paged> + fa_decode_combine_kernel<128>",
                "ms_per_call": pg_ms, "achieved": pg_bytes / (pg_ms * 1e-3) / 1e9,
                "unit": "GB/s", "peak": peaks["hbm_gbs"],
                "frac": pg_bytes / (pg_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "launches": 2 * min(K, 200),
                "traffic": NCU_TRAFFIC["paged_decode"].get(source_hash("decode.cuh", "sm100.cuh"))},
            "int4_decode": {
                "workload": "decode_int4: B=16, Hq=32, Hkv=8, Skv=32768, D=128, INT4 KV (two codes "
                            f"per byte, per-token scales, {i4_bytes / 1e6:.1f} MB per call), 16 splits",
                "kernel": "fa_decode_split_kernel<128, contiguous, 4-bit> + fa_decode_combine_kernel<128>",
                "ms_per_call": i4_ms, "achieved": i4_bytes / (i4_ms * 1e-3) / 1e9,
                "unit": "GB/s", "peak": peaks["hbm_gbs"],
                "frac": i4_bytes / (i4_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "launches": 2 * min(K, 200)},
            "masked_prefill": {
                "workload": "mha_causal (B=2, H=32, S=4096, D=128, causal) + per-head additive "
                            "fp32 bias mask [1, 32, 4096, 4096]",
                "kernel": "fa_prefill_kernel<128, mask>", "ms_per_call": mv["masked"][0],
                "achieved": mv["masked"][1] / (mv["masked"][0] * 1e-3) / 1e12, "unit": "TFLOP/s",
                "frac": mv["masked"][1] / (mv["masked"][0] * 1e-3) / 1e12 / tpeak},
            "global_local_prefill": {
                "workload": "gqa_sw512 (B=1, Hq=32, Hkv=8, S=4096, D=128, causal window 512) + "
                            "64 global tokens",
                "kernel": "fa_prefill_kernel<128, global>", "ms_per_call": mv["global_local"][0],
                "achieved": mv["global_local"][1] / (mv["global_local"][0] * 1e-3) / 1e12,
                "unit": "TFLOP/s",
                "frac": mv["global_local"][1] / (mv["global_local"][0] * 1e-3) / 1e12 / tpeak},
            "backward": {
                "workload": "mha_causal (B=2, H=32, S=4096, D=128, causal): fa_bwd after fa_fwd",
                "kernels": "fa_bwd_prep_kernel + fa_bwd_kernel<128> (dK, dV and the dQ shares) + "
                           "fa_bwd_dq_finalize_kernel",
                "ms_per_call": bw_ms, "flops_per_call": bw_flops,
                "achieved": bw_flops / (bw_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "frac": bw_flops / (bw_ms * 1e-3) / 1e12 / tpeak},
            "gqa_causal": prefill_row("gqa_causal", "GQA causal (B=1, Hq=32, Hkv=8, S=4096, "
                                                    "D=128)"),
            "gqa_sw512": prefill_row("gqa_sw512", "GQA causal, sliding window W=512 (B=1, Hq=32, "
                                                  "Hkv=8, S=4096, D=128); tile_ceiling = visible "
                                                  "pairs / computed tile area"),
            "mqa_causal": prefill_row("mqa_causal", "MQA causal (B=1, Hq=232, Hkv=1, S=2048, "
                                                    "D=64)"),
            "cpu_baseline": cpu,
            "cpu_baseline_decode": cpu_dec,
            "kv_quant_error": qerr,
            "e2e": e2e,
            "gpu_launches": 3 * K,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
