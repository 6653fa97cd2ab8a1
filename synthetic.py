"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle driver.

This module holds no attention arithmetic. It only draws numbers and names workloads:

* ``normal_bf16(seed, n)`` -- a counter-based stream: element pair ``m`` takes the
  splitmix64 outputs ``2m`` and ``2m+1`` of the generator started at ``seed``, turns
  them into two uniforms and then into two N(0,1) values by the Box-Muller transform
  (fp64).  Each value is rounded to fp32 (round-to-nearest-even) and then to bf16
  (round-to-nearest-even).  The result is returned as raw bf16 bit patterns (uint16).
* ``quantize_int4_per_token`` -- the INT4 recipe: the same with max|x| / 7 and codes in
  [-7, 7], packed two per byte (dim 2i in the low nibble), 4-bit two's complement.
* ``quantize_int8_per_token`` -- the INT8 KV-cache recipe of the decode workload:
  symmetric, one fp32 scale per (token, kv-head) equal to max|x| / 127, codes
  ``clamp(rint(x / scale), -127, 127)`` with the division in fp32 and ties to even.
  The pages ("Flash Attention on Ascend: three techniques", section on INT8/INT4 KV
  compression) state only that the cache is INT8 with the computation done on the
  compressed data; the per-token symmetric scheme is this project's reading.
* ``WORKLOADS`` -- the shapes of the pages' examples ("FlashAttention variants: GQA,
  MQA, sparse attention", benchmark section: seq 4096, 32 query heads, head dim 128;
  Llama-2-7B 32/32, Mistral-7B 32/8, Falcon-180B 232/1) plus a tiny parity case and
  an INT8-KV decode case.

* ``PAGED_WORKLOADS`` / ``make_paged_decode_inputs`` -- decode over a paged INT8 cache with a
  mix of sequence lengths in one batch ("Flash Attention on Ascend: three techniques", version
  section: sequences of different lengths computed together; "Sparse attention and MLA operators
  in ops-transformer", section 2.2: KV pages addressed through a block_table).  Lengths are uniform integers in
  [min_len, max_len] (splitmix64 value modulo the range; the modulo bias is below 2^-40), and
  the physical pages are handed out in the order of a seeded random permutation, so that each
  sequence's pages are scattered over the pool as in a long-running cache.

Seeds are ``20260 + 10 * workload_index + tensor_index`` with Q=0, K=1, V=2 (paged workloads
add lengths=3 and page permutation=4).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of splitmix64 started at state ``seed``."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def normal_f64(seed: int, n: int, chunk: int = 1 << 22) -> np.ndarray:
    """``n`` N(0,1) draws in fp64 (Box-Muller over splitmix64 pairs)."""
    out = np.empty(n, dtype=np.float64)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, chunk):
        p1 = min(npairs, p0 + chunk)
        raw = splitmix64(seed, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
        a = (raw[:, 0] >> np.uint64(11)).astype(np.float64)
        b = (raw[:, 1] >> np.uint64(11)).astype(np.float64)
        u1 = (a + 1.0) * (2.0 ** -53)  # (0, 1]
        u2 = b * (2.0 ** -53)  # [0, 1)
        r = np.sqrt(-2.0 * np.log(u1))
        t = 2.0 * math.pi * u2
        pair = np.stack([r * np.cos(t), r * np.sin(t)], axis=1).reshape(-1)
        lo = 2 * p0
        hi = min(n, 2 * p1)
        out[lo:hi] = pair[: hi - lo]
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    with np.errstate(over="ignore"):
        return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return f32_to_bf16_bits(normal_f64(seed, n).astype(np.float32)).reshape(shape)


def quantize_int8_per_token(x_bits: np.ndarray):
    """bf16 bits ``[B, S, H, D]`` -> (int8 codes ``[B, S, H, D]``, fp32 scales ``[B, H, S]``)."""
    x = bf16_bits_to_f32(x_bits)
    amax = np.max(np.abs(x), axis=-1)  # [B, S, H], fp32
    sc = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(sc > 0, sc, np.float32(1.0)).astype(np.float32)
    qf = np.rint((x / safe[..., None]).astype(np.float32))
    q = np.clip(qf, -127, 127).astype(np.int8)
    q[sc == 0] = 0
    return q, np.ascontiguousarray(np.transpose(sc, (0, 2, 1)))


def quantize_int4_per_token(x_bits: np.ndarray):
    """bf16 bits ``[B, S, H, D]`` -> (packed uint8 ``[B, S, H, D/2]``, fp32 scales ``[B, H, S]``).
    Symmetric INT4: scale = max|x| / 7 per (token, head), codes clamp(rint(x / scale), -7, 7)
    (fp32 division, ties to even), two codes per byte: dim 2i in the low nibble, dim 2i+1 in the
    high nibble, 4-bit two's complement."""
    x = bf16_bits_to_f32(x_bits)
    amax = np.max(np.abs(x), axis=-1)
    sc = (amax / np.float32(7.0)).astype(np.float32)
    safe = np.where(sc > 0, sc, np.float32(1.0)).astype(np.float32)
    qf = np.rint((x / safe[..., None]).astype(np.float32))
    q = np.clip(qf, -7, 7).astype(np.int8)
    q[sc == 0] = 0
    nib = (q.astype(np.int16) & 0xF).astype(np.uint8)
    packed = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    return packed, np.ascontiguousarray(np.transpose(sc, (0, 2, 1)))


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int
    D: int
    causal: int
    window: int = 0
    int8_kv: bool = False
    num_splits: int = 1
    note: str = ""

    @property
    def scale(self) -> float:
        """1/sqrt(D) rounded to fp32, the value both sides receive."""
        return float(np.float32(1.0 / math.sqrt(self.D)))

    def seed(self, tensor_index: int) -> int:
        return 20260 + 10 * self.index + tensor_index

    def q_shape(self):
        return (self.B, self.Sq, self.Hq, self.D)

    def kv_shape(self):
        return (self.B, self.Skv, self.Hkv, self.D)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 2, 2, 128, 128, 64, 0,
                     note="tiny MHA, non-causal, parity only"),
    "mha_causal": Workload("mha_causal", 2, 2, 32, 32, 4096, 4096, 128, 1,
                           note="MHA prefill, Llama-2-7B-like heads"),
    "gqa_causal": Workload("gqa_causal", 3, 1, 32, 8, 4096, 4096, 128, 1,
                           note="GQA prefill, Mistral-7B-like heads"),
    "gqa_sw512": Workload("gqa_sw512", 3, 1, 32, 8, 4096, 4096, 128, 1, window=512,
                          note="GQA prefill with a 512-key sliding window"),
    "mqa_causal": Workload("mqa_causal", 4, 1, 232, 1, 2048, 2048, 64, 1,
                           note="MQA prefill, Falcon-180B-like head layout"),
    "decode_int8": Workload("decode_int8", 5, 16, 32, 8, 1, 32768, 128, 1, int8_kv=True,
                            num_splits=16, note="GQA decode over an INT8 KV cache"),
    "decode_int4": Workload("decode_int4", 8, 16, 32, 8, 1, 32768, 128, 1, num_splits=16,
                            note="GQA decode over an INT4 KV cache (two codes per byte)"),
}


def make_qkv(w: Workload, q_seed=None, k_seed=None, v_seed=None):
    """bf16 bit patterns for Q, K, V of a workload (K, V in bf16 before any quantisation)."""
    q = normal_bf16(w.seed(0) if q_seed is None else q_seed, w.q_shape())
    k = normal_bf16(w.seed(1) if k_seed is None else k_seed, w.kv_shape())
    v = normal_bf16(w.seed(2) if v_seed is None else v_seed, w.kv_shape())
    return q, k, v


def make_decode_inputs(w: Workload):
    """Q bf16 bits [B,1,Hq,D]; K, V int8 [B,Skv,Hkv,D]; k/v scales fp32 [B,Hkv,Skv]."""
    q, k, v = make_qkv(w)
    kq, ks = quantize_int8_per_token(k)
    vq, vs = quantize_int8_per_token(v)
    return q, kq, vq, ks, vs


def make_decode_int4_inputs(w: Workload):
    """Q bf16 bits [B,1,Hq,D]; K, V packed INT4 uint8 [B,Skv,Hkv,D/2]; scales fp32 [B,Hkv,Skv]."""
    q, k, v = make_qkv(w)
    k4, ks = quantize_int4_per_token(k)
    v4, vs = quantize_int4_per_token(v)
    return q, k4, v4, ks, vs


# ---------------------------------------------------------------------------------------
# The same generator in torch (any device): used for workloads too large to draw in numpy.
# Integer steps are identical; the fp64 log/cos/sin of the device library may differ from
# numpy's in the last bit, so a value can (rarely) round to a neighbouring bf16.  Each test or
# benchmark draws its inputs once and hands the same tensors to both sides.
# ---------------------------------------------------------------------------------------
def _i64(u: int) -> int:
    u &= 0xFFFFFFFFFFFFFFFF
    return u - (1 << 64) if u >= 1 << 63 else u


def _lsr(z, k):
    import torch
    return (z >> k) & ((1 << (64 - k)) - 1)


def splitmix64_torch(seed: int, start: int, count: int, device="cpu"):
    import torch
    idx = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = idx * _i64(0x9E3779B97F4A7C15) + _i64(seed)
    z = (z ^ _lsr(z, 30)) * _i64(0xBF58476D1CE4E5B9)
    z = (z ^ _lsr(z, 27)) * _i64(0x94D049BB133111EB)
    return z ^ _lsr(z, 31)


def normal_bf16_torch(seed: int, shape, device="cpu", chunk: int = 1 << 24):
    """bf16 tensor of N(0,1) draws from the same stream as ``normal_bf16``."""
    import torch
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, chunk):
        p1 = min(npairs, p0 + chunk)
        raw = splitmix64_torch(seed, 2 * p0, 2 * (p1 - p0), device).view(-1, 2)
        a = _lsr(raw[:, 0], 11).to(torch.float64)
        b = _lsr(raw[:, 1], 11).to(torch.float64)
        u1 = (a + 1.0) * (2.0 ** -53)
        u2 = b * (2.0 ** -53)
        r = torch.sqrt(-2.0 * torch.log(u1))
        t = (2.0 * math.pi) * u2
        pair = torch.stack([r * torch.cos(t), r * torch.sin(t)], dim=1).reshape(-1)
        lo, hi = 2 * p0, min(n, 2 * p1)
        out[lo:hi] = pair[: hi - lo].to(torch.float32).to(torch.bfloat16)
        del raw, a, b, u1, u2, r, t, pair
    return out.view(*shape)


def quantize_int8_per_token_torch(x):
    """torch version of ``quantize_int8_per_token``: bf16 [B,S,H,D] -> (int8 [B,S,H,D],
    fp32 scales [B,H,S])."""
    import torch
    xf = x.to(torch.float32)
    amax = xf.abs().amax(dim=-1)
    sc = amax / 127.0
    safe = torch.where(sc > 0, sc, torch.ones_like(sc))
    q = torch.clamp(torch.round(xf / safe[..., None]), -127, 127).to(torch.int8)
    q[sc == 0] = 0
    return q, sc.permute(0, 2, 1).contiguous()


def quantize_int4_per_token_torch(x):
    """torch version of ``quantize_int4_per_token``: bf16 [B,S,H,D] -> (uint8 [B,S,H,D/2],
    fp32 scales [B,H,S])."""
    import torch
    xf = x.to(torch.float32)
    amax = xf.abs().amax(dim=-1)
    sc = amax / 7.0
    safe = torch.where(sc > 0, sc, torch.ones_like(sc))
    q = torch.clamp(torch.round(xf / safe[..., None]), -7, 7).to(torch.int16)
    q[sc == 0] = 0
    nib = (q & 0xF).to(torch.uint8)
    packed = nib[..., 0::2] | (nib[..., 1::2] << 4)
    return packed.contiguous(), sc.permute(0, 2, 1).contiguous()


def make_qkv_torch(w: Workload, device):
    return (normal_bf16_torch(w.seed(0), w.q_shape(), device),
            normal_bf16_torch(w.seed(1), w.kv_shape(), device),
            normal_bf16_torch(w.seed(2), w.kv_shape(), device))


def make_decode_int4_inputs_torch(w: Workload, device):
    q = normal_bf16_torch(w.seed(0), w.q_shape(), device)
    k4, ks = quantize_int4_per_token_torch(normal_bf16_torch(w.seed(1), w.kv_shape(), device))
    v4, vs = quantize_int4_per_token_torch(normal_bf16_torch(w.seed(2), w.kv_shape(), device))
    return q, k4, v4, ks, vs


def make_decode_inputs_torch(w: Workload, device):
    q = normal_bf16_torch(w.seed(0), w.q_shape(), device)
    kq, ks = quantize_int8_per_token_torch(normal_bf16_torch(w.seed(1), w.kv_shape(), device))
    vq, vs = quantize_int8_per_token_torch(normal_bf16_torch(w.seed(2), w.kv_shape(), device))
    return q, kq, vq, ks, vs


def sample_rows(B: int, H: int, S: int, seed: int, n_random: int, window: int = 0):
    """Deterministic row sample (b, h, i): the first and last 64 rows of every (b, h)
    capped by S, the window edges, and ``n_random`` rows drawn from splitmix64."""
    fixed = set()
    edge = [i for i in range(min(64, S))] + [i for i in range(max(0, S - 64), S)]
    if window > 0:
        edge += [i for i in (window - 2, window - 1, window, window + 1) if 0 <= i < S]
    for b in range(B):
        for h in range(H):
            for i in edge[:: max(1, len(edge) // 8)]:
                fixed.add((b, h, i))
    for b in range(B):
        fixed.add((b, 0, 0))
        fixed.add((b, H - 1, S - 1))
    raw = splitmix64(seed, 0, 3 * n_random).reshape(-1, 3)
    for r in raw:
        fixed.add((int(r[0] % np.uint64(B)), int(r[1] % np.uint64(H)), int(r[2] % np.uint64(S))))
    rows = np.array(sorted(fixed), dtype=np.int64)
    return rows


# ---------------------------------------------------------------------------------------
# Paged KV cache with per-sequence lengths.
# Layouts: K/V pages int8 [num_pages, P, Hkv, D]; scales fp32 [num_pages, Hkv, P];
# block_table int32 [B, max_pages] (entries past a sequence's last page are -1 and unused);
# seqlens int32 [B].
# ---------------------------------------------------------------------------------------
@dataclass(frozen=True)
class PagedDecodeWorkload:
    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    D: int
    page_size: int
    min_len: int
    max_len: int
    num_splits: int = 16
    note: str = ""

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.D)))

    @property
    def max_pages(self) -> int:
        return -(-self.max_len // self.page_size)

    def seed(self, tensor_index: int) -> int:
        return 20260 + 10 * self.index + tensor_index


PAGED_WORKLOADS = {
    "decode_int8_paged": PagedDecodeWorkload(
        "decode_int8_paged", 6, 16, 32, 8, 128, 64, 1, 32768, 8,
        note="GQA decode over a paged INT8 cache, lengths uniform in [1, 32768]"),
}


def paged_layout(w: PagedDecodeWorkload, seqlens=None):
    """(seqlens int32 [B], block_table int32 [B, max_pages], num_pages).  ``seqlens`` may be
    given explicitly; otherwise it is drawn uniformly from [min_len, max_len]."""
    if seqlens is None:
        u = splitmix64(w.seed(3), 0, w.B)
        span = np.uint64(w.max_len - w.min_len + 1)
        seqlens = (np.uint64(w.min_len) + u % span).astype(np.int64)
    seqlens = np.asarray(seqlens, dtype=np.int64)
    assert seqlens.shape == (w.B,) and seqlens.min() >= 0 and seqlens.max() <= w.max_len
    npages = -(-seqlens // w.page_size)
    num_pages = max(1, int(npages.sum()))
    perm = np.argsort(splitmix64(w.seed(4), 0, num_pages), kind="stable").astype(np.int32)
    bt = np.full((w.B, w.max_pages), -1, dtype=np.int32)
    off = 0
    for b in range(w.B):
        bt[b, : npages[b]] = perm[off: off + npages[b]]
        off += int(npages[b])
    return seqlens.astype(np.int32), bt, num_pages


def make_paged_decode_inputs(w: PagedDecodeWorkload, seqlens=None, bits: int = 8):
    """q bf16 bits [B,1,Hq,D]; K/V code pages (int8, or packed INT4 uint8 with ``bits=4``),
    fp32 scale pages, block_table, seqlens."""
    sl, bt, num_pages = paged_layout(w, seqlens)
    q = normal_bf16(w.seed(0), (w.B, 1, w.Hq, w.D))
    shape = (num_pages, w.page_size, w.Hkv, w.D)
    quant = quantize_int8_per_token if bits == 8 else quantize_int4_per_token
    kp, ksp = quant(normal_bf16(w.seed(1), shape))
    vp, vsp = quant(normal_bf16(w.seed(2), shape))
    return q, kp, vp, ksp, vsp, bt, sl


def make_paged_decode_inputs_torch(w: PagedDecodeWorkload, device, seqlens=None, bits: int = 8):
    """The same inputs drawn with the torch generator on ``device`` (large workloads)."""
    import torch
    sl, bt, num_pages = paged_layout(w, seqlens)
    q = normal_bf16_torch(w.seed(0), (w.B, 1, w.Hq, w.D), device)
    shape = (num_pages, w.page_size, w.Hkv, w.D)
    quant = quantize_int8_per_token_torch if bits == 8 else quantize_int4_per_token_torch
    kp, ksp = quant(normal_bf16_torch(w.seed(1), shape, device))
    vp, vsp = quant(normal_bf16_torch(w.seed(2), shape, device))
    return (q, kp, vp, ksp, vsp, torch.from_numpy(bt).to(device),
            torch.from_numpy(sl).to(device))
