"""fp64 CPU oracle for the fused attention path (ctypes wrapper over ``liboracle.so``).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with the CUDA
library, and the CUDA library never calls it.

Every function evaluates the attention definition softmax(Q K^T * scale + mask) V in fp64
("FlashAttention on Ascend NPUs", section on the attention formula); see ``oracle.cpp`` for
the passage each step follows.  Layouts: Q/O ``[B, Sq, Hq, D]``, K/V ``[B, Skv, Hkv, D]``,
LSE ``[B, Hq, Sq]`` (natural log), INT8 scales ``[B, Hkv, Skv]``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
_D = ctypes.c_double


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_max_threads.restype = _I
        L.oracle_attn_bf16_rows.argtypes = [_P, _P, _P] + [_I] * 6 + [_D, _I, _I, _P, _L, _P, _P, _I]
        L.oracle_attn_f64_rows.argtypes = [_P, _P, _P] + [_I] * 6 + [_D, _I, _I, _P, _L, _P, _P, _I]
        L.oracle_attn_brute.argtypes = [_P, _P, _P] + [_I] * 6 + [_D, _I, _I, _P, _P, _P]
        L.oracle_attn_tiled.argtypes = [_P, _P, _P] + [_I] * 6 + [_D, _I, _I, _I, _P, _P]
        L.oracle_decode_int8_rows.argtypes = [_P] * 5 + [_I] * 5 + [_D, _I, _P, _L, _P, _P, _I]
        L.oracle_decode_int8_paged_rows.argtypes = [_P] * 7 + [_I] * 7 + [_D, _I, _P, _L, _P, _P, _I]
        L.oracle_decode_int8_paged_rows.restype = _I
        L.oracle_attn_ext_rows.argtypes = ([_P, _P, _P] + [_I] * 6 + [_D, _I, _I, _I, _P, _L, _L]
                                           + [_P, _L, _P, _P, _I])
        L.oracle_attn_ext_rows.restype = _I
        L.oracle_attn_bwd.argtypes = [_P] * 4 + [_I] * 6 + [_D, _I, _I, _P, _P, _P, _I]
        L.oracle_attn_bwd.restype = _I
        L.oracle_unpack_int4.argtypes = [_P, _L, _P]
        L.oracle_unpack_int4.restype = _I
        for f in (L.oracle_attn_bf16_rows, L.oracle_attn_f64_rows, L.oracle_attn_brute,
                  L.oracle_attn_tiled, L.oracle_decode_int8_rows):
            f.restype = _I
        _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(q, k):
    B, Sq, Hq, D = q.shape
    B2, Skv, Hkv, D2 = k.shape
    assert B == B2 and D == D2
    return B, Hq, Hkv, Sq, Skv, D


def all_rows(B: int, H: int, S: int) -> np.ndarray:
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(S), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1).astype(np.int64)


def attn_rows(q, k, v, scale, causal, window, rows, nthreads=0):
    """Selected rows of the definition.  q/k/v: bf16 bit patterns (uint16) or fp64 arrays.
    rows: (n, 3) int64 array of (b, h, i).  Returns (o [n, D] fp64, lse [n] fp64)."""
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    n = rows.shape[0]
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    if q.dtype == np.uint16:
        f = lib().oracle_attn_bf16_rows
        q, k, v = (np.ascontiguousarray(t, dtype=np.uint16) for t in (q, k, v))
    else:
        f = lib().oracle_attn_f64_rows
        q, k, v = (np.ascontiguousarray(t, dtype=np.float64) for t in (q, k, v))
    rc = f(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D, float(scale), int(causal),
           int(window), _ptr(rows), n, _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attn_rows rejected its arguments")
    return o, lse


def attn(q, k, v, scale, causal=0, window=0, nthreads=0):
    """Full output by the definition: (O [B,Sq,Hq,D], LSE [B,Hq,Sq]) in fp64."""
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    rows = all_rows(B, Hq, Sq)
    o, lse = attn_rows(q, k, v, scale, causal, window, rows, nthreads)
    return (o.reshape(B, Hq, Sq, D).transpose(0, 2, 1, 3).copy(), lse.reshape(B, Hq, Sq))


def attn_brute(q, k, v, scale, causal=0, window=0, want_probs=False):
    """The naive multi-pass form with the full score matrix (fp64 inputs, small shapes)."""
    q, k, v = (np.ascontiguousarray(t, dtype=np.float64) for t in (q, k, v))
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    o = np.zeros((B, Sq, Hq, D))
    lse = np.zeros((B, Hq, Sq))
    probs = np.zeros((B, Hq, Sq, Skv)) if want_probs else None
    rc = lib().oracle_attn_brute(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D, float(scale),
                                 int(causal), int(window), _ptr(o), _ptr(lse),
                                 _ptr(probs) if want_probs else None)
    if rc != 0:
        raise ValueError("oracle_attn_brute rejected its arguments")
    return (o, lse, probs) if want_probs else (o, lse)


def attn_tiled(q, k, v, scale, causal=0, window=0, tile=128):
    """Tiled online-softmax evaluation (fp64 inputs)."""
    q, k, v = (np.ascontiguousarray(t, dtype=np.float64) for t in (q, k, v))
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    o = np.zeros((B, Sq, Hq, D))
    lse = np.zeros((B, Hq, Sq))
    rc = lib().oracle_attn_tiled(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D, float(scale),
                                 int(causal), int(window), int(tile), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_tiled rejected its arguments")
    return o, lse


def decode_int8_rows(q, kq, vq, ks, vs, scale, num_splits, rows, nthreads=0):
    """Decode over an INT8 KV cache.  q: bf16 bits [B,1,Hq,D]; kq/vq: int8 [B,Skv,Hkv,D];
    ks/vs: fp32 [B,Hkv,Skv]; rows: (n, 2) int64 (b, h).  Returns (o [n,D], lse [n])."""
    B, one, Hq, D = q.shape
    assert one == 1
    _, Skv, Hkv, _ = kq.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    n = rows.shape[0]
    o = np.zeros((n, D))
    lse = np.zeros(n)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    kq, vq = (np.ascontiguousarray(t, dtype=np.int8) for t in (kq, vq))
    ks, vs = (np.ascontiguousarray(t, dtype=np.float32) for t in (ks, vs))
    rc = lib().oracle_decode_int8_rows(_ptr(q), _ptr(kq), _ptr(vq), _ptr(ks), _ptr(vs), B, Hq, Hkv,
                                       Skv, D, float(scale), int(num_splits), _ptr(rows), n,
                                       _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode_int8_rows rejected its arguments")
    return o, lse


def decode_int8(q, kq, vq, ks, vs, scale, num_splits=1, nthreads=0):
    """All (b, h) of a decode step: (O [B,1,Hq,D], LSE [B,Hq])."""
    B, _, Hq, D = q.shape
    b, h = np.meshgrid(np.arange(B), np.arange(Hq), indexing="ij")
    rows = np.stack([b.ravel(), h.ravel()], axis=1).astype(np.int64)
    o, lse = decode_int8_rows(q, kq, vq, ks, vs, scale, num_splits, rows, nthreads)
    return o.reshape(B, 1, Hq, D), lse.reshape(B, Hq)


def decode_int8_paged_rows(q, kp, vp, ksp, vsp, block_table, seqlens, scale, num_splits, rows,
                           nthreads=0):
    """Decode over a paged INT8 KV cache with per-sequence lengths.  q: bf16 bits [B,1,Hq,D];
    kp/vp: int8 [num_pages,P,Hkv,D]; ksp/vsp: fp32 [num_pages,Hkv,P]; block_table: int32
    [B,max_pages]; seqlens: int32 [B]; rows: (n, 2) (b, h).  Returns (o [n,D], lse [n])."""
    B, _, Hq, D = q.shape
    num_pages, P, Hkv, _ = kp.shape
    max_pages = block_table.shape[1]
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    n = rows.shape[0]
    o = np.zeros((n, D))
    lse = np.zeros(n)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    kp, vp = (np.ascontiguousarray(t, dtype=np.int8) for t in (kp, vp))
    ksp, vsp = (np.ascontiguousarray(t, dtype=np.float32) for t in (ksp, vsp))
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    rc = lib().oracle_decode_int8_paged_rows(_ptr(q), _ptr(kp), _ptr(vp), _ptr(ksp), _ptr(vsp),
                                             _ptr(bt), _ptr(sl), B, Hq, Hkv, P, max_pages,
                                             num_pages, D, float(scale), int(num_splits),
                                             _ptr(rows), n, _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode_int8_paged_rows rejected its arguments")
    return o, lse


def decode_int8_paged(q, kp, vp, ksp, vsp, block_table, seqlens, scale, num_splits=1, nthreads=0):
    B, _, Hq, D = q.shape
    b, h = np.meshgrid(np.arange(B), np.arange(Hq), indexing="ij")
    rows = np.stack([b.ravel(), h.ravel()], axis=1).astype(np.int64)
    o, lse = decode_int8_paged_rows(q, kp, vp, ksp, vsp, block_table, seqlens, scale, num_splits,
                                    rows, nthreads)
    return o.reshape(B, 1, Hq, D), lse.reshape(B, Hq)


def unpack_int4(packed):
    """Packed INT4 codes (uint8 [..., n]) -> int8 codes [..., 2n]: byte i holds code 2i in its low
    nibble and code 2i+1 in its high nibble, 4-bit two's complement."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    codes = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), dtype=np.int8)
    if lib().oracle_unpack_int4(_ptr(packed), packed.size, _ptr(codes)) != 0:
        raise ValueError("oracle_unpack_int4 rejected its arguments")
    return codes


def decode_int4_rows(q, k4, v4, ks, vs, scale, num_splits, rows, nthreads=0):
    """Decode over an INT4 KV cache: k4/v4 uint8 [B, Skv, Hkv, D/2] packed codes, ks/vs fp32
    [B, Hkv, Skv].  The INT8 decode definition over the unpacked codes."""
    return decode_int8_rows(q, unpack_int4(k4), unpack_int4(v4), ks, vs, scale, num_splits, rows,
                            nthreads)


def decode_int4(q, k4, v4, ks, vs, scale, num_splits=1, nthreads=0):
    return decode_int8(q, unpack_int4(k4), unpack_int4(v4), ks, vs, scale, num_splits, nthreads)


def decode_int4_paged(q, kp4, vp4, ksp, vsp, block_table, seqlens, scale, num_splits=1,
                      nthreads=0):
    return decode_int8_paged(q, unpack_int4(kp4), unpack_int4(vp4), ksp, vsp, block_table,
                             seqlens, scale, num_splits, nthreads)


def attn_ext_rows(q, k, v, scale, causal, window, n_global, mask, rows, nthreads=0):
    """Rows of the definition with an additive mask and global tokens.  q/k/v: bf16 bits;
    mask: fp32 array broadcastable to [B, Hq, Sq, Skv] (leading dims of size 1 broadcast) or
    None; rows: (n, 3) (b, h, i).  Returns (o [n, D], lse [n])."""
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    n = rows.shape[0]
    o = np.zeros((n, D))
    lse = np.zeros(n)
    q, k, v = (np.ascontiguousarray(t, dtype=np.uint16) for t in (q, k, v))
    sb = sh = 0
    mptr = None
    if mask is not None:
        mask = np.ascontiguousarray(mask, dtype=np.float32)
        assert mask.ndim == 4 and mask.shape[2:] == (Sq, Skv)
        assert mask.shape[0] in (1, B) and mask.shape[1] in (1, Hq)
        sb = Sq * Skv * mask.shape[1] if mask.shape[0] == B else 0
        sh = Sq * Skv if mask.shape[1] == Hq else 0
        mptr = _ptr(mask)
    rc = lib().oracle_attn_ext_rows(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Skv, D,
                                    float(scale), int(causal), int(window), int(n_global), mptr,
                                    sb, sh, _ptr(rows), n, _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attn_ext_rows rejected its arguments")
    return o, lse


def attn_ext(q, k, v, scale, causal=0, window=0, n_global=0, mask=None, nthreads=0):
    """Full output: (O [B,Sq,Hq,D], LSE [B,Hq,Sq])."""
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    o, lse = attn_ext_rows(q, k, v, scale, causal, window, n_global, mask, all_rows(B, Hq, Sq),
                           nthreads)
    return (o.reshape(B, Hq, Sq, D).transpose(0, 2, 1, 3).copy(), lse.reshape(B, Hq, Sq))


def attn_bwd(q, k, v, dout, scale, causal=0, window=0, nthreads=0):
    """Gradients (dQ [B,Sq,Hq,D], dK, dV [B,Skv,Hkv,D]) of sum(dout * O) for the definition, in
    fp64, from bf16 bit patterns."""
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    q, k, v, dout = (np.ascontiguousarray(t, dtype=np.uint16) for t in (q, k, v, dout))
    dq = np.zeros((B, Sq, Hq, D))
    dk = np.zeros((B, Skv, Hkv, D))
    dv = np.zeros((B, Skv, Hkv, D))
    rc = lib().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, Hq, Hkv, Sq, Skv, D,
                               float(scale), int(causal), int(window), _ptr(dq), _ptr(dk),
                               _ptr(dv), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attn_bwd rejected its arguments")
    return dq, dk, dv
