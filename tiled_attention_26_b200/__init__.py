"""Python binding of ``libfa.so``, the fused tiled attention library for B200 (sm_100a).

The functions carry the C names of ``include/fa.h`` and only marshal arguments: they check
dtypes, shapes and devices of torch tensors, allocate outputs when none are given (torch is the
device-memory allocator here), and pass raw pointers and sizes to the C ABI.  Every step of the
computation runs in the library's CUDA kernels.  If ``libfa.so`` is missing or cannot be loaded,
every call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = ["FaError", "lib", "fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_decode_int8", "fa_decode_int8_paged",
           "fa_decode_int4", "fa_decode_int4_paged", "fa_decode_int8_workspace_bytes",
           "fa_status_string", "fa_device_status", "fa_selftest_bounded_wait", "LIB_PATH",
           "STATUS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")

STATUS = {
    "FA_OK": 0,
    "FA_ERR_INVALID_ARG": -1,
    "FA_ERR_UNSUPPORTED": -2,
    "FA_ERR_ALIGNMENT": -3,
    "FA_ERR_WORKSPACE": -4,
    "FA_ERR_CUDA": -5,
    "FA_ERR_TIMEOUT": -6,
    "FA_ERR_DEVICE_INDEX": -7,
}


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fa_status_string(status)} ({status})")


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """The loaded C library, with argument types declared.  Raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libfa.so is not built ({LIB_PATH}); run "
                               "`python tiled_attention_26_b200/build.py`")
        L = ctypes.CDLL(LIB_PATH)
        L.fa_fwd.argtypes = [_P, _P, _P, _P, _P] + [_I] * 6 + [_F, _I, _I, _P]
        L.fa_fwd.restype = _I
        L.fa_fwd_ext.argtypes = ([_P, _P, _P, _P, _P] + [_I] * 6 + [_F, _I, _I, _I, _P,
                                 ctypes.c_int64, ctypes.c_int64, _P])
        L.fa_fwd_ext.restype = _I
        L.fa_bwd_workspace_bytes.argtypes = [_I, _I, _I]
        L.fa_bwd_workspace_bytes.restype = _Z
        L.fa_bwd.argtypes = [_P] * 9 + [_I] * 6 + [_F, _I, _I, _P, _Z, _P]
        L.fa_bwd.restype = _I
        L.fa_decode_int8_workspace_bytes.argtypes = [_I, _I, _I, _I]
        L.fa_decode_int8_workspace_bytes.restype = _Z
        L.fa_decode_int8.argtypes = [_P] * 7 + [_I] * 5 + [_F, _I, _P, _Z, _P]
        L.fa_decode_int8.restype = _I
        L.fa_decode_int8_paged.argtypes = [_P] * 9 + [_I] * 7 + [_F, _I, _P, _Z, _P]
        L.fa_decode_int8_paged.restype = _I
        L.fa_decode_int4.argtypes = [_P] * 7 + [_I] * 5 + [_F, _I, _P, _Z, _P]
        L.fa_decode_int4.restype = _I
        L.fa_decode_int4_paged.argtypes = [_P] * 9 + [_I] * 7 + [_F, _I, _P, _Z, _P]
        L.fa_decode_int4_paged.restype = _I
        L.fa_status_string.argtypes = [_I]
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_device_status.argtypes = [_P]
        L.fa_device_status.restype = _I
        L.fa_selftest_bounded_wait.argtypes = [_I, _P]
        L.fa_selftest_bounded_wait.restype = _I
        _lib = L
    return _lib


def fa_status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, dtype, shape, device):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def fa_fwd(q, k, v, causal: bool = False, window: int = 0, scale: float | None = None,
           o=None, lse=None, return_lse: bool = True, stream=None, n_global: int = 0,
           mask=None):
    """Attention forward.  q: bf16 [B, Sq, Hq, D] on CUDA; k, v: bf16 [B, Skv, Hkv, D].
    ``n_global``: the first n_global positions attend to, and are attended by, every position.
    ``mask``: optional fp32 additive mask [Bm, Hm, Sq, Skv] with Bm in {1, B}, Hm in {1, Hq}
    (size-1 dims broadcast), added to scale * q.k; -inf drops a key.

    Returns ``(o, lse)``: o bf16 [B, Sq, Hq, D], lse fp32 [B, Hq, Sq] (natural log; None when
    ``return_lse`` is false and no ``lse`` buffer is given)."""
    import torch
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, S, H, D]")
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    _check(q, "q", torch.bfloat16, (B, Sq, Hq, D), dev)
    _check(k, "k", torch.bfloat16, (B, Skv, Hkv, D), dev)
    _check(v, "v", torch.bfloat16, (B, Skv, Hkv, D), dev)
    if o is None:
        o = torch.empty_like(q)
    _check(o, "o", torch.bfloat16, (B, Sq, Hq, D), dev)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, Hq, Sq), dev)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    sb = sh = 0
    if mask is not None:
        if mask.dim() != 4 or mask.shape[0] not in (1, B) or mask.shape[1] not in (1, Hq):
            raise ValueError("mask must be [1 or B, 1 or Hq, Sq, Skv]")
        _check(mask, "mask", torch.float32, (mask.shape[0], mask.shape[1], Sq, Skv), dev)
        sh = Sq * Skv if mask.shape[1] == Hq else 0
        sb = Sq * Skv * mask.shape[1] if mask.shape[0] == B else 0
    rc = lib().fa_fwd_ext(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                          lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Sq, Skv, D,
                          float(scale), int(bool(causal)), int(window), int(n_global),
                          mask.data_ptr() if mask is not None else None, sb, sh,
                          _stream_ptr(stream))
    if rc != 0:
        raise FaError(rc, "fa_fwd")
    return o, lse


def fa_bwd_workspace_bytes(B: int, Hq: int, Sq: int) -> int:
    return int(lib().fa_bwd_workspace_bytes(int(B), int(Hq), int(Sq)))


def fa_bwd(q, k, v, o, dout, lse, causal: bool = False, window: int = 0,
           scale: float | None = None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward pass of fa_fwd: gradients of sum(dout * o).  q, o, dout: bf16 [B, Sq, Hq, D];
    k, v: bf16 [B, Skv, Hkv, D]; lse: fp32 [B, Hq, Sq] from fa_fwd.  Returns (dq, dk, dv)."""
    import torch
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    _check(q, "q", torch.bfloat16, (B, Sq, Hq, D), dev)
    _check(k, "k", torch.bfloat16, (B, Skv, Hkv, D), dev)
    _check(v, "v", torch.bfloat16, (B, Skv, Hkv, D), dev)
    _check(o, "o", torch.bfloat16, (B, Sq, Hq, D), dev)
    _check(dout, "dout", torch.bfloat16, (B, Sq, Hq, D), dev)
    _check(lse, "lse", torch.float32, (B, Hq, Sq), dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq, "dq", torch.bfloat16, (B, Sq, Hq, D), dev)
    _check(dk, "dk", torch.bfloat16, (B, Skv, Hkv, D), dev)
    _check(dv, "dv", torch.bfloat16, (B, Skv, Hkv, D), dev)
    need = fa_bwd_workspace_bytes(B, Hq, Sq)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rc = lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                      lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv,
                      Sq, Skv, D, float(scale), int(bool(causal)), int(window),
                      workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                      _stream_ptr(stream))
    if rc != 0:
        raise FaError(rc, "fa_bwd")
    return dq, dk, dv


def fa_decode_int8_workspace_bytes(B: int, Hq: int, D: int, num_splits: int) -> int:
    return int(lib().fa_decode_int8_workspace_bytes(int(B), int(Hq), int(D), int(num_splits)))


def _decode(bits, q, k, v, k_scale, v_scale, num_splits, scale, o, lse, workspace, return_lse,
            stream):
    import torch
    name = f"fa_decode_int{bits}"
    B, one, Hq, D = q.shape
    if one != 1:
        raise ValueError("decode takes one query token per sequence")
    Skv, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    code = torch.int8 if bits == 8 else torch.uint8
    row = D if bits == 8 else D // 2
    _check(q, "q", torch.bfloat16, (B, 1, Hq, D), dev)
    _check(k, "k", code, (B, Skv, Hkv, row), dev)
    _check(v, "v", code, (B, Skv, Hkv, row), dev)
    _check(k_scale, "k_scale", torch.float32, (B, Hkv, Skv), dev)
    _check(v_scale, "v_scale", torch.float32, (B, Hkv, Skv), dev)
    if o is None:
        o = torch.empty_like(q)
    _check(o, "o", torch.bfloat16, (B, 1, Hq, D), dev)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, Hq), dev)
    need = fa_decode_int8_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rc = getattr(lib(), name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), k_scale.data_ptr(),
                              v_scale.data_ptr(), o.data_ptr(),
                              lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Skv, D,
                              float(scale), int(num_splits), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if rc != 0:
        raise FaError(rc, name)
    return o, lse


def fa_decode_int8(q, k, v, k_scale, v_scale, num_splits: int = 16, scale: float | None = None,
                   o=None, lse=None, workspace=None, return_lse: bool = True, stream=None):
    """Decode step over an INT8 KV cache.  q: bf16 [B, 1, Hq, D]; k, v: int8 [B, Skv, Hkv, D];
    k_scale, v_scale: fp32 [B, Hkv, Skv].  Returns ``(o, lse)`` with o bf16 [B, 1, Hq, D] and
    lse fp32 [B, Hq]."""
    return _decode(8, q, k, v, k_scale, v_scale, num_splits, scale, o, lse, workspace,
                   return_lse, stream)


def fa_decode_int4(q, k, v, k_scale, v_scale, num_splits: int = 16, scale: float | None = None,
                   o=None, lse=None, workspace=None, return_lse: bool = True, stream=None):
    """Decode step over an INT4 KV cache.  k, v: uint8 [B, Skv, Hkv, D/2], two 4-bit
    two's-complement codes per byte (dim 2i in the low nibble); otherwise as fa_decode_int8."""
    return _decode(4, q, k, v, k_scale, v_scale, num_splits, scale, o, lse, workspace,
                   return_lse, stream)


def _decode_paged(bits, q, k_pages, v_pages, k_scale_pages, v_scale_pages, block_table, seqlens,
                  num_splits, scale, o, lse, workspace, return_lse, stream):
    import torch
    name = f"fa_decode_int{bits}_paged"
    B, one, Hq, D = q.shape
    if one != 1:
        raise ValueError("decode takes one query token per sequence")
    if k_pages.dim() != 4 or block_table.dim() != 2:
        raise ValueError("k_pages must be [num_pages, P, Hkv, row], block_table [B, max_pages]")
    num_pages, P, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    max_pages = block_table.shape[1]
    dev = q.device
    code = torch.int8 if bits == 8 else torch.uint8
    row = D if bits == 8 else D // 2
    _check(q, "q", torch.bfloat16, (B, 1, Hq, D), dev)
    _check(k_pages, "k_pages", code, (num_pages, P, Hkv, row), dev)
    _check(v_pages, "v_pages", code, (num_pages, P, Hkv, row), dev)
    _check(k_scale_pages, "k_scale_pages", torch.float32, (num_pages, Hkv, P), dev)
    _check(v_scale_pages, "v_scale_pages", torch.float32, (num_pages, Hkv, P), dev)
    _check(block_table, "block_table", torch.int32, (B, max_pages), dev)
    _check(seqlens, "seqlens", torch.int32, (B,), dev)
    if o is None:
        o = torch.empty_like(q)
    _check(o, "o", torch.bfloat16, (B, 1, Hq, D), dev)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, Hq), dev)
    need = fa_decode_int8_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rc = getattr(lib(), name)(
        q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), k_scale_pages.data_ptr(),
        v_scale_pages.data_ptr(), block_table.data_ptr(), seqlens.data_ptr(), o.data_ptr(),
        lse.data_ptr() if lse is not None else None, B, Hq, Hkv, P, max_pages, num_pages, D,
        float(scale), int(num_splits), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if rc != 0:
        raise FaError(rc, name)
    return o, lse


def fa_decode_int8_paged(q, k_pages, v_pages, k_scale_pages, v_scale_pages, block_table,
                         seqlens, num_splits: int = 16, scale: float | None = None, o=None,
                         lse=None, workspace=None, return_lse: bool = True, stream=None):
    """Decode step over a paged INT8 KV cache with one length per sequence.
    q: bf16 [B, 1, Hq, D]; k_pages, v_pages: int8 [num_pages, P, Hkv, D]; k_scale_pages,
    v_scale_pages: fp32 [num_pages, Hkv, P]; block_table: int32 [B, max_pages]; seqlens: int32
    [B] (both on the device).  Returns ``(o, lse)`` with o bf16 [B, 1, Hq, D], lse fp32 [B, Hq]."""
    return _decode_paged(8, q, k_pages, v_pages, k_scale_pages, v_scale_pages, block_table,
                         seqlens, num_splits, scale, o, lse, workspace, return_lse, stream)


def fa_decode_int4_paged(q, k_pages, v_pages, k_scale_pages, v_scale_pages, block_table,
                         seqlens, num_splits: int = 16, scale: float | None = None, o=None,
                         lse=None, workspace=None, return_lse: bool = True, stream=None):
    """Paged, variable-length decode over an INT4 KV cache: k_pages, v_pages uint8
    [num_pages, P, Hkv, D/2] packed as for fa_decode_int4; otherwise as fa_decode_int8_paged."""
    return _decode_paged(4, q, k_pages, v_pages, k_scale_pages, v_scale_pages, block_table,
                         seqlens, num_splits, scale, o, lse, workspace, return_lse, stream)


def fa_device_status(stream=None) -> int:
    return int(lib().fa_device_status(_stream_ptr(stream)))


def fa_selftest_bounded_wait(timeout_us: int, stream=None) -> int:
    return int(lib().fa_selftest_bounded_wait(int(timeout_us), _stream_ptr(stream)))
