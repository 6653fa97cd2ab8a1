"""The allocation-free decode entry point (fa_decode_int8_noalloc) against the workspace entry
point (fa_decode_int8), through the C ABI, on two calls in a row.

fa_decode_int8_noalloc serves callers that cannot call cudaMalloc where they decode (a memory
manager that owns the whole device budget, latency-critical loops, C callers without an
allocator); it keeps its split partials in a fixed array inside the library instead of a
caller-provided workspace.  This file is collected last so that, if it fails, a run that stops at
the first failure has already run every other test."""
import ctypes
import math

import numpy as np
import pytest

import synthetic
from parity_util import LSE_TOL, O_MAX, O_MEAN

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    import tiled_attention_26_b200 as fa
    f = fa.lib().fa_decode_int8_noalloc
    f.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int,
                                                              ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _inputs(B, Hq, Hkv, Skv, D, seed):
    import torch
    w = synthetic.Workload("noalloc", 0, B, Hq, Hkv, 1, Skv, D, 1)
    q = synthetic.normal_bf16_torch(seed, w.q_shape(), "cuda")
    kq, ks = synthetic.quantize_int8_per_token_torch(
        synthetic.normal_bf16_torch(seed + 1, w.kv_shape(), "cuda"))
    vq, vs = synthetic.quantize_int8_per_token_torch(
        synthetic.normal_bf16_torch(seed + 2, w.kv_shape(), "cuda"))
    torch.cuda.synchronize()
    return q, kq, vq, ks, vs


@pytest.mark.parametrize("shape", [(16, 32, 8, 32768, 128, 16), (3, 12, 4, 777, 64, 5)])
def test_noalloc_matches_workspace_entry_point(shape):
    import torch
    import tiled_attention_26_b200 as fa
    B, Hq, Hkv, Skv, D, splits = shape
    scale = float(np.float32(1 / math.sqrt(D)))
    q, kq, vq, ks, vs = _inputs(B, Hq, Hkv, Skv, D, seed=9100 + D)
    o_ref, l_ref = fa.fa_decode_int8(q, kq, vq, ks, vs, num_splits=splits, scale=scale)
    torch.cuda.synchronize()
    f = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(l_ref, float("nan"))
        rc = f(q.data_ptr(), kq.data_ptr(), vq.data_ptr(), ks.data_ptr(), vs.data_ptr(),
               o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Skv, D, scale, splits, stream)
        assert rc == 0, fa.fa_status_string(rc)
        torch.cuda.synchronize()
        assert fa.fa_device_status() == 0
        err = (o.float() - o_ref.float()).abs()
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert err.max().item() <= O_MAX and err.mean().item() <= O_MEAN, call
        assert (lse - l_ref).abs().max().item() <= LSE_TOL, call


def test_noalloc_rejects_partials_larger_than_its_scratch():
    import torch
    import tiled_attention_26_b200 as fa
    f = _noalloc_fn()
    B, Hq, D, splits = 64, 64, 128, 16  # 32 MiB of partials > the fixed scratch
    assert fa.fa_decode_int8_workspace_bytes(B, Hq, D, splits) > (8 << 20)
    x = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    p = x.data_ptr()
    rc = f(p, p, p, p, p, p, None, B, Hq, 8, 100, D, 0.1, splits,
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == fa.STATUS["FA_ERR_WORKSPACE"]
