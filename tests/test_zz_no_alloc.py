"""The allocation-free decode entry point (fa_decode_int8_noalloc) against the workspace entry
point (fa_decode_int8), through the C ABI, on two calls in a row.

fa_decode_int8_noalloc serves callers that cannot call cudaMalloc where they decode (a memory
manager that owns the whole device budget, latency-critical loops, C callers without an
allocator); it keeps its split partials in a fixed array inside the library instead of a
caller-provided workspace.  Both entry points run the same kernels with the same split plan, so
their outputs must agree bit for bit.  This file is collected last so that, if it fails, a run
that stops at the first failure has already run every other test."""
import ctypes
import math

import numpy as np
import pytest

import synthetic

pytestmark = pytest.mark.gpu

# (B, Hq, Hkv, Skv, D, num_splits): the full decode workload (4.2 MiB of partials), and a small
# ragged one whose fifth split holds no keys.
LONG = (16, 32, 8, 32768, 128, 16)
SHORT = (3, 12, 4, 777, 64, 5)


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


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32)


class _Case:
    """Inputs of one shape and the workspace entry point's outputs on them."""

    def __init__(self, shape, seed):
        import torch
        import tiled_attention_26_b200 as fa
        self.shape = shape
        B, Hq, Hkv, Skv, D, splits = shape
        self.scale = float(np.float32(1 / math.sqrt(D)))
        self.x = _inputs(B, Hq, Hkv, Skv, D, seed)
        self.o_ref, self.l_ref = fa.fa_decode_int8(*self.x, num_splits=splits, scale=self.scale)
        torch.cuda.synchronize()
        self.o = torch.empty_like(self.o_ref)
        self.lse = torch.empty_like(self.l_ref)

    def call_noalloc(self, f):
        """One call of the allocation-free entry point into fresh NaN-filled outputs; returns the
        status code after the stream has finished."""
        import torch
        B, Hq, Hkv, Skv, D, splits = self.shape
        self.o.fill_(float("nan"))
        self.lse.fill_(float("nan"))
        torch.cuda.synchronize()
        q, kq, vq, ks, vs = self.x
        rc = f(q.data_ptr(), kq.data_ptr(), vq.data_ptr(), ks.data_ptr(), vs.data_ptr(),
               self.o.data_ptr(), self.lse.data_ptr(), B, Hq, Hkv, Skv, D, self.scale, splits,
               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        torch.cuda.synchronize()
        return rc

    def assert_bit_equal(self, what):
        import torch
        assert torch.equal(_bits(self.o), _bits(self.o_ref)), f"{what}: O differs"
        assert torch.equal(_bits(self.lse), _bits(self.l_ref)), f"{what}: LSE differs"


@pytest.mark.parametrize("shape", [LONG, SHORT])
def test_noalloc_bit_equal_to_workspace_entry_point(shape):
    import torch
    import tiled_attention_26_b200 as fa
    case = _Case(shape, seed=9100 + shape[4])
    f = _noalloc_fn()
    for call in range(2):
        # the first call may load the module on this device (documented); the second must not
        # change the device's free memory
        free_before = torch.cuda.mem_get_info()[0]
        rc = case.call_noalloc(f)
        free_after = torch.cuda.mem_get_info()[0]
        assert rc == 0, fa.fa_status_string(rc)
        assert fa.fa_device_status() == 0
        case.assert_bit_equal(f"{shape} call {call}")
        if call == 1:
            assert free_after == free_before, "the allocation-free call changed free memory"


def test_noalloc_long_then_short_leaves_no_stale_partials():
    """The scratch array keeps the last call's contents: a short call right after a long one (a
    different partials layout, and a split with no keys) must not read any of it."""
    import tiled_attention_26_b200 as fa
    f = _noalloc_fn()
    long_case, short_case = _Case(LONG, seed=9300), _Case(SHORT, seed=9400)
    for what, case in (("long", long_case), ("short after long", short_case),
                       ("long after short", long_case), ("short again", short_case)):
        rc = case.call_noalloc(f)
        assert rc == 0, fa.fa_status_string(rc)
        assert fa.fa_device_status() == 0
        case.assert_bit_equal(what)


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
