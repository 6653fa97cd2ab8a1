"""Host-only checks of the C ABI: the library loads without a GPU, exports every function that
include/fa.h declares, and rejects bad arguments with the documented status codes before it
touches the device."""
import ctypes
import os
import re

import pytest

import tiled_attention_26_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails before any CUDA call


@pytest.fixture(scope="module")
def L():
    from tiled_attention_26_b200 import build
    build.build()
    return fa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*FA_API\s+(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fa_fwd", "fa_decode_int8", "fa_decode_int8_workspace_bytes", "fa_status_string",
              "fa_device_status", "fa_selftest_bounded_wait", "fa_decode_int8_noalloc",
              "fa_decode_int8_paged", "fa_decode_int4", "fa_decode_int4_paged", "fa_fwd_ext", "fa_bwd",
              "fa_bwd_workspace_bytes"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_codes_match_header():
    text = open(HEADER).read()
    for name, value in fa.STATUS.items():
        assert re.search(rf"\b{name}\s*=\s*{value}\b", text), name


def test_status_strings(L):
    for name, value in fa.STATUS.items():
        assert fa.fa_status_string(value).startswith(name)
    assert fa.fa_status_string(12345) == "unknown fa_status"


def fwd(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=2, Hkv=2, Sq=128, Skv=128, D=64,
        scale=0.125, causal=0, window=0):
    return L.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, window, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(o=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(B=0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(Sq=-1), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(Hq=6, Hkv=4), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(window=16), fa.STATUS["FA_ERR_INVALID_ARG"]),          # window needs causal
    (dict(window=-1, causal=1), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(causal=2), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(scale=0.0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(scale=float("nan")), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(scale=float("inf")), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(D=96), fa.STATUS["FA_ERR_UNSUPPORTED"]),
    (dict(D=256), fa.STATUS["FA_ERR_UNSUPPORTED"]),
    (dict(q=FAKE + 8), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(o=FAKE + 2), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(lse=FAKE + 1), fa.STATUS["FA_ERR_ALIGNMENT"]),
])
def test_fwd_rejects(L, kw, code):
    assert fwd(L, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(n_global=-1), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(sb=-4), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(mask=FAKE + 4), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(window=8), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(D=32), fa.STATUS["FA_ERR_UNSUPPORTED"]),
])
def test_fwd_ext_rejects(L, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=2, Hkv=2, Sq=128, Skv=128, D=64,
             scale=0.125, causal=0, window=0, n_global=0, mask=FAKE, sb=0, sh=0)
    a.update(kw)
    assert L.fa_fwd_ext(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                        a["Sq"], a["Skv"], a["D"], a["scale"], a["causal"], a["window"],
                        a["n_global"], a["mask"], a["sb"], a["sh"], None) == code


@pytest.mark.parametrize("kw,code", [
    (dict(lse=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(dk=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(window=4), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(D=80), fa.STATUS["FA_ERR_UNSUPPORTED"]),
    (dict(dq=FAKE + 8), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(ws_bytes=64), fa.STATUS["FA_ERR_WORKSPACE"]),
])
def test_bwd_rejects(L, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, do=FAKE, lse=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1,
             Hq=2, Hkv=2, Sq=128, Skv=128, D=64, scale=0.125, causal=0, window=0, ws=FAKE,
             ws_bytes=None)
    a.update(kw)
    if a["ws_bytes"] is None:
        a["ws_bytes"] = L.fa_bwd_workspace_bytes(a["B"], a["Hq"], a["Sq"])
    assert L.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"],
                    a["B"], a["Hq"], a["Hkv"], a["Sq"], a["Skv"], a["D"], a["scale"], a["causal"],
                    a["window"], a["ws"], a["ws_bytes"], None) == code


def test_bwd_workspace_bytes(L):
    # -L log2(e) and -D per padded row, then the fp32 dQ accumulator [B, Sq, Hq, 128]
    assert fa.fa_bwd_workspace_bytes(2, 4, 300) == 2 * 2 * 4 * 384 * 4 + 2 * 300 * 4 * 128 * 4
    assert fa.fa_bwd_workspace_bytes(0, 4, 300) == 0


def dec(L, q=FAKE, k=FAKE, v=FAKE, ks=FAKE, vs=FAKE, o=FAKE, lse=None, B=2, Hq=8, Hkv=2, Skv=100,
        D=128, scale=0.1, splits=4, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = L.fa_decode_int8_workspace_bytes(B, Hq, D, splits)
    return L.fa_decode_int8(q, k, v, ks, vs, o, lse, B, Hq, Hkv, Skv, D, scale, splits, ws,
                            ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(vs=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(splits=0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(Skv=0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(Hq=6, Hkv=4), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(scale=-1.0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(D=80), fa.STATUS["FA_ERR_UNSUPPORTED"]),
    (dict(ks=FAKE + 4), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(ws=None), fa.STATUS["FA_ERR_WORKSPACE"]),
    (dict(ws_bytes=16), fa.STATUS["FA_ERR_WORKSPACE"]),
])
def test_decode_rejects(L, kw, code):
    assert dec(L, **kw) == code


def paged(L, q=FAKE, k=FAKE, v=FAKE, ks=FAKE, vs=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=None, B=2,
          Hq=8, Hkv=2, P=64, max_pages=8, num_pages=16, D=128, scale=0.1, splits=4, ws=FAKE,
          ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = L.fa_decode_int8_workspace_bytes(B, Hq, D, splits)
    return L.fa_decode_int8_paged(q, k, v, ks, vs, bt, sl, o, lse, B, Hq, Hkv, P, max_pages,
                                  num_pages, D, scale, splits, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(bt=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(sl=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(P=48), fa.STATUS["FA_ERR_INVALID_ARG"]),        # not a power of two
    (dict(P=8), fa.STATUS["FA_ERR_INVALID_ARG"]),         # below 16
    (dict(P=1 << 17), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(max_pages=0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(num_pages=0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(max_pages=1 << 25, P=64), fa.STATUS["FA_ERR_INVALID_ARG"]),  # > 2^30 keys
    (dict(Hq=6, Hkv=4), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(splits=0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(D=96), fa.STATUS["FA_ERR_UNSUPPORTED"]),
    (dict(k=FAKE + 8), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(bt=FAKE + 2), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(sl=FAKE + 1), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(ws=None), fa.STATUS["FA_ERR_WORKSPACE"]),
    (dict(ws_bytes=64), fa.STATUS["FA_ERR_WORKSPACE"]),
])
def test_paged_decode_rejects(L, kw, code):
    assert paged(L, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(Skv=0), fa.STATUS["FA_ERR_INVALID_ARG"]),
    (dict(D=96), fa.STATUS["FA_ERR_UNSUPPORTED"]),
    (dict(v=FAKE + 4), fa.STATUS["FA_ERR_ALIGNMENT"]),
    (dict(ws_bytes=16), fa.STATUS["FA_ERR_WORKSPACE"]),
])
def test_int4_decode_rejects(L, kw, code):
    args = dict(q=FAKE, k=FAKE, v=FAKE, ks=FAKE, vs=FAKE, o=FAKE, lse=None, B=2, Hq=8, Hkv=2,
                Skv=100, D=128, scale=0.1, splits=4, ws=FAKE, ws_bytes=None)
    args.update(kw)
    if args["ws_bytes"] is None:
        args["ws_bytes"] = L.fa_decode_int8_workspace_bytes(args["B"], args["Hq"], args["D"],
                                                            args["splits"])
    a = args
    assert L.fa_decode_int4(a["q"], a["k"], a["v"], a["ks"], a["vs"], a["o"], a["lse"], a["B"],
                            a["Hq"], a["Hkv"], a["Skv"], a["D"], a["scale"], a["splits"], a["ws"],
                            a["ws_bytes"], None) == code


def test_workspace_bytes(L):
    B, Hq, D, S = 16, 32, 128, 16
    o_bytes = S * B * Hq * D * 4
    lse_bytes = S * B * Hq * 4
    got = fa.fa_decode_int8_workspace_bytes(B, Hq, D, S)
    assert got >= o_bytes + lse_bytes and got % 256 == 0 and got - (o_bytes + lse_bytes) < 512
    assert fa.fa_decode_int8_workspace_bytes(0, Hq, D, S) == 0
    assert fa.fa_decode_int8_workspace_bytes(B, Hq, D, 0) == 0


def test_selftest_rejects_bad_timeout(L):
    assert L.fa_selftest_bounded_wait(0, None) == fa.STATUS["FA_ERR_INVALID_ARG"]
    assert L.fa_selftest_bounded_wait(10 ** 8, None) == fa.STATUS["FA_ERR_INVALID_ARG"]
