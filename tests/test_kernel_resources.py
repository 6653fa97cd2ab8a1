"""Resource budgets of the sm_100a kernels, read from ptxas (compile only, no GPU): the register
counts that set how many CTAs share an SM and that the prefill's warpgroup register split
assumes, and spills in the hot kernels.  A source change that silently costs occupancy (the
8-bit decode kernel once grew to 137 registers, which leaves room for 2 CTAs per SM instead of 3)
fails here before it reaches a GPU."""
import os
import re
import subprocess
import tempfile

import pytest

from tiled_attention_26_b200 import build

REGFILE = 65536


@pytest.fixture(scope="module")
def kernels():
    with tempfile.TemporaryDirectory() as d:
        cmd = [build.nvcc()] + build.NVCC_FLAGS + ["-Xptxas", "-v", "-I",
                                                   os.path.join(build.ROOT, "include")] + \
            build.SOURCES + ["-o", os.path.join(d, "libfa_check.so")]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr[-2000:]
    out, cur = {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            cur = m.group(1)
            out[cur] = {"spill": 0}
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes spill stores", line)
        if m:
            out[cur]["spill"] = int(m.group(1))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            out[cur]["regs"] = int(m.group(1))
    return out


def _select(kernels, prefix):
    found = {k: v for k, v in kernels.items() if k.startswith(prefix)}
    assert found, prefix
    return found


def test_decode_8bit_kernels_fit_three_ctas_per_sm(kernels):
    # _ZN2fa22fa_decode_split_kernelILi<D>ELb<paged>ELi8EEE...: 160 threads, 3 CTAs per SM
    for name, v in _select(kernels, "_ZN2fa22fa_decode_split_kernelI").items():
        if "ELi8EE" in name:
            assert v["regs"] * 160 * 3 <= REGFILE, (name, v)
            assert v["spill"] <= 32, (name, v)


def test_decode_4bit_kernels_fit_three_ctas_per_sm(kernels):
    # the 4-bit kernels run the same 160-thread, 3-CTA-per-SM configuration
    for name, v in _select(kernels, "_ZN2fa22fa_decode_split_kernelI").items():
        if "ELi4EE" in name:
            assert v["regs"] * 160 * 3 <= REGFILE, (name, v)
            assert v["spill"] <= 32, (name, v)


def test_prefill_launch_registers_match_the_warpgroup_split(kernels):
    # 384 threads at 168 registers: softmax warpgroups 2 x 128 x 216 plus the producer / MMA
    # warpgroup 128 x 72 use exactly the launch's 384 x 168
    for name, v in _select(kernels, "_ZN2fa17fa_prefill_kernelI").items():
        assert v["regs"] == 168, (name, v)
    for name, v in _select(kernels, "_ZN2fa17fa_prefill_kernelI").items():
        if re.search(r"ILi(64|128)ELi0EE", name):  # the plain causal / window kernels
            assert v["spill"] == 0, (name, v)


def test_backward_kernels_fit_one_cta(kernels):
    found = _select(kernels, "_ZN2fa13fa_bwd_kernelI")
    assert len(found) == 2, sorted(kernels)  # D = 64 and D = 128
    for name, v in found.items():
        assert v["regs"] * 320 <= REGFILE, (name, v)
        assert v["spill"] <= 16, (name, v)  # (D = 64 keeps one 8-byte value in local memory)
