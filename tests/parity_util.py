"""Helpers shared by the GPU parity tests: moving seeded inputs between numpy and torch, and the
parity bar (O: max |err| <= 2e-2 and mean |err| <= 2e-3 against the fp64 oracle; LSE: |err| <=
1e-3, and -inf exactly where the oracle has -inf)."""
import numpy as np

O_MAX = 2e-2
O_MEAN = 2e-3
LSE_TOL = 1e-3


def to_dev_bf16(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def to_host_bits(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def o_to_f64(o) -> np.ndarray:
    import torch
    return o.to(torch.float32).cpu().numpy().astype(np.float64)


def check_o(o_gpu: np.ndarray, o_ref: np.ndarray, what=""):
    err = np.abs(o_gpu - o_ref)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    assert err.max() <= O_MAX, f"{what}: max |err| {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: mean |err| {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def check_lse(lse_gpu: np.ndarray, lse_ref: np.ndarray, what=""):
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), np.isneginf(lse_ref)), f"{what}: -inf pattern"
    assert np.all(np.isfinite(lse_gpu[fin])), f"{what}: non-finite LSE"
    if fin.any():
        d = np.abs(lse_gpu[fin] - lse_ref[fin]).max()
        assert d <= LSE_TOL, f"{what}: LSE |err| {d:.3e}"
        return float(d)
    return 0.0
