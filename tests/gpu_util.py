"""Helpers for the GPU parity tests: upload seeded numpy inputs and compare
device results with the oracle under the library's tolerance.

Tolerance (fp32-accumulated outputs): |gpu - ref| <= 2e-3 + 1e-3 |ref|.
For outputs stored as bf16 the bf16 store adds at most half a bf16 ulp of the
value, bounded here by 2^-8 |ref| (``bf16_out=True``). When both sides store
bf16 (the oracle rounds too, e.g. K/V cache rows), values a hair apart can
round to neighbouring bf16 numbers: one full ulp, 2^-7 |ref| (``ulps=1``).
Downstream of a bf16 rounding tie (a value within float32 error of a
rounding midpoint), an output may move by the tie's exact linear effect,
which the oracle computes (``lm_head_tie_bound``); it is passed as ``extra``.
"""
import numpy as np
import torch

ATOL = 2e-3
RTOL = 1e-3
BF16_HALF_ULP_REL = 2.0 ** -8


def dev(a, device="cuda"):
    """numpy -> torch on the device; uint16/uint32 travel as int16/int32."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    elif a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(a).to(device)


def bf16_dev(bits, device="cuda"):
    return dev(bits, device).view(torch.bfloat16)


def host64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_parity(gpu, ref, bf16_out=False, what="", ulps=0.5, extra=None):
    """``extra``: an added per-element bound, for outputs downstream of bf16
    roundings that sit on a tie (the oracle's ``lm_head_tie_bound``)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    tol = ATOL + RTOL * np.abs(ref)
    if extra is not None:
        tol = tol + np.asarray(extra, dtype=np.float64)
    if bf16_out:
        tol = tol + 2 * ulps * BF16_HALF_ULP_REL * np.abs(ref)
    err = np.abs(gpu - ref)
    bad = ~(err <= tol)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - tol, -np.inf)), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())}/{bad.size} outside tolerance; worst at {i}: "
            f"gpu={gpu[i]!r} ref={ref[i]!r} err={err[i]:.3e} tol={tol[i]:.3e}")
    return float(err.max()) if err.size else 0.0
