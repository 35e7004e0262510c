"""Shared test utilities: device upload of seeded inputs, comparison metrics.

Tolerances for bf16 I/O with fp32 accumulation, checked against the fp64
oracle over the whole compared tensor:
    rel-L2  = ||y - y_ref|| / ||y_ref||                          <= REL_L2_TOL
    max-abs = max (|y - y_ref| - 2^-8 |y_ref|)_+ / rms(y_ref)     <= MAX_ABS_TOL
The max-abs bound applies to the error in excess of the output's own bf16
rounding (at most half an ulp, i.e. 2^-8 |y|): rounding the exact result to
bf16 alone exceeds 2e-2 rms(y) wherever |y| > ~5 rms(y), which products of
Gaussian signals reach routinely.  For inputs with a wide per-channel dynamic
range the bound is also applied per channel (each channel against its own
rms).
"""
from __future__ import annotations

import numpy as np

REL_L2_TOL = 5e-3
MAX_ABS_TOL = 2e-2


def to_dev_bf16(bits: np.ndarray, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def to_dev_f32(a, device="cuda"):
    import torch
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def from_dev_bf16(t) -> np.ndarray:
    """bf16 device tensor -> fp64 numpy (exact)."""
    import torch
    u = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bits_of(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


ROUNDING_ALLOWANCE = 2.0 ** -8  # half a bf16 ulp, relative


def metrics(y: np.ndarray, ref: np.ndarray):
    """(rel-L2, max-abs error beyond bf16 rounding / rms(ref))."""
    d = np.abs(y - ref)
    nref = np.linalg.norm(ref.ravel())
    rel = float(np.linalg.norm(d.ravel()) / max(nref, 1e-300))
    rms = float(np.sqrt(np.mean(ref.astype(np.float64) ** 2))) if ref.size else 0.0
    excess = np.maximum(d - ROUNDING_ALLOWANCE * np.abs(ref), 0.0)
    mabs = float(np.max(excess)) / max(rms, 1e-300) if d.size else 0.0
    return rel, mabs


def assert_close(y, ref, what="y", per_channel=False):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite values"
    rel, mabs = metrics(y, ref)
    assert rel <= REL_L2_TOL, f"{what}: rel-L2 {rel:.3e} > {REL_L2_TOL}"
    assert mabs <= MAX_ABS_TOL, f"{what}: max-abs/rms {mabs:.3e} > {MAX_ABS_TOL}"
    if per_channel:
        d = np.abs(y - ref).reshape(-1, y.shape[-1])
        r = ref.reshape(-1, ref.shape[-1])
        excess = np.maximum(d - ROUNDING_ALLOWANCE * np.abs(r), 0.0)
        rms_c = np.sqrt(np.mean(r ** 2, axis=0))
        worst = float(np.max(np.max(excess, axis=0) / np.maximum(rms_c, 1e-300)))
        assert worst <= MAX_ABS_TOL, f"{what}: per-channel max-abs {worst:.3e} > {MAX_ABS_TOL}"
        return rel, worst
    return rel, mabs
