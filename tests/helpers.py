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
        print(f"{what}: rel-L2 {rel:.3e}, max-abs/rms {mabs:.3e}, per-channel max-abs worst {worst:.3e}")
        return rel, worst
    print(f"{what}: rel-L2 {rel:.3e}, max-abs/rms {mabs:.3e}")
    return rel, mabs


class StreamedCompare:
    """The acceptance metrics of ``metrics`` / ``assert_close`` over a whole
    output tensor that is compared block of channels by block of channels
    (the oracle of a long workload does not fit in host memory at once).

    Feed it (y block, reference block, first channel) pairs covering every
    channel once; ``result()`` gives (rel-L2, max-abs beyond the bf16
    rounding / rms(ref)) over the whole tensor and, per channel, the worst
    max-abs against that channel's own rms and its rel-L2.
    """

    def __init__(self, D):
        self.D = D
        self.sq_err = 0.0
        self.sq_ref = 0.0
        self.count = 0
        self.max_excess = 0.0
        self.ch_excess = np.zeros(D)
        self.ch_sq_ref = np.zeros(D)
        self.ch_sq_err = np.zeros(D)
        self.ch_count = np.zeros(D)
        self.seen = np.zeros(D, dtype=bool)
        self.finite = True

    def add(self, y, ref, c0):
        y = np.asarray(y, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        assert y.shape == ref.shape, (y.shape, ref.shape)
        cb = y.shape[-1]
        assert not self.seen[c0:c0 + cb].any(), "channel compared twice"
        self.seen[c0:c0 + cb] = True
        self.finite &= bool(np.all(np.isfinite(y)))
        d = np.abs(y - ref).reshape(-1, cb)
        r = ref.reshape(-1, cb)
        excess = np.maximum(d - ROUNDING_ALLOWANCE * np.abs(r), 0.0)
        self.sq_err += float(np.sum(d * d))
        self.sq_ref += float(np.sum(r * r))
        self.count += r.size
        self.max_excess = max(self.max_excess, float(excess.max()) if excess.size else 0.0)
        self.ch_excess[c0:c0 + cb] = np.max(excess, axis=0)
        self.ch_sq_ref[c0:c0 + cb] = np.sum(r * r, axis=0)
        self.ch_sq_err[c0:c0 + cb] = np.sum(d * d, axis=0)
        self.ch_count[c0:c0 + cb] = r.shape[0]

    def result(self):
        assert self.seen.all(), "some channels were never compared"
        rel = float(np.sqrt(self.sq_err / max(self.sq_ref, 1e-300)))
        rms = float(np.sqrt(self.sq_ref / max(self.count, 1)))
        mabs = self.max_excess / max(rms, 1e-300)
        rms_c = np.sqrt(self.ch_sq_ref / np.maximum(self.ch_count, 1))
        ch_mabs = self.ch_excess / np.maximum(rms_c, 1e-300)
        ch_rel = np.sqrt(self.ch_sq_err / np.maximum(self.ch_sq_ref, 1e-300))
        return rel, mabs, ch_mabs, ch_rel

    def check(self, what, per_channel=False):
        assert self.finite, f"{what}: non-finite values"
        rel, mabs, ch_mabs, ch_rel = self.result()
        assert rel <= REL_L2_TOL, f"{what}: rel-L2 {rel:.3e} > {REL_L2_TOL}"
        assert mabs <= MAX_ABS_TOL, f"{what}: max-abs/rms {mabs:.3e} > {MAX_ABS_TOL}"
        if per_channel:
            worst = float(ch_mabs.max())
            assert worst <= MAX_ABS_TOL, f"{what}: per-channel max-abs {worst:.3e} > {MAX_ABS_TOL}"
        pct = np.percentile(ch_rel, [50, 99, 100])
        print(f"{what}: rel-L2 {rel:.3e}, max-abs/rms {mabs:.3e}, per-channel max-abs worst "
              f"{float(ch_mabs.max()):.3e}, per-channel rel-L2 p50/p99/max {pct[0]:.3e}/{pct[1]:.3e}/{pct[2]:.3e}")
        return rel, mabs
