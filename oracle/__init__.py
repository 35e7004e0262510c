"""fp64 CPU oracle for the gated Hyena cascade operator -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The CUDA library and its Python binding never
import it, and it imports nothing from them.

The arithmetic lives in ``hyena_oracle.c`` (plain loops, double precision,
OpenMP over (batch, channel)); this module builds that file with gcc, wraps it
with ctypes and adds the chunked drivers, which simply call the single-pass
functions chunk after chunk while passing the fp64 state or FIR history along.
``brute.py`` is a separate pure-Python restatement for tiny inputs.

Parity pins: every function here is pinned by tests in tests/test_oracle_*.py
against closed forms, scipy's textbook IIR/FIR routine, hand-derived golden
fixtures and brute force (none of these re-type the oracle's own loops).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hyena_oracle.c")
_SO = os.path.join(_HERE, "libhyena_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile hyena_oracle.c into a shared library next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_SO)
            P = ctypes.c_void_p
            I = ctypes.c_int
            I64 = ctypes.c_int64
            lib.hyena_oracle_modal_recurrence.argtypes = [I, I, I, I, P, P, P, I64, P, P, P, P, P, P]
            lib.hyena_oracle_modal_direct.argtypes = [I, I, I, I, P, P, P, I64, P, P, P, P, P, P, P, I]
            lib.hyena_oracle_fir.argtypes = [I, I, I, I, P, P, P, I64, P, P, P, P, P]
            lib.hyena_oracle_cmodal_recurrence.argtypes = [I, I, I, I, P, P, P, I64, P, P, P, P, P, P]
            lib.hyena_oracle_cmodal_direct.argtypes = [I, I, I, I, P, P, P, I64, P, P, P, P, P, P, P, I]
            for f in (lib.hyena_oracle_modal_recurrence, lib.hyena_oracle_modal_direct,
                      lib.hyena_oracle_fir, lib.hyena_oracle_cmodal_recurrence,
                      lib.hyena_oracle_cmodal_direct):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _xs(x1, x2, x3):
    x1 = np.asarray(x1)
    B, L, ld = x1.shape
    out = []
    for x in (x1, x2, x3):
        x = np.ascontiguousarray(x, dtype=np.uint16)
        if x.shape != (B, L, ld):
            raise ValueError("x1, x2, x3 must share one [B, L, ld] shape")
        out.append(x)
    return out, B, L, ld


def _f32(a, shape=None):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.float32)
    if shape is not None and a.shape != shape:
        raise ValueError(f"expected shape {shape}, got {a.shape}")
    return a


def _f64(a, shape=None):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.float64)
    if shape is not None and a.shape != shape:
        raise ValueError(f"expected shape {shape}, got {a.shape}")
    return a


def set_threads(n: int) -> None:
    """Set the OpenMP thread count the oracle uses (process-wide)."""
    os.environ["OMP_NUM_THREADS"] = str(int(n))


def modal_recurrence(x1, x2, x3, log_poles, residues, Dskip=None, state_in=None, D=None):
    """Modal long conv by per-mode first-order recurrences (fp64).

    x1, x2, x3: uint16 bf16 bits [B, L, ld] (ld >= D; columns >= D ignored).
    log_poles, residues: fp32 [D, N].  Dskip: fp32 [D] or None (zero skip).
    state_in: float [B, D, N] or None (zero state).
    Returns (y fp64 [B, L, D], state_out fp64 [B, D, N]).
    """
    (x1, x2, x3), B, L, ld = _xs(x1, x2, x3)
    a = _f32(log_poles)
    Dc, N = a.shape
    D = Dc if D is None else D
    R = _f32(residues, (Dc, N))
    Ds = _f32(Dskip, (Dc,))
    Sin = _f64(state_in, (B, Dc, N))
    y = np.empty((B, L, D), dtype=np.float64)
    Sout = np.empty((B, D, N), dtype=np.float64)
    rc = _load().hyena_oracle_modal_recurrence(B, L, D, N, _ptr(x1), _ptr(x2), _ptr(x3), ld,
                                               _ptr(a), _ptr(R), _ptr(Ds), _ptr(Sin),
                                               _ptr(y), _ptr(Sout))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, Sout


def modal_direct(x1, x2, x3, log_poles, residues, Dskip=None, state_in=None):
    """Modal long conv as a direct O(L^2) convolution with h[k] = sum R e^{a k}."""
    (x1, x2, x3), B, L, ld = _xs(x1, x2, x3)
    a = _f32(log_poles)
    D, N = a.shape
    R = _f32(residues, (D, N))
    Ds = _f32(Dskip, (D,))
    Sin = _f64(state_in, (B, D, N))
    y = np.empty((B, L, D), dtype=np.float64)
    Sout = np.empty((B, D, N), dtype=np.float64)
    slots = max(1, min(os.cpu_count() or 1, B * D))
    scratch = np.empty(max(1, 2 * L * slots), dtype=np.float64)
    rc = _load().hyena_oracle_modal_direct(B, L, D, N, _ptr(x1), _ptr(x2), _ptr(x3), ld,
                                           _ptr(a), _ptr(R), _ptr(Ds), _ptr(Sin),
                                           _ptr(y), _ptr(Sout), _ptr(scratch), slots)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, Sout


def cmodal_recurrence(x1, x2, x3, poles, residues, Dskip=None, state_in=None):
    """Complex-mode long conv by per-mode complex recurrences (fp64).

    poles, residues: fp32 [D, N, 2] (real, imaginary); the filter is
    h[k] = Re sum_n R_n p_n^k.  state_in: float [B, D, N, 2] or None.
    Returns (y fp64 [B, L, D], state_out fp64 [B, D, N, 2]).
    """
    (x1, x2, x3), B, L, ld = _xs(x1, x2, x3)
    p = _f32(poles)
    D, N, two = p.shape
    if two != 2:
        raise ValueError("poles must be [D, N, 2]")
    R = _f32(residues, (D, N, 2))
    Ds = _f32(Dskip, (D,))
    Sin = _f64(state_in, (B, D, N, 2))
    y = np.empty((B, L, D), dtype=np.float64)
    Sout = np.empty((B, D, N, 2), dtype=np.float64)
    rc = _load().hyena_oracle_cmodal_recurrence(B, L, D, N, _ptr(x1), _ptr(x2), _ptr(x3), ld,
                                                _ptr(p), _ptr(R), _ptr(Ds), _ptr(Sin),
                                                _ptr(y), _ptr(Sout))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, Sout


def cmodal_direct(x1, x2, x3, poles, residues, Dskip=None, state_in=None):
    """Complex-mode long conv as a direct O(L^2) convolution with the filter
    taken from the polar form of each mode (independent of the recurrence)."""
    (x1, x2, x3), B, L, ld = _xs(x1, x2, x3)
    p = _f32(poles)
    D, N, _ = p.shape
    R = _f32(residues, (D, N, 2))
    Ds = _f32(Dskip, (D,))
    Sin = _f64(state_in, (B, D, N, 2))
    y = np.empty((B, L, D), dtype=np.float64)
    Sout = np.empty((B, D, N, 2), dtype=np.float64)
    slots = max(1, min(os.cpu_count() or 1, B * D))
    scratch = np.empty(max(1, 2 * L * slots), dtype=np.float64)
    rc = _load().hyena_oracle_cmodal_direct(B, L, D, N, _ptr(x1), _ptr(x2), _ptr(x3), ld,
                                            _ptr(p), _ptr(R), _ptr(Ds), _ptr(Sin),
                                            _ptr(y), _ptr(Sout), _ptr(scratch), slots)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, Sout


def fir(x1, x2, x3, taps, Dskip=None, hist_in=None):
    """Explicit causal FIR (hcs/hcm) in fp64.

    taps: uint16 bf16 bits [D, K], lag order.  hist_in: float [B, K-1, D] or None.
    Returns (y fp64 [B, L, D], hist_out fp64 [B, K-1, D]).
    """
    (x1, x2, x3), B, L, ld = _xs(x1, x2, x3)
    taps = np.ascontiguousarray(taps, dtype=np.uint16)
    D, K = taps.shape
    Ds = _f32(Dskip, (D,))
    Hin = _f64(hist_in, (B, K - 1, D)) if K > 1 else None
    y = np.empty((B, L, D), dtype=np.float64)
    Hout = np.empty((B, max(K - 1, 0), D), dtype=np.float64)
    rc = _load().hyena_oracle_fir(B, L, D, K, _ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(taps),
                                  _ptr(Ds), _ptr(Hin), _ptr(y), _ptr(Hout) if K > 1 else None)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return y, Hout


def _splits(L, chunks):
    """chunks: an int chunk size or an explicit list of chunk lengths."""
    if isinstance(chunks, (int, np.integer)):
        c = int(chunks)
        return [min(c, L - s) for s in range(0, L, c)] or [0]
    lens = [int(c) for c in chunks]
    if sum(lens) != L:
        raise ValueError("chunk lengths must sum to L")
    return lens


def modal_chunked(x1, x2, x3, log_poles, residues, Dskip=None, state_in=None, chunks=1024):
    """Feed the sequence chunk by chunk, carrying the fp64 modal state."""
    L = np.asarray(x1).shape[1]
    ys = []
    S = state_in
    t0 = 0
    for n in _splits(L, chunks):
        y, S = modal_recurrence(x1[:, t0:t0 + n], x2[:, t0:t0 + n], x3[:, t0:t0 + n],
                                log_poles, residues, Dskip, S)
        ys.append(y)
        t0 += n
    return np.concatenate(ys, axis=1), S


def fir_chunked(x1, x2, x3, taps, Dskip=None, hist_in=None, chunks=1024):
    """Feed the sequence chunk by chunk, carrying the fp64 FIR history."""
    L = np.asarray(x1).shape[1]
    ys = []
    H = hist_in
    t0 = 0
    for n in _splits(L, chunks):
        y, H = fir(x1[:, t0:t0 + n], x2[:, t0:t0 + n], x3[:, t0:t0 + n], taps, Dskip, H)
        ys.append(y)
        t0 += n
    return np.concatenate(ys, axis=1), H


def cmodal_chunked(x1, x2, x3, poles, residues, Dskip=None, state_in=None, chunks=1024):
    """Complex modes fed chunk by chunk, carrying the fp64 complex state."""
    L = np.asarray(x1).shape[1]
    ys = []
    S = state_in
    t0 = 0
    for n in _splits(L, chunks):
        y, S = cmodal_recurrence(x1[:, t0:t0 + n], x2[:, t0:t0 + n], x3[:, t0:t0 + n],
                                 poles, residues, Dskip, S)
        ys.append(y)
        t0 += n
    return np.concatenate(ys, axis=1), S
