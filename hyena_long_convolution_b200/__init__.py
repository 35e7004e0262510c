"""Gated Hyena cascade operator on NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in include/hyena.h: every function below
only checks and marshals torch tensors (device memory and streams) into raw
pointers and sizes and calls the CUDA library; all arithmetic happens in the
library's kernels.  There is no CPU path.

    y = x3 * (h_c * (x1 * x2)) + Dskip * (x1 * x2)

with h_c either an explicit short FIR (hcs 7 taps / hcm 128 taps,
``short_conv``) or the long modal filter h_c[t] = sum_n R[c,n] exp(a[c,n] t)
(hcl, ``modal_long_conv``).  Layout [B, L, D] bf16, channel-contiguous; a row
stride ld >= D is allowed, so x1, x2, x3 may be views of one [B, L, 3D]
projection output.  The ``*_packed`` variants read the three inputs from one
[B, L, >= 3D] projection buffer whose rows hold channel groups of ``group``
channels as [x1 | x2 | x3] (group = 1: per-channel triples x1_c x2_c x3_c).
The ``*_complex`` variants take complex modes (poles and residues as [D, N, 2]
fp32 pairs; h_c[t] = Re sum_n R p^t), and the ``*_decode`` functions advance
the modal state or the FIR window by one generated token.
"""
from __future__ import annotations

import ctypes

from ._lib import HyenaError, check, lib  # noqa: F401

__all__ = [
    "HyenaError",
    "ModalWorkspace",
    "last_launch_count",
    "modal_decode",
    "modal_decode_complex",
    "modal_decode_complex_packed",
    "modal_decode_packed",
    "modal_long_conv",
    "modal_long_conv_complex",
    "modal_long_conv_complex_packed",
    "HostWorkspace",
    "modal_long_conv_host",
    "modal_prepare",
    "modal_long_conv_prepared",
    "short_conv_host",
    "modal_long_conv_packed",
    "modal_state_init",
    "short_conv",
    "short_conv_packed",
    "short_conv_dft",
    "short_decode",
    "short_decode_packed",
    "workspace_check",
    "workspace_size",
]

MAX_MODES = 64
MAX_COMPLEX_MODES = 32
MAX_TAPS = 128


def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        # the current stream of the current device; torch's raw query skips
        # building a Stream object (3.5 us of a ~19 us decode call)
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        if raw is not None:
            return raw(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t):
    # a plain integer: ctypes converts it through the entry point's c_void_p
    # argument type (None is NULL)
    return None if t is None else t.data_ptr()


def _bld(x, name):
    """[B, L, D] bf16 view with unit channel stride -> (B, L, D, ld)."""
    torch = _torch()
    if x.dtype != torch.bfloat16 or x.dim() != 3 or not x.is_cuda:
        raise ValueError(f"{name} must be a 3-D bf16 CUDA tensor [B, L, D]")
    B, L, D = x.shape
    if x.stride(2) != 1:
        raise ValueError(f"{name} must be channel-contiguous")
    ld = x.stride(1) if L > 1 else (x.stride(0) // max(L, 1) if B > 1 else D)
    if B > 1 and L > 0 and x.stride(0) != L * ld:
        raise ValueError(f"{name}: batch stride must equal L * row stride")
    return B, L, D, ld


def _same_ld(*xs):
    lds = {x[3] for x in xs}
    if len(lds) != 1:
        raise ValueError("x1, x2, x3 must share one row stride")


def _f32(t, shape, name, allow_none=True):
    torch = _torch()
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if t.dtype != torch.float32 or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous fp32 tensor of shape {tuple(shape)}")
    return t


def last_launch_count() -> int:
    """Kernels/memsets enqueued by the most recent call on this thread."""
    return int(lib().hyena_last_launch_count())


def workspace_size(B: int, D: int, N: int) -> int:
    return int(lib().hyena_modal_long_conv_workspace_size(B, D, N))


class ModalWorkspace:
    """Device workspace for modal_long_conv, zero-filled once at creation."""

    def __init__(self, B: int, D: int, N: int, device=None, stream=None):
        torch = _torch()
        n = workspace_size(B, D, N)
        if n == 0:
            raise ValueError("invalid workspace shape")
        self.nbytes = n
        self.buf = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
        check("hyena_modal_workspace_init",
              lib().hyena_modal_workspace_init(_ptr(self.buf), n, _stream(stream)))

    def fits(self, B: int, D: int, N: int) -> bool:
        return workspace_size(B, D, N) <= self.nbytes


def workspace_check(ws: ModalWorkspace, stream=None) -> None:
    """Synchronise and raise if a bounded device wait of an earlier call ran out."""
    check("hyena_workspace_check", lib().hyena_workspace_check(_ptr(ws.buf), _stream(stream)))


def modal_state_init(state, stream=None):
    """Zero a [B, D, N] fp32 modal state (start of chunked prefill)."""
    B, D, N = state.shape
    _f32(state, (B, D, N), "state", allow_none=False)
    check("hyena_modal_state_init", lib().hyena_modal_state_init(_ptr(state), B, D, N, _stream(stream)))
    return state


def modal_long_conv(x1, x2, x3, log_poles, residues, Dskip=None, y=None, state_in=None,
                    state_out=None, workspace: ModalWorkspace | None = None, stream=None):
    """Long modal-form Hyena filter (hcl) with fused gates.

    x1, x2, x3: [B, L, D] bf16 (views sharing a row stride); log_poles,
    residues: [D, N] fp32; Dskip: [D] fp32 or None; state_in/state_out:
    [B, D, N] fp32 or None (may be the same tensor).  Returns y ([B, L, D]
    bf16, allocated if not given).
    """
    torch = _torch()
    s1, s2, s3 = _bld(x1, "x1"), _bld(x2, "x2"), _bld(x3, "x3")
    _same_ld(s1, s2, s3)
    B, L, D, ld = s1
    if s2[:3] != (B, L, D) or s3[:3] != (B, L, D):
        raise ValueError("x1, x2, x3 shapes differ")
    Dn, N = log_poles.shape
    if Dn != D:
        raise ValueError("log_poles must be [D, N]")
    _f32(log_poles, (D, N), "log_poles", False)
    _f32(residues, (D, N), "residues", False)
    _f32(Dskip, (D,), "Dskip")
    _f32(state_in, (B, D, N), "state_in")
    _f32(state_out, (B, D, N), "state_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16, device=x1.device)
    yB, yL, yD, ld_y = _bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y shape differs from x")
    if workspace is None:
        workspace = ModalWorkspace(B, D, N, device=x1.device, stream=stream)
    rc = lib().hyena_modal_long_conv(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(log_poles), _ptr(residues),
                                     _ptr(Dskip), _ptr(y), ld_y, _ptr(state_in), _ptr(state_out),
                                     B, L, D, N, _ptr(workspace.buf), workspace.nbytes, _stream(stream))
    check("hyena_modal_long_conv", rc)
    return y


def modal_prepare(log_poles, residues, Dskip, workspace: ModalWorkspace, B: int = 1, stream=None):
    """Form the coefficient table of a real-mode filter in ``workspace`` once,
    for the chunks of one sequence that follow (modal_long_conv_prepared)."""
    D, N = log_poles.shape
    _f32(log_poles, (D, N), "log_poles", False)
    _f32(residues, (D, N), "residues", False)
    _f32(Dskip, (D,), "Dskip")
    rc = lib().hyena_modal_prepare(_ptr(log_poles), _ptr(residues), _ptr(Dskip), B, D, N, _ptr(workspace.buf),
                                   workspace.nbytes, _stream(stream))
    check("hyena_modal_prepare", rc)


def modal_long_conv_prepared(x1, x2, x3, N: int, workspace: ModalWorkspace, y=None, state_in=None, state_out=None,
                             stream=None):
    """modal_long_conv with the table of the last modal_prepare on ``workspace``
    (the same bits as modal_long_conv with those parameters)."""
    torch = _torch()
    s1, s2, s3 = _bld(x1, "x1"), _bld(x2, "x2"), _bld(x3, "x3")
    _same_ld(s1, s2, s3)
    B, L, D, ld = s1
    if s2[:3] != (B, L, D) or s3[:3] != (B, L, D):
        raise ValueError("x1, x2, x3 shapes differ")
    _f32(state_in, (B, D, N), "state_in")
    _f32(state_out, (B, D, N), "state_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16, device=x1.device)
    yB, yL, yD, ld_y = _bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y shape differs from x")
    rc = lib().hyena_modal_long_conv_prepared(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(y), ld_y, _ptr(state_in),
                                              _ptr(state_out), B, L, D, N, _ptr(workspace.buf), workspace.nbytes,
                                              _stream(stream))
    check("hyena_modal_long_conv_prepared", rc)
    return y


def _host_bld(x, name):
    """[B, L, D] bf16 (or int16 bits) host tensor with unit channel stride ->
    (B, L, D, ld)."""
    torch = _torch()
    if x.dtype not in (torch.bfloat16, torch.int16) or x.dim() != 3 or x.is_cuda:
        raise ValueError(f"{name} must be a 3-D bf16 host tensor [B, L, D]")
    B, L, D = x.shape
    if x.stride(2) != 1:
        raise ValueError(f"{name} must be channel-contiguous")
    ld = x.stride(1) if L > 1 else (x.stride(0) // max(L, 1) if B > 1 else D)
    if B > 1 and L > 0 and x.stride(0) != L * ld:
        raise ValueError(f"{name}: batch stride must equal L * row stride")
    return B, L, D, ld


class HostWorkspace:
    """Device workspace of modal_long_conv_host (the scan's workspace, two
    staging slots of `chunk` tokens and the carried state), zero-filled once."""

    def __init__(self, B: int, D: int, N: int, chunk: int = 2048, device=None, stream=None):
        torch = _torch()
        n = int(lib().hyena_modal_host_workspace_size(B, D, N, chunk))
        if n == 0:
            raise ValueError("invalid host-workspace shape (chunk must be a positive multiple of 128)")
        self.nbytes, self.chunk = n, chunk
        self.buf = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
        check("hyena_modal_workspace_init",
              lib().hyena_modal_workspace_init(_ptr(self.buf), n, _stream(stream)))


def modal_long_conv_host(x1, x2, x3, log_poles, residues, Dskip=None, y=None, state_in=None,
                         state_out=None, workspace: HostWorkspace | None = None, stream=None):
    """modal_long_conv with x1, x2, x3 and y in host memory ([B, L, D] bf16
    host tensors, pinned for overlapped copies): the sequence is streamed
    through the device in chunks of ``workspace.chunk`` tokens with the copies
    in both directions overlapping the scan.  Parameters and state are device
    tensors.  Returns y (a host tensor, allocated pinned if not given); it is
    valid once ``stream`` has been synchronised."""
    torch = _torch()
    s1, s2, s3 = _host_bld(x1, "x1"), _host_bld(x2, "x2"), _host_bld(x3, "x3")
    _same_ld(s1, s2, s3)
    B, L, D, ld = s1
    if s2[:3] != (B, L, D) or s3[:3] != (B, L, D):
        raise ValueError("x1, x2, x3 shapes differ")
    Dn, N = log_poles.shape
    if Dn != D:
        raise ValueError("log_poles must be [D, N]")
    _f32(log_poles, (D, N), "log_poles", False)
    _f32(residues, (D, N), "residues", False)
    _f32(Dskip, (D,), "Dskip")
    _f32(state_in, (B, D, N), "state_in")
    _f32(state_out, (B, D, N), "state_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16).pin_memory()
    yB, yL, yD, ld_y = _host_bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y shape differs from x")
    if workspace is None:
        workspace = HostWorkspace(B, D, N, device=log_poles.device, stream=stream)
    rc = lib().hyena_modal_long_conv_host(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(log_poles), _ptr(residues),
                                          _ptr(Dskip), _ptr(y), ld_y, _ptr(state_in), _ptr(state_out),
                                          B, L, D, N, workspace.chunk, _ptr(workspace.buf), workspace.nbytes,
                                          _stream(stream))
    check("hyena_modal_long_conv_host", rc)
    return y


def short_conv_host(x1, x2, x3, taps, Dskip=None, y=None, hist_in=None, hist_out=None, chunk=2048,
                    workspace=None, stream=None):
    """short_conv with x1, x2, x3 and y in host memory ([B, L, D] bf16 host
    tensors, pinned for overlapped copies), streamed through the device in
    chunks with the FIR window carried.  taps [D, K] bf16, Dskip, hist_in and
    hist_out ([B, K-1, D] fp32) are device tensors; ``workspace`` is a device
    uint8 tensor of at least short_host_workspace_size bytes (allocated if
    not given).  Returns y, valid once ``stream`` has been synchronised."""
    torch = _torch()
    s1, s2, s3 = _host_bld(x1, "x1"), _host_bld(x2, "x2"), _host_bld(x3, "x3")
    _same_ld(s1, s2, s3)
    B, L, D, ld = s1
    if s2[:3] != (B, L, D) or s3[:3] != (B, L, D):
        raise ValueError("x1, x2, x3 shapes differ")
    if taps.dtype != torch.bfloat16 or taps.dim() != 2 or taps.shape[0] != D or not taps.is_contiguous():
        raise ValueError("taps must be a contiguous [D, K] bf16 tensor")
    K = taps.shape[1]
    _f32(Dskip, (D,), "Dskip")
    _f32(hist_in, (B, K - 1, D), "hist_in")
    _f32(hist_out, (B, K - 1, D), "hist_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16).pin_memory()
    yB, yL, yD, ld_y = _host_bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y shape differs from x")
    need = int(lib().hyena_short_host_workspace_size(B, D, K, chunk))
    if need == 0:
        raise ValueError("invalid host-workspace shape")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=taps.device)
    rc = lib().hyena_short_conv_host(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(taps), _ptr(Dskip), _ptr(y), ld_y,
                                     _ptr(hist_in), _ptr(hist_out), B, L, D, K, chunk, _ptr(workspace),
                                     workspace.numel(), _stream(stream))
    check("hyena_short_conv_host", rc)
    return y


def _bd(x, name):
    """One token per batch row: [B, D] or [B, 1, D] bf16 with unit channel
    stride -> (B, D, ld), element (b, c) at b * ld + c."""
    torch = _torch()
    sh = x.shape  # one query each of shape and strides: this runs once per tensor per token
    if x.dtype is not torch.bfloat16 or not x.is_cuda or len(sh) not in (2, 3) or (len(sh) == 3 and sh[1] != 1):
        raise ValueError(f"{name} must be a bf16 CUDA tensor [B, D] or [B, 1, D]")
    st = x.stride()
    if st[-1] != 1:
        raise ValueError(f"{name} must have unit channel stride")
    return sh[0], sh[-1], st[0]


def modal_decode(x1, x2, x3, log_poles, residues, Dskip, state, y=None, stream=None):
    """One generated token through the long modal filter: advances ``state``
    ([B, D, N] fp32, in place) and returns y ([B, D] or [B, 1, D] like x1).
    Equals ``modal_long_conv`` on a one-token sequence with state_in =
    state_out = state, bit for bit."""
    torch = _torch()
    (B, D, ld), b2, b3 = _bd(x1, "x1"), _bd(x2, "x2"), _bd(x3, "x3")
    if b2 != (B, D, ld) or b3 != (B, D, ld):
        raise ValueError("x1, x2, x3 must share shape and row stride")
    Dn, N = log_poles.shape
    if Dn != D:
        raise ValueError("log_poles must be [D, N]")
    _f32(log_poles, (D, N), "log_poles", False)
    _f32(residues, (D, N), "residues", False)
    _f32(Dskip, (D,), "Dskip")
    _f32(state, (B, D, N), "state", False)
    if y is None:
        y = torch.empty_like(x1, memory_format=torch.contiguous_format)
    yB, yD, ld_y = _bd(y, "y")
    if (yB, yD) != (B, D):
        raise ValueError("y shape differs from x")
    rc = lib().hyena_modal_decode(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(log_poles), _ptr(residues), _ptr(Dskip),
                                  _ptr(y), ld_y, _ptr(state), B, D, N, _stream(stream))
    check("hyena_modal_decode", rc)
    return y


def short_decode(x1, x2, x3, taps, Dskip, hist, y=None, stream=None):
    """One generated token through an explicit FIR: advances the window
    ``hist`` ([B, K-1, D] fp32, in place; None when K = 1) and returns y.
    Equals ``short_conv`` on a one-token sequence with hist_in = hist_out =
    hist, bit for bit."""
    torch = _torch()
    (B, D, ld), b2, b3 = _bd(x1, "x1"), _bd(x2, "x2"), _bd(x3, "x3")
    if b2 != (B, D, ld) or b3 != (B, D, ld):
        raise ValueError("x1, x2, x3 must share shape and row stride")
    if taps.dtype != torch.bfloat16 or taps.dim() != 2 or taps.shape[0] != D or not taps.is_contiguous():
        raise ValueError("taps must be a contiguous bf16 [D, K] tensor")
    K = taps.shape[1]
    _f32(Dskip, (D,), "Dskip")
    if K > 1:
        _f32(hist, (B, K - 1, D), "hist", False)
    if y is None:
        y = torch.empty_like(x1, memory_format=torch.contiguous_format)
    yB, yD, ld_y = _bd(y, "y")
    if (yB, yD) != (B, D):
        raise ValueError("y shape differs from x")
    rc = lib().hyena_short_decode(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(taps), _ptr(Dskip), _ptr(y), ld_y,
                                  _ptr(hist) if K > 1 else None, B, D, K, _stream(stream))
    check("hyena_short_decode", rc)
    return y


def short_conv(x1, x2, x3, taps, Dskip=None, y=None, hist_in=None, hist_out=None, stream=None):
    """Explicit short Hyena FIR (hcs/hcm) with fused gates.

    taps: [D, K] bf16 in lag order (taps[c, k] multiplies v[t-k]);
    hist_in/hist_out: [B, K-1, D] fp32 or None (may be the same tensor).
    """
    return _short_conv("hyena_short_conv", x1, x2, x3, taps, Dskip, y, hist_in, hist_out, stream)


def short_conv_dft(x1, x2, x3, taps, Dskip=None, y=None, hist_in=None, hist_out=None, stream=None):
    """short_conv computed on the tensor cores as overlap-save DFT-as-GEMM
    (hyena_short_conv_dft): the same arguments; results agree with short_conv
    to tf32 rounding.  The first call on a device copies the DFT tables with a
    synchronous copy (make it before any CUDA graph capture).
    """
    return _short_conv("hyena_short_conv_dft", x1, x2, x3, taps, Dskip, y, hist_in, hist_out, stream)


def _short_conv(entry, x1, x2, x3, taps, Dskip, y, hist_in, hist_out, stream):
    torch = _torch()
    s1, s2, s3 = _bld(x1, "x1"), _bld(x2, "x2"), _bld(x3, "x3")
    _same_ld(s1, s2, s3)
    B, L, D, ld = s1
    if s2[:3] != (B, L, D) or s3[:3] != (B, L, D):
        raise ValueError("x1, x2, x3 shapes differ")
    if taps.dtype != torch.bfloat16 or taps.dim() != 2 or taps.shape[0] != D or not taps.is_contiguous():
        raise ValueError("taps must be a contiguous bf16 [D, K] tensor")
    K = taps.shape[1]
    _f32(Dskip, (D,), "Dskip")
    _f32(hist_in, (B, K - 1, D), "hist_in")
    _f32(hist_out, (B, K - 1, D), "hist_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16, device=x1.device)
    yB, yL, yD, ld_y = _bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y shape differs from x")
    rc = getattr(lib(), entry)(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(taps), _ptr(Dskip), _ptr(y), ld_y,
                               _ptr(hist_in), _ptr(hist_out), B, L, D, K, _stream(stream))
    check(entry, rc)
    return y


# ---------------------------------------------------------------- packed inputs

def _packed(xp, D, decode=False):
    """Projection buffer [B, L, W] (decode: [B, W] or [B, 1, W]) with W >= 3D
    and unit element stride -> (B, L, ld)."""
    if decode:
        B, W, ld = _bd(xp, "xp")
        L = 1
    else:
        B, L, W, ld = _bld(xp, "xp")
    if W < 3 * D:
        raise ValueError(f"xp rows hold {W} values, fewer than 3 D = {3 * D}")
    return B, L, ld


def modal_long_conv_packed(xp, group, log_poles, residues, Dskip=None, y=None, state_in=None,
                           state_out=None, workspace: ModalWorkspace | None = None, stream=None):
    """``modal_long_conv`` with x1, x2, x3 read from one projection buffer xp
    ([B, L, W >= 3D] bf16) in channel groups of ``group`` (x_k of channel c at
    column 3 group (c // group) + (k-1) group + c % group).  D is taken from
    log_poles ([D, N])."""
    torch = _torch()
    D, N = log_poles.shape
    B, L, ld = _packed(xp, D)
    _f32(log_poles, (D, N), "log_poles", False)
    _f32(residues, (D, N), "residues", False)
    _f32(Dskip, (D,), "Dskip")
    _f32(state_in, (B, D, N), "state_in")
    _f32(state_out, (B, D, N), "state_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16, device=xp.device)
    yB, yL, yD, ld_y = _bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y must be [B, L, D]")
    if workspace is None:
        workspace = ModalWorkspace(B, D, N, device=xp.device, stream=stream)
    rc = lib().hyena_modal_long_conv_packed(_ptr(xp), ld, int(group), _ptr(log_poles), _ptr(residues),
                                            _ptr(Dskip), _ptr(y), ld_y, _ptr(state_in), _ptr(state_out),
                                            B, L, D, N, _ptr(workspace.buf), workspace.nbytes, _stream(stream))
    check("hyena_modal_long_conv_packed", rc)
    return y


def short_conv_packed(xp, group, taps, Dskip=None, y=None, hist_in=None, hist_out=None, stream=None):
    """``short_conv`` with x1, x2, x3 read from one projection buffer xp in
    channel groups of ``group`` (see ``modal_long_conv_packed``).  D is taken
    from taps ([D, K])."""
    torch = _torch()
    if taps.dtype != torch.bfloat16 or taps.dim() != 2 or not taps.is_contiguous():
        raise ValueError("taps must be a contiguous bf16 [D, K] tensor")
    D, K = taps.shape
    B, L, ld = _packed(xp, D)
    _f32(Dskip, (D,), "Dskip")
    _f32(hist_in, (B, K - 1, D), "hist_in")
    _f32(hist_out, (B, K - 1, D), "hist_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16, device=xp.device)
    yB, yL, yD, ld_y = _bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y must be [B, L, D]")
    rc = lib().hyena_short_conv_packed(_ptr(xp), ld, int(group), _ptr(taps), _ptr(Dskip), _ptr(y), ld_y,
                                       _ptr(hist_in), _ptr(hist_out), B, L, D, K, _stream(stream))
    check("hyena_short_conv_packed", rc)
    return y


def modal_decode_packed(xp, group, log_poles, residues, Dskip, state, y=None, stream=None):
    """``modal_decode`` with the token's x1, x2, x3 read from one projection
    row per batch row (xp [B, W] or [B, 1, W], W >= 3D) in channel groups of
    ``group``."""
    torch = _torch()
    D, N = log_poles.shape
    B, _, ld = _packed(xp, D, decode=True)
    _f32(log_poles, (D, N), "log_poles", False)
    _f32(residues, (D, N), "residues", False)
    _f32(Dskip, (D,), "Dskip")
    _f32(state, (B, D, N), "state", False)
    if y is None:
        y = torch.empty((B, D), dtype=torch.bfloat16, device=xp.device)
    yB, yD, ld_y = _bd(y, "y")
    if (yB, yD) != (B, D):
        raise ValueError("y must be [B, D] or [B, 1, D]")
    rc = lib().hyena_modal_decode_packed(_ptr(xp), ld, int(group), _ptr(log_poles), _ptr(residues), _ptr(Dskip),
                                         _ptr(y), ld_y, _ptr(state), B, D, N, _stream(stream))
    check("hyena_modal_decode_packed", rc)
    return y


def short_decode_packed(xp, group, taps, Dskip, hist, y=None, stream=None):
    """``short_decode`` with the token's x1, x2, x3 read from one projection
    row per batch row in channel groups of ``group``."""
    torch = _torch()
    if taps.dtype != torch.bfloat16 or taps.dim() != 2 or not taps.is_contiguous():
        raise ValueError("taps must be a contiguous bf16 [D, K] tensor")
    D, K = taps.shape
    B, _, ld = _packed(xp, D, decode=True)
    _f32(Dskip, (D,), "Dskip")
    if K > 1:
        _f32(hist, (B, K - 1, D), "hist", False)
    if y is None:
        y = torch.empty((B, D), dtype=torch.bfloat16, device=xp.device)
    yB, yD, ld_y = _bd(y, "y")
    if (yB, yD) != (B, D):
        raise ValueError("y must be [B, D] or [B, 1, D]")
    rc = lib().hyena_short_decode_packed(_ptr(xp), ld, int(group), _ptr(taps), _ptr(Dskip), _ptr(y), ld_y,
                                         _ptr(hist) if K > 1 else None, B, D, K, _stream(stream))
    check("hyena_short_decode_packed", rc)
    return y


# ---------------------------------------------------------------- complex modes

def _cpar(poles, residues):
    """poles, residues fp32 [D, N, 2] (real, imaginary) -> (D, N)."""
    if poles.dim() != 3 or poles.shape[2] != 2:
        raise ValueError("poles must be a [D, N, 2] fp32 tensor")
    D, N, _ = poles.shape
    _f32(poles, (D, N, 2), "poles", False)
    _f32(residues, (D, N, 2), "residues", False)
    return D, N


def modal_long_conv_complex(x1, x2, x3, poles, residues, Dskip=None, y=None, state_in=None,
                            state_out=None, workspace: ModalWorkspace | None = None, stream=None):
    """Long modal filter with complex modes, h[t] = Re sum_n R_n p_n^t, with
    fused gates.  poles, residues: [D, N, 2] fp32 (real, imaginary);
    state_in/state_out: [B, D, N, 2] fp32 or None.  The workspace is that of
    2N real modes."""
    torch = _torch()
    s1, s2, s3 = _bld(x1, "x1"), _bld(x2, "x2"), _bld(x3, "x3")
    _same_ld(s1, s2, s3)
    B, L, D, ld = s1
    if s2[:3] != (B, L, D) or s3[:3] != (B, L, D):
        raise ValueError("x1, x2, x3 shapes differ")
    Dp, N = _cpar(poles, residues)
    if Dp != D:
        raise ValueError("poles must be [D, N, 2]")
    _f32(Dskip, (D,), "Dskip")
    _f32(state_in, (B, D, N, 2), "state_in")
    _f32(state_out, (B, D, N, 2), "state_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16, device=x1.device)
    yB, yL, yD, ld_y = _bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y shape differs from x")
    if workspace is None:
        workspace = ModalWorkspace(B, D, 2 * N, device=x1.device, stream=stream)
    rc = lib().hyena_modal_long_conv_complex(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(poles), _ptr(residues),
                                             _ptr(Dskip), _ptr(y), ld_y, _ptr(state_in), _ptr(state_out),
                                             B, L, D, N, _ptr(workspace.buf), workspace.nbytes, _stream(stream))
    check("hyena_modal_long_conv_complex", rc)
    return y


def modal_decode_complex(x1, x2, x3, poles, residues, Dskip, state, y=None, stream=None):
    """One generated token through the complex-mode filter: advances
    ``state`` ([B, D, N, 2] fp32, in place); equals ``modal_long_conv_complex``
    on a one-token sequence bit for bit."""
    torch = _torch()
    (B, D, ld), b2, b3 = _bd(x1, "x1"), _bd(x2, "x2"), _bd(x3, "x3")
    if b2 != (B, D, ld) or b3 != (B, D, ld):
        raise ValueError("x1, x2, x3 must share shape and row stride")
    Dp, N = _cpar(poles, residues)
    if Dp != D:
        raise ValueError("poles must be [D, N, 2]")
    _f32(Dskip, (D,), "Dskip")
    _f32(state, (B, D, N, 2), "state", False)
    if y is None:
        y = torch.empty_like(x1, memory_format=torch.contiguous_format)
    yB, yD, ld_y = _bd(y, "y")
    if (yB, yD) != (B, D):
        raise ValueError("y shape differs from x")
    rc = lib().hyena_modal_decode_complex(_ptr(x1), _ptr(x2), _ptr(x3), ld, _ptr(poles), _ptr(residues),
                                          _ptr(Dskip), _ptr(y), ld_y, _ptr(state), B, D, N, _stream(stream))
    check("hyena_modal_decode_complex", rc)
    return y


def modal_long_conv_complex_packed(xp, group, poles, residues, Dskip=None, y=None, state_in=None,
                                   state_out=None, workspace: ModalWorkspace | None = None, stream=None):
    """``modal_long_conv_complex`` with x1, x2, x3 read from one projection
    buffer xp in channel groups of ``group`` (see ``modal_long_conv_packed``)."""
    torch = _torch()
    D, N = _cpar(poles, residues)
    B, L, ld = _packed(xp, D)
    _f32(Dskip, (D,), "Dskip")
    _f32(state_in, (B, D, N, 2), "state_in")
    _f32(state_out, (B, D, N, 2), "state_out")
    if y is None:
        y = torch.empty((B, L, D), dtype=torch.bfloat16, device=xp.device)
    yB, yL, yD, ld_y = _bld(y, "y")
    if (yB, yL, yD) != (B, L, D):
        raise ValueError("y must be [B, L, D]")
    if workspace is None:
        workspace = ModalWorkspace(B, D, 2 * N, device=xp.device, stream=stream)
    rc = lib().hyena_modal_long_conv_complex_packed(_ptr(xp), ld, int(group), _ptr(poles), _ptr(residues),
                                                    _ptr(Dskip), _ptr(y), ld_y, _ptr(state_in), _ptr(state_out),
                                                    B, L, D, N, _ptr(workspace.buf), workspace.nbytes,
                                                    _stream(stream))
    check("hyena_modal_long_conv_complex_packed", rc)
    return y


def modal_decode_complex_packed(xp, group, poles, residues, Dskip, state, y=None, stream=None):
    """``modal_decode_complex`` with the token's x1, x2, x3 read from one
    projection row per batch row in channel groups of ``group``."""
    torch = _torch()
    D, N = _cpar(poles, residues)
    B, _, ld = _packed(xp, D, decode=True)
    _f32(Dskip, (D,), "Dskip")
    _f32(state, (B, D, N, 2), "state", False)
    if y is None:
        y = torch.empty((B, D), dtype=torch.bfloat16, device=xp.device)
    yB, yD, ld_y = _bd(y, "y")
    if (yB, yD) != (B, D):
        raise ValueError("y must be [B, D] or [B, 1, D]")
    rc = lib().hyena_modal_decode_complex_packed(_ptr(xp), ld, int(group), _ptr(poles), _ptr(residues),
                                                 _ptr(Dskip), _ptr(y), ld_y, _ptr(state), B, D, N, _stream(stream))
    check("hyena_modal_decode_complex_packed", rc)
    return y
