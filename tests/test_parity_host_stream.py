"""The host-buffer entry points (hyena_modal_long_conv_host,
hyena_short_conv_host).

Inputs and outputs live in page-locked host memory and are streamed through
the device in chunks (whole 128-token units for the modal filter, any length
for the FIR) with the state or window carried, so y and the final state must
equal the device-resident single pass bit for bit,
for ragged sequence lengths, several batch rows, padded host rows, a carried
input state or window and every chunk size; and stay within tolerance of the
fp64 oracle.
"""
import numpy as np
import pytest

import oracle
from synth import make_modal_inputs

from .helpers import assert_close, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


def _host_bf16(bits, ld=None):
    """Pinned bf16 host tensor [B, L, D] (row stride ld >= D) from bf16 bits."""
    import torch
    B, L, D = bits.shape
    ld = ld or D
    full = np.zeros((B, L, ld), np.uint16)
    full[..., :D] = bits
    t = torch.from_numpy(full.view(np.int16)).pin_memory()
    return t[..., :D]


def _run_both(B, L, D, N, chunk, seed, ld=None, with_state=True):
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_modal_inputs(B, L, D, N, seed)
    a, R, Ds = (to_dev_f32(inp[k]) for k in ("log_poles", "residues", "Dskip"))
    S0 = np.random.default_rng(seed).standard_normal((B, D, N)).astype(np.float32) if with_state else None
    S_in = torch.from_numpy(S0).cuda() if with_state else None
    # device-resident single pass
    xd = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    S_dev = torch.empty((B, D, N), device="cuda")
    y_dev = hy.modal_long_conv(*xd, a, R, Ds, state_in=S_in, state_out=S_dev)
    # host buffers, streamed in chunks
    xh = [_host_bf16(inp[k], ld) for k in ("x1", "x2", "x3")]
    yh = _host_bf16(np.zeros((B, L, D), np.uint16), ld)
    S_host = torch.empty((B, D, N), device="cuda")
    ws = hy.HostWorkspace(B, D, N, chunk=chunk)
    hy.modal_long_conv_host(*xh, a, R, Ds, y=yh, state_in=S_in, state_out=S_host, workspace=ws)
    torch.cuda.synchronize()
    return inp, S0, y_dev, S_dev, yh, S_host


@pytest.mark.parametrize("B,L,D,N,chunk,ld", [
    (1, 5000, 136, 12, 1024, None),   # ragged length and channels, short-path chunks
    (2, 3000, 64, 16, 128, 72),       # one unit per chunk, padded host rows
    (1, 9000, 256, 16, 4096, None),   # look-back chunks
    (1, 100, 64, 4, 2048, None),      # a single partial chunk
])
def test_host_stream_is_bitwise_the_device_single_pass(B, L, D, N, chunk, ld):
    import torch
    inp, S0, y_dev, S_dev, yh, S_host = _run_both(B, L, D, N, chunk, seed=L + D, ld=ld)
    y_host_bits = yh.contiguous().view(torch.int16)
    assert torch.equal(y_host_bits, y_dev.view(torch.int16).cpu())
    assert torch.equal(S_host, S_dev)


def test_host_stream_against_the_oracle():
    inp, S0, y_dev, S_dev, yh, S_host = _run_both(1, 4100, 128, 16, 1024, seed=7)
    import torch
    ref_y, ref_S = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"],
                                           inp["Dskip"], S0.astype(np.float64))
    y = from_dev_bf16(yh.contiguous().view(torch.bfloat16))
    assert_close(y, ref_y, "host-buffer modal conv")
    rel, _ = metrics(S_host.cpu().numpy().astype(np.float64), ref_S)
    assert rel < 1e-4


@pytest.mark.parametrize("B,L,D,K,chunk", [
    (2, 3000, 136, 7, 1000),     # hcs, chunks not a multiple of anything
    (1, 5000, 256, 128, 777),    # hcm, chunks longer than the window, ragged
    (1, 300, 64, 128, 64),       # every chunk shorter than the window
])
def test_short_host_stream_is_bitwise_the_device_single_pass(B, L, D, K, chunk):
    import torch
    import hyena_long_convolution_b200 as hy
    from synth import make_fir_inputs
    inp = make_fir_inputs(B, L, D, K, seed=L + K, with_skip=True)
    taps = to_dev_bf16(inp["taps"])
    Ds = to_dev_f32(inp["Dskip"])
    H0 = np.random.default_rng(K).standard_normal((B, K - 1, D)).astype(np.float32)
    H_in = torch.from_numpy(H0).cuda()
    xd = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    H_dev = torch.empty_like(H_in)
    y_dev = hy.short_conv(*xd, taps, Ds, hist_in=H_in, hist_out=H_dev)
    xh = [_host_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    yh = _host_bf16(np.zeros((B, L, D), np.uint16))
    H_host = torch.empty_like(H_in)
    hy.short_conv_host(*xh, taps, Ds, y=yh, hist_in=H_in, hist_out=H_host, chunk=chunk)
    torch.cuda.synchronize()
    assert torch.equal(yh.contiguous().view(torch.int16), y_dev.view(torch.int16).cpu())
    assert torch.equal(H_host, H_dev)
    if K == 128 and L == 5000:
        ref_y, ref_H = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"], H0.astype(np.float64))
        assert_close(from_dev_bf16(yh.contiguous().view(torch.bfloat16)), ref_y, "host-buffer short conv")


def test_host_stream_with_pageable_memory():
    # pageable host buffers: the copies do not overlap, the result is the same
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, N = 1, 2000, 64, 8
    inp = make_modal_inputs(B, L, D, N, seed=3)
    a, R, Ds = (to_dev_f32(inp[k]) for k in ("log_poles", "residues", "Dskip"))
    y_dev = hy.modal_long_conv(*(to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")), a, R, Ds)
    xh = [torch.from_numpy(np.ascontiguousarray(inp[k]).view(np.int16)) for k in ("x1", "x2", "x3")]
    yh = torch.zeros((B, L, D), dtype=torch.int16)
    hy.modal_long_conv_host(*xh, a, R, Ds, y=yh, workspace=hy.HostWorkspace(B, D, N, chunk=512))
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.view(torch.int16).cpu())
