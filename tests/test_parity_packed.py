"""Packed projection inputs: x1, x2, x3 read from one [B, L, >= 3D] buffer in
channel groups (group = 1: per-channel triples x1_c x2_c x3_c), against the
fp64 oracle and bit for bit against the plain entry points on the same values
(both layouts feed identical operands to identical arithmetic).
"""
import numpy as np
import pytest

import oracle
from synth import make_cmodal_inputs, make_fir_inputs, make_modal_inputs

from .helpers import assert_close, bits_of, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


def pack(x1, x2, x3, group, ld_pad=0):
    """[B, L, D] bf16 bit arrays -> [B, L, 3D + ld_pad] with x_k of channel c at
    column 3 group (c // group) + (k-1) group + c % group."""
    B, L, D = x1.shape
    g = np.stack([x.reshape(B, L, D // group, group) for x in (x1, x2, x3)], axis=3)
    xp = g.reshape(B, L, 3 * D)
    if ld_pad:
        xp = np.concatenate([xp, np.full((B, L, ld_pad), 0x7FC0, np.uint16)], axis=2)  # NaN padding
    return np.ascontiguousarray(xp)


def dev_packed(inp, group, ld_pad=0):
    return to_dev_bf16(pack(inp["x1"], inp["x2"], inp["x3"], group, ld_pad))


def test_pack_layout_formula():
    """The test's packing puts x_k[b, t, c] at 3 G (c // G) + (k-1) G + c % G."""
    rng = np.random.default_rng(0)
    xs = [rng.integers(0, 1 << 16, (2, 3, 48), dtype=np.uint16) for _ in range(3)]
    for G in (1, 8, 16, 48):
        xp = pack(*xs, G)
        for c in range(48):
            for k in range(3):
                assert np.array_equal(xp[:, :, 3 * G * (c // G) + k * G + c % G], xs[k][:, :, c])


MODAL_CASES = [
    # B, L, D, N, group, ld_pad
    (1, 700, 64, 16, 1, 0),
    (2, 300, 136, 8, 1, 8),
    (1, 1000, 128, 16, 8, 0),
    (1, 1000, 128, 12, 16, 0),
    (2, 257, 128, 16, 32, 16),
    (2, 500, 192, 5, 64, 0),
    (1, 300, 256, 16, 128, 0),
    (1, 300, 136, 16, 136, 0),
    (1, 300, 48, 8, 48, 0),
    (1, 300, 48, 8, 1, 8),
    (1, 4100, 520, 16, 1, 0),
]


@pytest.mark.parametrize("B,L,D,N,group,ld_pad", MODAL_CASES)
def test_modal_packed(B, L, D, N, group, ld_pad):
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_modal_inputs(B, L, D, N, seed=B + L + D + N + group)
    S0 = np.random.default_rng(L).standard_normal((B, D, N)).astype(np.float32)
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    xp = dev_packed(inp, group, ld_pad)
    S_in = torch.from_numpy(S0).cuda()
    S_p = torch.empty_like(S_in)
    ws = hy.ModalWorkspace(B, D, N)
    y = hy.modal_long_conv_packed(xp, group, a, R, Ds, state_in=S_in, state_out=S_p, workspace=ws)
    hy.workspace_check(ws)
    # plain entry point on the same values
    S_q = torch.empty_like(S_in)
    yq = hy.modal_long_conv(*(to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")), a, R, Ds,
                            state_in=S_in, state_out=S_q)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y), bits_of(yq))
    assert np.array_equal(S_p.cpu().numpy().view(np.uint32), S_q.cpu().numpy().view(np.uint32))
    ref_y, ref_S = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"],
                                           inp["Dskip"], S0.astype(np.float64))
    assert_close(from_dev_bf16(y), ref_y, "packed y")
    rel, _ = metrics(S_p.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= 1e-4, rel


def test_modal_packed_chunked_matches_single_pass():
    """Chunks of whole 128-token units through the triples path reproduce the
    single pass bit for bit (the views advance along L of the packed buffer)."""
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, N = 1, 1024, 128, 16
    inp = make_modal_inputs(B, L, D, N, seed=5)
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    xp = dev_packed(inp, 1)
    y1 = hy.modal_long_conv_packed(xp, 1, a, R, Ds)
    S = torch.zeros((B, D, N), device="cuda")
    y2 = torch.empty_like(y1)
    for t0 in range(0, L, 256):
        hy.modal_long_conv_packed(xp[:, t0:t0 + 256], 1, a, R, Ds, y=y2[:, t0:t0 + 256], state_in=S, state_out=S)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y1), bits_of(y2))


FIR_CASES = [
    # B, L, D, K, group, ld_pad
    (1, 300, 64, 7, 1, 0),
    (2, 257, 136, 128, 1, 8),
    (1, 300, 64, 1, 1, 0),
    (2, 520, 128, 33, 1, 0),
    (1, 300, 128, 128, 8, 0),
    (2, 257, 192, 7, 64, 16),
    (1, 300, 256, 128, 128, 0),
    (1, 200, 136, 15, 136, 0),
    (1, 200, 48, 128, 48, 0),
    (1, 200, 48, 7, 1, 0),
]


@pytest.mark.parametrize("B,L,D,K,group,ld_pad", FIR_CASES)
def test_short_conv_packed(B, L, D, K, group, ld_pad):
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_fir_inputs(B, L, D, K, seed=K + L + group, with_skip=True)
    H0 = np.random.default_rng(K).standard_normal((B, K - 1, D)).astype(np.float32)
    taps, Ds = to_dev_bf16(inp["taps"]), to_dev_f32(inp["Dskip"])
    xp = dev_packed(inp, group, ld_pad)
    H_in = torch.from_numpy(H0).cuda() if K > 1 else None
    H_p = torch.empty_like(H_in) if K > 1 else None
    y = hy.short_conv_packed(xp, group, taps, Ds, hist_in=H_in, hist_out=H_p)
    H_q = torch.empty_like(H_in) if K > 1 else None
    yq = hy.short_conv(*(to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")), taps, Ds, hist_in=H_in, hist_out=H_q)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y), bits_of(yq))
    ref_y, ref_H = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"],
                              H0.astype(np.float64) if K > 1 else None)
    assert_close(from_dev_bf16(y), ref_y, "packed fir y")
    if K > 1:
        assert np.array_equal(H_p.cpu().numpy().view(np.uint32), H_q.cpu().numpy().view(np.uint32))
        assert np.array_equal(H_p.cpu().numpy().astype(np.float64), ref_H)


@pytest.mark.parametrize("group", [1, 16, 128])
def test_decode_packed(group):
    import torch
    import hyena_long_convolution_b200 as hy
    B, D, N, K = 3, 128, 16, 128
    inp = make_modal_inputs(B, 1, D, N, seed=31 + group)
    xp = dev_packed(inp, group, ld_pad=8)
    xp = xp[:, 0]  # [B, W]: one token per batch row
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    S0 = torch.randn((B, D, N), device="cuda")
    S1, S2 = S0.clone(), S0.clone()
    y = hy.modal_decode_packed(xp, group, a, R, Ds, S1)
    yq = hy.modal_decode(*(to_dev_bf16(inp[k])[:, 0] for k in ("x1", "x2", "x3")), a, R, Ds, S2)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y), bits_of(yq))
    assert torch.equal(S1, S2)
    ref_y, _ = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"],
                                       inp["Dskip"], S0.cpu().numpy().astype(np.float64))
    assert_close(from_dev_bf16(y)[:, None, :], ref_y, "packed decode y")

    taps = to_dev_bf16(make_fir_inputs(1, 1, D, K, seed=3)["taps"])
    H0 = torch.randn((B, K - 1, D), device="cuda")
    H1, H2 = H0.clone(), H0.clone()
    yf = hy.short_decode_packed(xp, group, taps, Ds, H1)
    yfq = hy.short_decode(*(to_dev_bf16(inp[k])[:, 0] for k in ("x1", "x2", "x3")), taps, Ds, H2)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(yf), bits_of(yfq))
    assert torch.equal(H1, H2)


@pytest.mark.parametrize("group", [1, 64])
def test_complex_modes_packed(group):
    """Complex modes from a packed buffer: bit-equal to the plain complex call,
    prefill and decode."""
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, N = 2, 300, 128, 8
    inp = make_cmodal_inputs(B, L, D, N, seed=17 + group)
    p, R, Ds = to_dev_f32(inp["poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    xp = dev_packed(inp, group, ld_pad=8)
    S0 = torch.randn((B, D, N, 2), device="cuda")
    S1, S2 = torch.empty_like(S0), torch.empty_like(S0)
    y = hy.modal_long_conv_complex_packed(xp, group, p, R, Ds, state_in=S0, state_out=S1)
    xs = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    yq = hy.modal_long_conv_complex(*xs, p, R, Ds, state_in=S0, state_out=S2)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y), bits_of(yq))
    assert torch.equal(S1, S2)
    ref_y, _ = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"],
                                        inp["Dskip"], S0.cpu().numpy().astype(np.float64))
    assert_close(from_dev_bf16(y), ref_y, "complex packed y")
    # one decode step from the packed buffer's first row
    S3, S4 = S0.clone(), S0.clone()
    yd = hy.modal_decode_complex_packed(xp[:, 0], group, p, R, Ds, S3)
    ydq = hy.modal_decode_complex(*(x[:, 0] for x in xs), p, R, Ds, S4)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(yd), bits_of(ydq))
    assert torch.equal(S3, S4)
