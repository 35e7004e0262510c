"""Decode steps (one generated token) against the fp64 oracle, and against the
prefill entry points on one-token sequences (which they must match bit for
bit).  The oracle's recurrence form with L = 1 and a carried state is the
decode step by definition; a run of decode steps is the oracle's chunked
evaluation with chunks of one token.
"""
import numpy as np
import pytest

import oracle
from synth import make_fir_inputs, make_modal_inputs

from .helpers import assert_close, bits_of, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,D,N", [(1, 64, 1), (2, 136, 5), (3, 200, 8), (1, 4096, 16), (1, 64, 17),
                                   (2, 136, 32), (1, 200, 50), (2, 4096, 64)])
def test_modal_decode_step_matches_oracle_and_prefill(B, D, N):
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_modal_inputs(B, 1, D, N, seed=7 + D + N)
    S0 = np.random.default_rng(D).standard_normal((B, D, N)).astype(np.float32)
    x = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    S = torch.from_numpy(S0).cuda()
    y = hy.modal_decode(*x, a, R, Ds, S)
    ref_y, ref_S = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"],
                                           inp["Dskip"], S0)
    assert_close(from_dev_bf16(y), ref_y, "decode y")
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= 1e-5, rel
    # the one-token prefill call gives the same bits
    S2 = torch.from_numpy(S0).cuda()
    y2 = hy.modal_long_conv(*x, a, R, Ds, state_in=S2, state_out=S2)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y), bits_of(y2))
    assert np.array_equal(S.cpu().numpy().view(np.uint32), S2.cpu().numpy().view(np.uint32))


def test_modal_decode_continues_a_prefill():
    import torch
    import hyena_long_convolution_b200 as hy
    B, L0, T, D, N = 2, 300, 40, 128, 16
    inp = make_modal_inputs(B, L0 + T, D, N, seed=11)
    x = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    S = torch.zeros((B, D, N), device="cuda")
    # the prefill layout needs batch stride = L * row stride: contiguous copies
    y0 = hy.modal_long_conv(*(v[:, :L0].contiguous() for v in x), a, R, Ds, state_out=S)
    ys = [from_dev_bf16(y0)]
    for t in range(L0, L0 + T):
        ys.append(from_dev_bf16(hy.modal_decode(*(v[:, t:t + 1] for v in x), a, R, Ds, S)))
    y = np.concatenate(ys, axis=1)
    ref_y, ref_S = oracle.modal_chunked(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"],
                                        inp["Dskip"], None, chunks=[L0] + [1] * T)
    assert_close(y, ref_y, "prefill + decode")
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= 1e-5, rel


@pytest.mark.parametrize("B,D,K", [(1, 64, 1), (2, 136, 7), (1, 200, 33), (2, 4096, 128)])
def test_short_decode_step_matches_oracle_and_prefill(B, D, K):
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_fir_inputs(B, 1, D, K, seed=5 + K)
    H0 = np.random.default_rng(K).standard_normal((B, max(K - 1, 0), D)).astype(np.float32)
    x = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    taps = to_dev_bf16(inp["taps"])
    Ds = to_dev_f32(inp["Dskip"]) if inp["Dskip"] is not None else None
    Hd = torch.from_numpy(H0).cuda() if K > 1 else None
    y = hy.short_decode(*x, taps, Ds, Hd)
    ref_y, ref_H = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"], H0 if K > 1 else None)
    assert_close(from_dev_bf16(y), ref_y, "fir decode y")
    if K > 1:
        assert np.array_equal(Hd.cpu().numpy().astype(np.float64), ref_H)  # the window holds exact v values
    H2 = torch.from_numpy(H0).cuda() if K > 1 else None
    y2 = hy.short_conv(*x, taps, Ds, hist_in=H2, hist_out=H2)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y), bits_of(y2))
    if K > 1:
        assert np.array_equal(Hd.cpu().numpy().view(np.uint32), H2.cpu().numpy().view(np.uint32))


def test_short_decode_continues_a_prefill():
    import torch
    import hyena_long_convolution_b200 as hy
    B, L0, T, D, K = 2, 200, 30, 64, 128
    inp = make_fir_inputs(B, L0 + T, D, K, seed=3)
    x = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    taps = to_dev_bf16(inp["taps"])
    Ds = to_dev_f32(inp["Dskip"]) if inp["Dskip"] is not None else None
    H = torch.zeros((B, K - 1, D), device="cuda")
    ys = [from_dev_bf16(hy.short_conv(*(v[:, :L0].contiguous() for v in x), taps, Ds, hist_out=H))]
    for t in range(L0, L0 + T):
        ys.append(from_dev_bf16(hy.short_decode(*(v[:, t:t + 1] for v in x), taps, Ds, H)))
    ref_y, ref_H = oracle.fir_chunked(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"], None,
                                      chunks=[L0] + [1] * T)
    assert_close(np.concatenate(ys, axis=1), ref_y, "fir prefill + decode")
    assert np.array_equal(H.cpu().numpy().astype(np.float64), ref_H)


def test_decode_accepts_projection_views():
    """x1, x2, x3 as views of one [B, 1, 3D] projection row (ld = 3D)."""
    import torch
    import hyena_long_convolution_b200 as hy
    B, D, N = 2, 128, 8
    inp = make_modal_inputs(B, 1, D, N, seed=21)
    packed = np.concatenate([inp["x1"], inp["x2"], inp["x3"]], axis=2)
    xp = to_dev_bf16(packed)
    x = [xp[:, :, i * D:(i + 1) * D] for i in range(3)]
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    S = torch.zeros((B, D, N), device="cuda")
    y = hy.modal_decode(*x, a, R, Ds, S)
    ref_y, _ = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"],
                                       inp["Dskip"])
    assert_close(from_dev_bf16(y), ref_y, "decode from views")
