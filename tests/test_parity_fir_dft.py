"""GPU parity of the tensor-core FIR (hyena_short_conv_dft: overlap-save
DFT-as-GEMM, tf32 operands) against the fp64 oracle.

The DFT path rounds its operands to tf32, so it is held to the acceptance
tolerance (not to the SIMT kernels' bits); the history it writes is the exact
fp32 v, as in the oracle.  Chunk boundaries at multiples of its 128-token
block keep every block, so such chunkings reproduce the single pass bit for
bit.
"""
import numpy as np
import pytest

import oracle
from synth import WORKLOAD_SHAPES, make_fir_inputs

from .helpers import MAX_ABS_TOL, REL_L2_TOL, assert_close, bits_of, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


def run_dft(inp, hist_in=None, chunks=None):
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, K = inp["B"], inp["L"], inp["D"], inp["K"]
    xs = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    taps, Ds = to_dev_bf16(inp["taps"]), to_dev_f32(inp["Dskip"])
    H = to_dev_f32(hist_in) if hist_in is not None else torch.zeros((B, K - 1, D), device="cuda")
    if chunks is None:
        H_out = torch.empty_like(H)
        y = hy.short_conv_dft(*xs, taps, Ds, hist_in=H if hist_in is not None else None,
                              hist_out=H_out if K > 1 else None)
    else:
        H_out = H
        parts, t0 = [], 0
        for n in chunks:
            parts.append(hy.short_conv_dft(*(x[:, t0:t0 + n].contiguous() for x in xs), taps, Ds,
                                           hist_in=H_out if K > 1 else None, hist_out=H_out if K > 1 else None))
            t0 += n
        y = torch.cat(parts, dim=1)
    torch.cuda.synchronize()
    return y, H_out


def check(inp, hist_in=None, **kw):
    y, H = run_dft(inp, hist_in, **kw)
    ref_y, ref_H = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"], hist_in)
    assert_close(from_dev_bf16(y), ref_y, "dft fir y")
    if inp["K"] > 1:
        assert np.array_equal(H.cpu().numpy().astype(np.float64), ref_H)
    return y, H


@pytest.mark.parametrize("K", [1, 7, 33, 128])
@pytest.mark.parametrize("B,L,D", [(1, 300, 64), (2, 257, 136), (1, 130, 48)])
def test_shapes(K, B, L, D):
    inp = make_fir_inputs(B, L, D, K, seed=K * 5 + L, with_skip=True)
    H = np.random.default_rng(K).standard_normal((B, K - 1, D)).astype(np.float32).astype(np.float64)
    check(inp, H)
    check(inp)


@pytest.mark.parametrize("L", [1, 127, 128, 129])
def test_short_sequences(L):
    inp = make_fir_inputs(1, L, 64, 128, seed=L + 3, with_skip=True)
    H = np.random.default_rng(L).standard_normal((1, 127, 64)).astype(np.float32).astype(np.float64)
    check(inp, H)


def test_many_ctas_and_chunks():
    # 3 x 17 x 8 CTAs, ragged L and D; chunks at multiples of 128 keep every
    # block (bit for bit), other chunkings stay within the tolerance
    inp = make_fir_inputs(3, 1000, 1032, 128, seed=21, with_skip=True)
    H = np.random.default_rng(4).standard_normal((3, 127, 1032)).astype(np.float32).astype(np.float64)
    y, Hout = check(inp, H)
    yc, Hc = run_dft(inp, H, chunks=[256, 512, 232])
    assert np.array_equal(bits_of(yc), bits_of(y))
    assert np.array_equal(Hc.cpu().numpy(), Hout.cpu().numpy())
    check(inp, H, chunks=[100, 333, 567])


def test_against_the_simt_kernel():
    # The two implementations of the operator, both checked against the
    # oracle above, agree to the acceptance bounds; each output carries its
    # own bf16 rounding, so two of them may differ by a whole bf16 ulp where
    # one and the exact value differ by half: the max-abs bound doubles.
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_fir_inputs(2, 2048, 256, 128, seed=8, with_skip=True)
    xs = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    taps, Ds = to_dev_bf16(inp["taps"]), to_dev_f32(inp["Dskip"])
    y_simt = from_dev_bf16(hy.short_conv(*xs, taps, Ds))
    y_dft = from_dev_bf16(hy.short_conv_dft(*xs, taps, Ds))
    torch.cuda.synchronize()
    rel, mabs = metrics(y_dft, y_simt)
    print(f"dft vs simt: rel-L2 {rel:.3e}, max-abs/rms {mabs:.3e}")
    assert rel <= REL_L2_TOL and mabs <= 2 * MAX_ABS_TOL


@pytest.mark.slow
def test_fir128_full_size():
    # every element of the B=2, L=8192, D=4096, K=128 output against the oracle
    c = WORKLOAD_SHAPES["fir_8k"]
    inp = make_fir_inputs(c["B"], c["L"], c["D"], 128, c["seed"])
    y, _ = run_dft(inp)
    ref, _ = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], None, None)
    assert_close(from_dev_bf16(y), ref, "dft FIR 8K K=128")


def test_row_strides_and_aliased_window():
    # x1, x2, x3 as three views of one [B, L, 3D + pad] buffer (row stride >
    # D), y with a padded row stride, and hist_in == hist_out
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, K = 2, 700, 192, 128
    inp = make_fir_inputs(B, L, D, K, seed=33, with_skip=True)
    H0 = np.random.default_rng(5).standard_normal((B, K - 1, D)).astype(np.float32)
    wide = np.concatenate([inp["x1"], inp["x2"], inp["x3"], np.zeros((B, L, 64), np.uint16)], axis=2)
    buf = to_dev_bf16(wide)
    xs = [buf[..., :D], buf[..., D:2 * D], buf[..., 2 * D:3 * D]]
    ybuf = torch.zeros((B, L, D + 32), dtype=torch.bfloat16, device="cuda")
    y = ybuf[..., :D]
    H = torch.from_numpy(H0).cuda()
    hy.short_conv_dft(*xs, to_dev_bf16(inp["taps"]), to_dev_f32(inp["Dskip"]), y=y, hist_in=H, hist_out=H)
    torch.cuda.synchronize()
    ref_y, ref_H = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"], H0.astype(np.float64))
    assert_close(from_dev_bf16(y), ref_y, "dft fir, strided views")
    assert np.array_equal(H.cpu().numpy().astype(np.float64), ref_H)
    assert torch.count_nonzero(ybuf[..., D:]) == 0  # the padding columns are not written
