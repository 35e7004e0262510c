"""GPU parity of the explicit short FIR (hcs / hcm) against the fp64 oracle."""
import numpy as np
import pytest

import oracle
from synth import WORKLOAD_SHAPES, make_fir_inputs

from .helpers import assert_close, bits_of, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


def run_gpu(inp, hist_in=None, chunks=None, alias=False, ld_pad=0):
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, K = inp["B"], inp["L"], inp["D"], inp["K"]
    if ld_pad:
        wide = np.concatenate([inp["x1"], inp["x2"], inp["x3"],
                               np.zeros((B, L, ld_pad), np.uint16)], axis=2)
        buf = to_dev_bf16(wide)
        xs = [buf[..., :D], buf[..., D:2 * D], buf[..., 2 * D:3 * D]]
    else:
        xs = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    taps = to_dev_bf16(inp["taps"])
    Ds = to_dev_f32(inp["Dskip"])
    y = torch.empty((B, L, D), dtype=torch.bfloat16, device="cuda")
    H = to_dev_f32(hist_in) if hist_in is not None else torch.zeros((B, K - 1, D), device="cuda")
    if chunks is None:
        H_out = H if alias else torch.empty_like(H)
        hy.short_conv(*xs, taps, Ds, y=y, hist_in=H if hist_in is not None else None,
                      hist_out=H_out if K > 1 else None)
    else:
        H_out = H
        t0 = 0
        for n in chunks:
            hy.short_conv(*(x[:, t0:t0 + n] for x in xs), taps, Ds, y=y[:, t0:t0 + n],
                          hist_in=H_out if K > 1 else None, hist_out=H_out if K > 1 else None)
            t0 += n
    torch.cuda.synchronize()
    return y, H_out


def check(inp, hist_in=None, **kw):
    y, H = run_gpu(inp, hist_in, **kw)
    ref_y, ref_H = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"], hist_in)
    assert_close(from_dev_bf16(y), ref_y)
    if inp["K"] > 1:
        # the history holds exact fp32 products of bf16 values
        assert np.array_equal(H.cpu().numpy().astype(np.float64), ref_H)
    return y, H


@pytest.mark.parametrize("K", [1, 2, 7, 8, 9, 15, 64, 127, 128])
@pytest.mark.parametrize("B,L,D", [(1, 300, 64), (2, 257, 136), (1, 130, 48)])
def test_shapes(K, B, L, D):
    inp = make_fir_inputs(B, L, D, K, seed=K * 7 + L, with_skip=True)
    H = np.random.default_rng(K).standard_normal((B, K - 1, D)).astype(np.float32).astype(np.float64)
    check(inp, H)
    check(inp)


@pytest.mark.parametrize("L", [1, 2, 5, 128, 129])
def test_short_sequences(L):
    inp = make_fir_inputs(1, L, 64, 128, seed=L, with_skip=True)
    H = np.random.default_rng(L).standard_normal((1, 127, 64)).astype(np.float32).astype(np.float64)
    check(inp, H)


def test_row_stride_and_alias():
    inp = make_fir_inputs(2, 500, 128, 7, seed=5, with_skip=True)
    H = np.random.default_rng(2).standard_normal((2, 6, 128)).astype(np.float32).astype(np.float64)
    check(inp, H, ld_pad=16, alias=True)


@pytest.mark.parametrize("K", [7, 128])
@pytest.mark.parametrize("chunks", [[1, 2, 3, 994], [100] * 10, [1000]])
def test_chunked_is_bitwise_single_pass(K, chunks):
    inp = make_fir_inputs(1, 1000, 128, K, seed=K, with_skip=True)
    y1, H1 = run_gpu(inp)
    yc, Hc = run_gpu(inp, chunks=chunks)
    assert np.array_equal(bits_of(yc), bits_of(y1))
    assert np.array_equal(Hc.cpu().numpy(), H1.cpu().numpy())


@pytest.mark.parametrize("K", [33, 128])
def test_ranges_of_many_tiles(K):
    # 3 x 17 x 8 = 408 tiles of 64 channels x 128 tokens, more than a B200 has
    # SMs: the long-filter kernel then walks ranges of several tiles that cross
    # from one (batch row, channel group) sequence into the next, with ragged
    # L and D, a carried window and both input layouts.
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D = 3, 1000, 1032
    inp = make_fir_inputs(B, L, D, K, seed=K + 11, with_skip=True)
    H = np.random.default_rng(K).standard_normal((B, K - 1, D)).astype(np.float32).astype(np.float64)
    y, Hout = check(inp, H)
    # the interleaved per-channel triples give the same bits
    xp = to_dev_bf16(np.stack([inp["x1"], inp["x2"], inp["x3"]], axis=3).reshape(B, L, 3 * D))
    yt = hy.short_conv_packed(xp, 1, to_dev_bf16(inp["taps"]), to_dev_f32(inp["Dskip"]), hist_in=to_dev_f32(H))
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(yt), bits_of(y))
    # chunk boundaries move every range and tile; each output's sum does not change
    xs = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    taps, Ds = to_dev_bf16(inp["taps"]), to_dev_f32(inp["Dskip"])
    Hc = to_dev_f32(H)
    parts = []
    for t0, t1 in ((0, 500), (500, 1000)):
        parts.append(hy.short_conv(*(x[:, t0:t1].contiguous() for x in xs), taps, Ds, hist_in=Hc, hist_out=Hc))
    yc = torch.cat(parts, dim=1)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(yc), bits_of(y))
    assert np.array_equal(Hc.cpu().numpy(), Hout.cpu().numpy())


@pytest.mark.slow
@pytest.mark.parametrize("K", list(WORKLOAD_SHAPES["fir_8k"]["K"]))
def test_fir_8k_full_size(K):
    # every element of the B=2, L=8192, D=4096 output against the oracle
    c = WORKLOAD_SHAPES["fir_8k"]
    inp = make_fir_inputs(c["B"], c["L"], c["D"], K, c["seed"])
    y, _ = run_gpu(inp)
    ref, _ = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], None, None)
    assert_close(from_dev_bf16(y), ref, f"FIR 8K K={K}")
