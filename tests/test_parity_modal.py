"""GPU parity of the long modal conv (hcl) against the fp64 oracle.

Every case runs through the C ABI (via the thin binding) on seeded inputs and
compares every output element with the oracle (rel-L2 <= 5e-3, max-abs <=
2e-2 rms), plus the fp32 state (rel-L2 <= 1e-4).  Sizes span several units
(128 tokens x 64 channels) with ragged tails in time and channels.
"""
import numpy as np
import pytest

import oracle
from synth import WORKLOAD_SHAPES, make_modal_inputs

from .helpers import assert_close, bits_of, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu

STATE_TOL = 1e-4


def run_gpu(inp, state_in=None, chunks=None, ld_pad=0, alias=False):
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, N = inp["B"], inp["L"], inp["D"], inp["N"]
    if ld_pad:
        wide = np.concatenate([inp["x1"], inp["x2"], inp["x3"],
                               np.zeros((B, L, ld_pad), np.uint16)], axis=2)
        buf = to_dev_bf16(wide)
        x1, x2, x3 = buf[..., :D], buf[..., D:2 * D], buf[..., 2 * D:3 * D]
    else:
        x1, x2, x3 = (to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3"))
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    ws = hy.ModalWorkspace(B, D, N)
    S = to_dev_f32(state_in) if state_in is not None else torch.zeros((B, D, N), device="cuda")
    y = torch.empty((B, L, D), dtype=torch.bfloat16, device="cuda")
    if chunks is None:
        S_out = S if alias else torch.empty_like(S)
        hy.modal_long_conv(x1, x2, x3, a, R, Ds, y=y, state_in=S if state_in is not None else None,
                           state_out=S_out, workspace=ws)
    else:
        S_out = S
        t0 = 0
        for n in chunks:
            hy.modal_long_conv(x1[:, t0:t0 + n], x2[:, t0:t0 + n], x3[:, t0:t0 + n], a, R, Ds,
                               y=y[:, t0:t0 + n], state_in=S_out, state_out=S_out, workspace=ws)
            t0 += n
    hy.workspace_check(ws)
    torch.cuda.synchronize()
    return y, S_out


def check(inp, state_in=None, what="y", **kw):
    y, S = run_gpu(inp, state_in, **kw)
    ref_y, ref_S = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                           inp["residues"], inp["Dskip"], state_in)
    assert_close(from_dev_bf16(y), ref_y, what)
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= STATE_TOL, f"state rel-L2 {rel:.3e}"
    return y, S


def test_modal_1k_full():
    c = WORKLOAD_SHAPES["modal_1k"]
    inp = make_modal_inputs(c["B"], c["L"], c["D"], c["N"], c["seed"])
    check(inp, what="modal 1K (B=1 L=1024 D=64 N=8)")


def test_modal_1k_with_state_and_direct_form():
    c = WORKLOAD_SHAPES["modal_1k"]
    inp = make_modal_inputs(c["B"], c["L"], c["D"], c["N"], c["seed"])
    S = np.random.default_rng(1).standard_normal((1, 64, 8))
    y, _ = check(inp, S)
    # also against the independent direct O(L^2) form
    ref_d, _ = oracle.modal_direct(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                   inp["residues"], inp["Dskip"], S)
    assert_close(from_dev_bf16(y), ref_d)


@pytest.mark.parametrize("B,L,D,N", [
    (1, 1, 64, 16), (1, 2, 8, 1), (2, 127, 72, 3), (1, 128, 64, 8), (2, 129, 136, 16),
    (3, 1000, 200, 5), (1, 2048, 64, 16), (2, 4100, 520, 12), (1, 40000, 64, 4), (2, 300, 24, 4),
    # more than 16 modes: two or four lanes share a channel pair, narrower chains
    (1, 1, 32, 17), (2, 1000, 72, 20), (1, 4100, 96, 32), (1, 129, 16, 33), (2, 700, 40, 48),
    (1, 3000, 64, 64), (1, 64, 8, 64),
])
def test_shapes_ragged(B, L, D, N):
    inp = make_modal_inputs(B, L, D, N, seed=B * 1000 + L + D + N)
    S = np.random.default_rng(L).standard_normal((B, D, N))
    check(inp, S)


def test_row_stride_views_of_projection_buffer():
    inp = make_modal_inputs(2, 700, 128, 16, seed=42)
    check(inp, ld_pad=8)


def test_state_in_out_alias():
    inp = make_modal_inputs(1, 900, 64, 16, seed=43)
    S = np.random.default_rng(3).standard_normal((1, 64, 16))
    check(inp, S, alias=True)


def test_zero_length_copies_state():
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_modal_inputs(1, 0, 64, 8, seed=1)
    S = torch.randn((1, 64, 8), device="cuda")
    S2 = torch.full_like(S, 7.0)
    x = torch.empty((1, 0, 64), dtype=torch.bfloat16, device="cuda")
    hy.modal_long_conv(x, x, x, to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]),
                       state_in=S, state_out=S2)
    torch.cuda.synchronize()
    assert torch.equal(S, S2)
    hy.modal_long_conv(x, x, x, to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), state_out=S2)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S2).item() == 0


@pytest.mark.parametrize("chunks", [[128] * 8, [1024], [64] * 16, [1, 127, 300, 2, 594], [500, 524]])
def test_chunked_matches_oracle_and_single_pass(chunks):
    inp = make_modal_inputs(1, 1024, 192, 16, seed=77)
    S0 = np.random.default_rng(5).standard_normal((1, 192, 16))
    y1, s1 = check(inp, S0)
    yc, sc = check(inp, S0, chunks=chunks)
    if all(c % 128 == 0 for c in chunks):
        # chunks made of whole 128-token units reproduce the single pass bit for bit
        assert np.array_equal(bits_of(yc), bits_of(y1))
        assert np.array_equal(sc.cpu().numpy(), s1.cpu().numpy())


def test_deterministic_across_runs():
    inp = make_modal_inputs(1, 8192, 4096, 16, seed=3)
    y1, s1 = run_gpu(inp)
    y2, s2 = run_gpu(inp)
    assert np.array_equal(bits_of(y1), bits_of(y2))
    assert np.array_equal(s1.cpu().numpy(), s2.cpu().numpy())


def test_special_values_propagate():
    # Inf in x1 at t0 makes v infinite there: outputs at t < t0 stay finite and
    # bitwise unchanged.
    inp = make_modal_inputs(1, 512, 64, 4, seed=9)
    y0, _ = run_gpu(inp)
    x1 = inp["x1"].copy()
    x1[0, 300, 5] = 0x7F80  # +inf
    inp2 = dict(inp, x1=x1)
    y1, _ = run_gpu(inp2)
    b0, b1 = bits_of(y0), bits_of(y1)
    assert np.array_equal(b0[:, :300], b1[:, :300])
    assert np.array_equal(b0[:, :, :5], b1[:, :, :5]) and np.array_equal(b0[:, :, 6:], b1[:, :, 6:])
    assert not np.all(np.isfinite(from_dev_bf16(y1)[0, 300:, 5]))


@pytest.mark.parametrize("N", [32, 64])
def test_many_modes_8k_by_1024_channels(N):
    # 1 <= N <= 64 real modes at a longer size: every element against the oracle
    inp = make_modal_inputs(1, 8192, 1024, N, seed=N)
    S = np.random.default_rng(N).standard_normal((1, 1024, N))
    check(inp, S)


@pytest.mark.parametrize("N", [20, 64])
def test_many_modes_whole_unit_chunks_are_bit_exact(N):
    inp = make_modal_inputs(1, 1024, 64, N, seed=7 + N)
    S0 = np.random.default_rng(9).standard_normal((1, 64, N))
    y1, s1 = check(inp, S0)
    yc, sc = check(inp, S0, chunks=[256, 128, 640])
    assert np.array_equal(bits_of(yc), bits_of(y1))
    assert np.array_equal(sc.cpu().numpy(), s1.cpu().numpy())


@pytest.mark.parametrize("chunks", [[1024] * 6, [3072, 3072], [4096, 2048], [128, 5888, 128]])
def test_short_and_lookback_paths_agree_bitwise(chunks):
    # The single pass (48 units per chain) runs the look-back kernel; chunks of
    # at most 24 units run the two-pass short-sequence path, longer ones the
    # look-back kernel again.  Both form every value by the same operations,
    # so any mix of them reproduces the single pass bit for bit.
    inp = make_modal_inputs(1, 6144, 520, 12, seed=31)
    S0 = np.random.default_rng(31).standard_normal((1, 520, 12))
    y1, s1 = check(inp, S0)
    yc, sc = run_gpu(inp, S0, chunks=chunks)
    assert np.array_equal(bits_of(yc), bits_of(y1))
    assert np.array_equal(sc.cpu().numpy(), s1.cpu().numpy())


@pytest.mark.parametrize("chunks", [[1024] * 6, [4096, 2048]])
def test_prepared_chunks_equal_the_plain_calls(chunks):
    # the filter synthesised once (hyena_modal_prepare) and the chunks run
    # without it give the bits of the plain calls and of the single pass
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_modal_inputs(1, 6144, 520, 12, seed=41)
    S0 = np.random.default_rng(41).standard_normal((1, 520, 12))
    y1, s1 = check(inp, S0)
    x = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    a, R, Ds = (to_dev_f32(inp[k]) for k in ("log_poles", "residues", "Dskip"))
    ws = hy.ModalWorkspace(1, 520, 12)
    S = to_dev_f32(S0)
    y = torch.empty((1, 6144, 520), dtype=torch.bfloat16, device="cuda")
    hy.modal_prepare(a, R, Ds, ws)
    t0 = 0
    for n in chunks:
        hy.modal_long_conv_prepared(*(v[:, t0:t0 + n] for v in x), 12, ws, y=y[:, t0:t0 + n], state_in=S,
                                    state_out=S)
        t0 += n
    hy.workspace_check(ws)
    assert np.array_equal(bits_of(y), bits_of(y1))
    assert np.array_equal(S.cpu().numpy(), s1.cpu().numpy())


@pytest.mark.parametrize("L", [1000, 5000])
def test_degenerate_filters(L):
    # p = 1 (a = 0: every mode a running sum), p underflowing to a denormal or
    # zero (a = -100, -200: the filter is R at lag 0 only), R = 0 (y = D v),
    # N = 1, and ordinary modes, channel block by channel block; the short
    # path (L = 1000) and the look-back kernel (L = 5000) against the oracle,
    # each channel against its own scale.
    inp = make_modal_inputs(1, L, 64, 4, seed=L)
    a = inp["log_poles"].copy()
    R = inp["residues"].copy()
    a[0:16] = 0.0
    a[16:24] = -100.0
    a[24:32] = -200.0
    R[32:48] = 0.0
    inp = dict(inp, log_poles=a, residues=R)
    y, S = run_gpu(inp)
    ref_y, ref_S = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], a, R, inp["Dskip"])
    assert_close(from_dev_bf16(y), ref_y, f"degenerate filters L={L}", per_channel=True)
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= STATE_TOL
    # a single real mode
    one = make_modal_inputs(2, L, 72, 1, seed=L + 1)
    check(one, np.random.default_rng(L).standard_normal((2, 72, 1)), what=f"N=1 L={L}")
