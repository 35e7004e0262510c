"""GPU parity of the complex-mode long modal filter (h[t] = Re sum R p^t)
against the fp64 oracle, chunking, and the complex decode step.
"""
import numpy as np
import pytest

import oracle
from synth import make_cmodal_inputs

from .helpers import assert_close, bits_of, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu

STATE_TOL = 1e-4


def dev(inp):
    x = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    return x, to_dev_f32(inp["poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])


@pytest.mark.parametrize("B,L,D,N", [
    (1, 1, 64, 8), (1, 700, 64, 8), (2, 300, 136, 3), (1, 1000, 128, 1), (3, 129, 72, 5),
    (2, 257, 24, 2), (1, 4100, 520, 8), (1, 20000, 64, 4),
    # more than 8 complex modes (16 slots): lanes share a channel pair
    (1, 1000, 64, 9), (2, 300, 48, 16), (1, 2100, 40, 32),
])
def test_shapes_with_state(B, L, D, N):
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_cmodal_inputs(B, L, D, N, seed=B + L + D + N)
    S0 = np.random.default_rng(L).standard_normal((B, D, N, 2)).astype(np.float32)
    x, p, R, Ds = dev(inp)
    ws = hy.ModalWorkspace(B, D, 2 * N)
    S_out = torch.empty((B, D, N, 2), device="cuda")
    y = hy.modal_long_conv_complex(*x, p, R, Ds, state_in=torch.from_numpy(S0).cuda(), state_out=S_out,
                                   workspace=ws)
    hy.workspace_check(ws)
    ref_y, ref_S = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"],
                                            inp["Dskip"], S0.astype(np.float64))
    assert_close(from_dev_bf16(y), ref_y, "complex y")
    rel, _ = metrics(S_out.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= STATE_TOL, rel


def test_evo1_shape_full_tensor():
    """B=1, L=8192, D=4096, N=8 complex modes (the Evo 1 width, state size and
    context), every output compared."""
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_cmodal_inputs(1, 8192, 4096, 8, seed=8)
    x, p, R, Ds = dev(inp)
    S = torch.empty((1, 4096, 8, 2), device="cuda")
    y = hy.modal_long_conv_complex(*x, p, R, Ds, state_out=S)
    ref_y, ref_S = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"],
                                            inp["Dskip"])
    assert_close(from_dev_bf16(y), ref_y, "evo1-shape y", per_channel=True)
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= STATE_TOL, rel


def test_whole_unit_chunks_are_bit_exact_and_ragged_chunks_close():
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, N = 1, 1024, 128, 6  # one batch row: time slices stay valid [B, L, D] views
    inp = make_cmodal_inputs(B, L, D, N, seed=4)
    x, p, R, Ds = dev(inp)
    S1 = torch.empty((B, D, N, 2), device="cuda")
    y1 = hy.modal_long_conv_complex(*x, p, R, Ds, state_out=S1)
    ws = hy.ModalWorkspace(B, D, 2 * N)
    for chunks in ([128] * 8, [256, 512, 256]):
        S = torch.zeros((B, D, N, 2), device="cuda")
        y2 = torch.empty_like(y1)
        t0 = 0
        for n in chunks:
            hy.modal_long_conv_complex(*(v[:, t0:t0 + n] for v in x), p, R, Ds, y=y2[:, t0:t0 + n],
                                       state_in=S, state_out=S, workspace=ws)
            t0 += n
        torch.cuda.synchronize()
        assert np.array_equal(bits_of(y1), bits_of(y2))
        assert torch.equal(S, S1)
    chunks = [1, 127, 300, 2, 594]
    S = torch.zeros((B, D, N, 2), device="cuda")
    y3 = torch.empty_like(y1)
    t0 = 0
    for n in chunks:
        hy.modal_long_conv_complex(*(v[:, t0:t0 + n] for v in x), p, R, Ds, y=y3[:, t0:t0 + n],
                                   state_in=S, state_out=S, workspace=ws)
        t0 += n
    ref_y, ref_S = oracle.cmodal_chunked(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"],
                                         inp["Dskip"], None, chunks=chunks)
    assert_close(from_dev_bf16(y3), ref_y, "ragged chunks")
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= STATE_TOL, rel


@pytest.mark.parametrize("B,D,N", [(1, 64, 1), (2, 136, 5), (3, 4096, 8), (1, 64, 9), (2, 96, 32)])
def test_decode_step_matches_oracle_and_prefill(B, D, N):
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_cmodal_inputs(B, 1, D, N, seed=3 + N)
    S0 = np.random.default_rng(D).standard_normal((B, D, N, 2)).astype(np.float32)
    x, p, R, Ds = dev(inp)
    S = torch.from_numpy(S0).cuda()
    y = hy.modal_decode_complex(*x, p, R, Ds, S)  # [B, 1, D] views, y like x1
    ref_y, ref_S = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"],
                                            inp["Dskip"], S0.astype(np.float64))
    assert_close(from_dev_bf16(y), ref_y, "complex decode y")
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= 1e-5, rel
    S2 = torch.from_numpy(S0).cuda()
    y2 = hy.modal_long_conv_complex(*x, p, R, Ds, state_in=S2, state_out=S2)
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(y), bits_of(y2))
    assert np.array_equal(S.cpu().numpy().view(np.uint32), S2.cpu().numpy().view(np.uint32))


def test_decode_continues_a_prefill():
    import torch
    import hyena_long_convolution_b200 as hy
    B, L0, T, D, N = 2, 300, 40, 128, 8
    inp = make_cmodal_inputs(B, L0 + T, D, N, seed=12)
    x, p, R, Ds = dev(inp)
    S = torch.zeros((B, D, N, 2), device="cuda")
    ys = [from_dev_bf16(hy.modal_long_conv_complex(*(v[:, :L0].contiguous() for v in x), p, R, Ds, state_out=S))]
    for t in range(L0, L0 + T):
        ys.append(from_dev_bf16(hy.modal_decode_complex(*(v[:, t:t + 1] for v in x), p, R, Ds, S)))
    ref_y, ref_S = oracle.cmodal_chunked(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"],
                                         inp["Dskip"], None, chunks=[L0] + [1] * T)
    assert_close(np.concatenate(ys, axis=1), ref_y, "prefill + decode")
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel <= 1e-5, rel


def test_conjugated_parameters_give_the_same_output():
    """Re(R p^t) = Re(conj R conj p^t): the GPU output is unchanged (within
    rounding) and the state comes out conjugated."""
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, N = 1, 600, 64, 4
    inp = make_cmodal_inputs(B, L, D, N, seed=21)
    x, p, R, Ds = dev(inp)
    conj = torch.tensor([1.0, -1.0], device="cuda")
    S1 = torch.empty((B, D, N, 2), device="cuda")
    S2 = torch.empty((B, D, N, 2), device="cuda")
    y1 = hy.modal_long_conv_complex(*x, p, R, Ds, state_out=S1)
    y2 = hy.modal_long_conv_complex(*x, (p * conj).contiguous(), (R * conj).contiguous(), Ds, state_out=S2)
    assert_close(from_dev_bf16(y2), from_dev_bf16(y1), "conjugated")
    rel, _ = metrics((S2 * conj).cpu().numpy().astype(np.float64), S1.cpu().numpy().astype(np.float64))
    assert rel <= 1e-5, rel
