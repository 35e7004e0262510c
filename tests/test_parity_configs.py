"""Parity at the five acceptance workloads' full sizes, in the launch
configuration the benchmark times.

Every element of every output tensor is compared with the fp64 oracle: the
32K-token modal workload in one oracle call, the 131K- and 262K-token
workloads with the oracle run block of channels by block of channels (its
fp64 output for the whole tensor would not fit in host memory at once), and
the FIR workloads in their own file.  Chunked feeding in whole 128-token units
must also reproduce the single pass bit for bit over the whole tensor, so the
chunked results are covered by the same comparison.  The 262K-token workload
(wide per-channel dynamic range) is also held to the max-abs bound channel by
channel, and its per-channel rel-L2 percentiles are printed.
"""
import numpy as np
import pytest

import oracle
from synth import WORKLOAD_SHAPES, make_workload_inputs

from .helpers import StreamedCompare, assert_close, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CHANNEL_BLOCK = 256


class Dev:
    def __init__(self, inp):
        self.x = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
        self.a = to_dev_f32(inp["log_poles"])
        self.R = to_dev_f32(inp["residues"])
        self.Ds = to_dev_f32(inp["Dskip"])


def modal_run(dev, inp, chunk=None):
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, N = inp["B"], inp["L"], inp["D"], inp["N"]
    ws = hy.ModalWorkspace(B, D, N)
    y = torch.empty((B, L, D), dtype=torch.bfloat16, device="cuda")
    S = torch.zeros((B, D, N), device="cuda")
    if chunk is None:
        hy.modal_long_conv(*dev.x, dev.a, dev.R, dev.Ds, y=y, state_out=S, workspace=ws)
    else:
        for t0 in range(0, L, chunk):
            sl = slice(t0, min(L, t0 + chunk))
            hy.modal_long_conv(*(x[:, sl] for x in dev.x), dev.a, dev.R, dev.Ds, y=y[:, sl],
                               state_in=S, state_out=S, workspace=ws)
    hy.workspace_check(ws)
    torch.cuda.synchronize()
    return y, S


def streamed_oracle_check(y, S, inp, what, per_channel=False):
    """Every element of y and of the final state against the fp64 recurrence
    oracle, one block of channels at a time."""
    D = inp["D"]
    cmp = StreamedCompare(D)
    S_host = S.cpu().numpy().astype(np.float64)
    s_err = s_ref = 0.0
    for c0 in range(0, D, CHANNEL_BLOCK):
        c1 = min(D, c0 + CHANNEL_BLOCK)
        sub = [np.ascontiguousarray(inp[k][:, :, c0:c1]) for k in ("x1", "x2", "x3")]
        ref_y, ref_S = oracle.modal_recurrence(*sub, inp["log_poles"][c0:c1], inp["residues"][c0:c1],
                                               inp["Dskip"][c0:c1])
        cmp.add(from_dev_bf16(y[:, :, c0:c1]), ref_y, c0)
        s_err += float(np.sum((S_host[:, c0:c1] - ref_S) ** 2))
        s_ref += float(np.sum(ref_S ** 2))
    cmp.check(what, per_channel=per_channel)
    assert np.sqrt(s_err / s_ref) < 1e-4, f"{what}: state rel-L2 {np.sqrt(s_err / s_ref):.3e}"


def test_modal_32k_full_tensor():
    import torch
    inp = make_workload_inputs("modal_32k")
    dev = Dev(inp)
    y, S = modal_run(dev, inp)
    ref_y, ref_S = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                           inp["residues"], inp["Dskip"])
    assert_close(from_dev_bf16(y), ref_y, "modal 32K")
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
    assert rel < 1e-4
    del y
    torch.cuda.empty_cache()


def test_modal_131k_chunked_prefill():
    import torch
    inp = make_workload_inputs("modal_131k_chunked")
    dev = Dev(inp)
    y1, S1 = modal_run(dev, inp)
    yc, Sc = modal_run(dev, inp, chunk=WORKLOAD_SHAPES["modal_131k_chunked"]["chunk"])
    # 1024-token chunks are whole 128-token units: bitwise equal to the single
    # pass over the whole tensor
    assert torch.equal(yc.view(torch.int16), y1.view(torch.int16))
    assert torch.equal(Sc, S1)
    del y1
    torch.cuda.empty_cache()
    streamed_oracle_check(yc, Sc, inp, "modal 131K in 1024-token chunks")


def test_modal_262k_long_context_wide_range():
    import torch
    inp = make_workload_inputs("modal_262k_wide")
    dev = Dev(inp)
    y1, S1 = modal_run(dev, inp)
    yc, Sc = modal_run(dev, inp, chunk=1024)
    # the 1024-chunked feed equals the single pass bit for bit, whole tensor
    assert torch.equal(yc.view(torch.int16), y1.view(torch.int16))
    assert torch.equal(Sc, S1)
    del yc
    torch.cuda.empty_cache()
    streamed_oracle_check(y1, S1, inp, "modal 262K single pass (and 1024-chunked)", per_channel=True)
