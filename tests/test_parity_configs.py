"""Parity at the five acceptance workloads' full sizes, in the launch
configuration the benchmark times.

The 1K- and 32K-token modal workloads (and both FIR workloads, in their own
files) are compared element by element with the fp64 oracle over the whole
output tensor.  For the 131K- and 262K-token workloads the
oracle runs on a sample of channels (every position of those channels), and
the whole tensor is checked through properties that hold at any size:
chunked feeding in whole 128-token units reproduces the single pass bit for
bit, and all outputs are finite.
"""
import numpy as np
import pytest

import oracle
from synth import WORKLOAD_SHAPES, make_workload_inputs

from .helpers import assert_close, bits_of, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def sample_channels(D, k=40, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 62, 63, 64, D // 2, D - 2, D - 1]
    return np.unique(np.concatenate([fixed, rng.choice(D, size=k, replace=False)]))


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


def sampled_oracle(inp, chans):
    sub = {k: np.ascontiguousarray(inp[k][:, :, chans]) for k in ("x1", "x2", "x3")}
    return oracle.modal_recurrence(sub["x1"], sub["x2"], sub["x3"], inp["log_poles"][chans],
                                   inp["residues"][chans], inp["Dskip"][chans])


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
    # 1024-token chunks are whole 128-token units: bitwise equal to the single pass
    assert torch.equal(yc.view(torch.int16), y1.view(torch.int16))
    assert torch.equal(Sc, S1)
    chans = sample_channels(inp["D"], seed=3)
    ref_y, ref_S = sampled_oracle(inp, chans)
    idx = torch.from_numpy(chans).cuda()
    assert_close(from_dev_bf16(yc.index_select(2, idx)), ref_y, "modal 131K in 1024-token chunks (sampled channels)")
    rel, _ = metrics(Sc[:, chans].cpu().numpy().astype(np.float64), ref_S)
    assert rel < 1e-4


def test_modal_262k_long_context_wide_range():
    import torch
    inp = make_workload_inputs("modal_262k_wide")
    dev = Dev(inp)
    y1, S1 = modal_run(dev, inp)
    assert bool(torch.isfinite(y1.float()).all())
    chans = sample_channels(inp["D"], seed=4)
    ref_y, ref_S = sampled_oracle(inp, chans)
    idx = torch.from_numpy(chans).cuda()
    assert_close(from_dev_bf16(y1.index_select(2, idx)), ref_y, "modal 262K single pass", per_channel=True)
    rel, _ = metrics(S1[:, chans].cpu().numpy().astype(np.float64), ref_S)
    assert rel < 1e-4
    y1_bits = bits_of(y1.index_select(2, idx))
    del y1
    torch.cuda.empty_cache()
    yc, Sc = modal_run(dev, inp, chunk=1024)
    assert np.array_equal(bits_of(yc.index_select(2, idx)), y1_bits)
    assert torch.equal(Sc, S1)
