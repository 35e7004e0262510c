"""Failure detection of the modal scan's device-side waits, without a GPU
fault: the test takes group 0's ticket away before the launch (a flag that
nothing will set), so the look-back of group 1 waits for a predecessor that
never runs.  That wait gives up after its bounded time (about one second of
%globaltimer), records an error bit, every other wait gives up on seeing it,
the launch ends normally, and ``workspace_check`` reports HYENA_ERR_TIMEOUT.
The same workspace then serves a correct call.
"""
import numpy as np
import pytest

import oracle
from synth import make_modal_inputs

from .helpers import assert_close, from_dev_bf16, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # HYENA_ERR_TIMEOUT


def test_lookback_wait_runs_out_and_is_reported():
    import torch
    import hyena_long_convolution_b200 as hy
    B, L, D, N = 1, 4096, 64, 8  # one chain of 32 units: 8 four-unit groups
    inp = make_modal_inputs(B, L, D, N, seed=77)
    x = [to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3")]
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    ws = hy.ModalWorkspace(B, D, N)
    # header word 0 is the next ticket: start at 1, so group 0 is never run
    ws.buf[0] = 1
    hy.modal_long_conv(*x, a, R, Ds, workspace=ws)
    with pytest.raises(hy.HyenaError) as err:
        hy.workspace_check(ws)
    assert err.value.status == TIMEOUT
    # the launch reset its ticket and the check cleared the error: the same
    # workspace now gives a correct result
    y = hy.modal_long_conv(*x, a, R, Ds, workspace=ws)
    hy.workspace_check(ws)
    ref, _ = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"],
                                     inp["Dskip"])
    assert_close(from_dev_bf16(y), ref, "after recovery")
    assert np.isfinite(from_dev_bf16(y)).all()
