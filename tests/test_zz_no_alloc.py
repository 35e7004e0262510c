"""The allocation-free modal conv entry point (hyena_modal_long_conv_noalloc).

It serves callers that must not allocate device memory (for example a plugin
inside a framework that owns and accounts for all device memory): its scratch
is a fixed array the library owns instead of a caller-provided workspace.
Called through the C ABI, it must give the same result as the workspace
entry point, on two calls in a row (the second call reuses the array the
first one left behind), and must refuse sizes beyond its fixed scratch.

This file is collected last on purpose, and runs alone as well as after the
rest of the suite.
"""
import ctypes

import numpy as np
import pytest

from synth import make_modal_inputs

from .helpers import REL_L2_TOL, assert_close, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _run_both(B, L, D, N, seed):
    import torch
    import hyena_long_convolution_b200 as hy
    inp = make_modal_inputs(B, L, D, N, seed)
    x1, x2, x3 = (to_dev_bf16(inp[k]) for k in ("x1", "x2", "x3"))
    a, R, Ds = to_dev_f32(inp["log_poles"]), to_dev_f32(inp["residues"]), to_dev_f32(inp["Dskip"])
    S_in = torch.from_numpy(np.random.default_rng(seed).standard_normal((B, D, N)).astype(np.float32)).cuda()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    # existing entry point, caller-provided workspace
    S_ref = torch.empty_like(S_in)
    y_ref = hy.modal_long_conv(x1, x2, x3, a, R, Ds, state_in=S_in, state_out=S_ref)

    # allocation-free entry point, straight through the C ABI
    y = torch.empty_like(y_ref)
    S = torch.empty_like(S_in)
    rc = hy.lib().hyena_modal_long_conv_noalloc(_p(x1), _p(x2), _p(x3), D, _p(a), _p(R), _p(Ds), _p(y), D,
                                                _p(S_in), _p(S), B, L, D, N, stream)
    assert rc == 0, hy.lib().hyena_last_error_message().decode()
    torch.cuda.synchronize()
    return y_ref, S_ref, y, S


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_matches_workspace_entry_point(call):
    # two calls in a row with different shapes and data: the second call finds
    # the scratch array exactly as the first one left it
    shape = [(1, 4096 + 37, 256, 16), (2, 1000, 136, 12)][call]
    y_ref, S_ref, y, S = _run_both(*shape, seed=100 + call)
    assert_close(from_dev_bf16(y), from_dev_bf16(y_ref), "allocation-free y")
    rel, _ = metrics(S.cpu().numpy().astype(np.float64), S_ref.cpu().numpy().astype(np.float64))
    assert rel <= REL_L2_TOL, rel


def test_noalloc_refuses_sizes_beyond_its_scratch():
    import torch
    import hyena_long_convolution_b200 as hy
    lib = hy.lib()
    limit = 24 << 20
    assert hy.workspace_size(1, 4672, 16) <= limit < hy.workspace_size(1, 4736, 16)
    x = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    rc = lib.hyena_modal_long_conv_noalloc(_p(x), _p(x), _p(x), 4736, _p(x), _p(x), None, _p(x), 4736,
                                           None, None, 1, 16, 4736, 16, None)
    assert rc == 6  # HYENA_ERR_WORKSPACE, nothing launched
    assert b"limit" in lib.hyena_last_error_message()
