"""The allocation-free modal conv entry point (hyena_modal_long_conv_noalloc).

It serves callers that must not allocate device memory (for example a plugin
inside a framework that owns and accounts for all device memory, or code on a
latency-critical path where an allocation could synchronise the device): its
scratch is a fixed array the library owns instead of a caller-provided
workspace.  Called through the C ABI it runs the same deterministic kernel as
the workspace entry point, so y and the final state must be bit-identical to
it, on two calls in a row (the second call reuses the array the first one left
behind), and within tolerance of the fp64 oracle.  It must refuse sizes beyond
its fixed scratch, and a device-side wait that runs out must be reported by
hyena_modal_noalloc_check.

This file is collected last on purpose, and runs alone as well as after the
rest of the suite.
"""
import ctypes

import numpy as np
import pytest

import oracle
from synth import make_modal_inputs

from .helpers import assert_close, from_dev_bf16, metrics, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu

OK, TIMEOUT, WORKSPACE = 0, 5, 6


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


class Case:
    def __init__(self, B, L, D, N, seed):
        import torch
        self.B, self.L, self.D, self.N = B, L, D, N
        self.inp = make_modal_inputs(B, L, D, N, seed)
        self.x = [to_dev_bf16(self.inp[k]) for k in ("x1", "x2", "x3")]
        self.a, self.R, self.Ds = (to_dev_f32(self.inp[k]) for k in ("log_poles", "residues", "Dskip"))
        self.S0 = np.random.default_rng(seed).standard_normal((B, D, N)).astype(np.float32)
        self.S_in = torch.from_numpy(self.S0).cuda()

    def workspace_call(self):
        import torch
        import hyena_long_convolution_b200 as hy
        S = torch.empty_like(self.S_in)
        y = hy.modal_long_conv(*self.x, self.a, self.R, self.Ds, state_in=self.S_in, state_out=S)
        torch.cuda.synchronize()
        return y, S

    def noalloc_call(self):
        import torch
        import hyena_long_convolution_b200 as hy
        y = torch.empty((self.B, self.L, self.D), dtype=torch.bfloat16, device="cuda")
        S = torch.empty_like(self.S_in)
        x1, x2, x3 = self.x
        rc = hy.lib().hyena_modal_long_conv_noalloc(_p(x1), _p(x2), _p(x3), self.D, _p(self.a), _p(self.R),
                                                    _p(self.Ds), _p(y), self.D, _p(self.S_in), _p(S),
                                                    self.B, self.L, self.D, self.N, _stream())
        assert rc == OK, hy.lib().hyena_last_error_message().decode()
        torch.cuda.synchronize()
        return y, S


def _device_words(address, n):
    """A torch view of n 32-bit words of device memory at `address`."""
    import torch

    class _View:
        __cuda_array_interface__ = {"shape": (n,), "typestr": "<i4", "data": (address, False), "version": 3}

    return torch.as_tensor(_View(), device="cuda")


def _check():
    import hyena_long_convolution_b200 as hy
    return hy.lib().hyena_modal_noalloc_check(_stream())


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_is_bitwise_the_workspace_entry_point(call):
    import torch
    # two calls in a row with different shapes and data: the second call finds
    # the scratch array exactly as the first one left it
    case = Case(*[(1, 4096 + 37, 256, 16), (2, 1000, 136, 12)][call], seed=100 + call)
    y_ref, S_ref = case.workspace_call()
    y, S = case.noalloc_call()
    assert _check() == OK
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(S, S_ref)
    if call == 0:
        ref_y, ref_S = oracle.modal_recurrence(case.inp["x1"], case.inp["x2"], case.inp["x3"],
                                               case.inp["log_poles"], case.inp["residues"], case.inp["Dskip"],
                                               case.S0.astype(np.float64))
        assert_close(from_dev_bf16(y), ref_y, "allocation-free y against the oracle")
        rel, _ = metrics(S.cpu().numpy().astype(np.float64), ref_S)
        assert rel < 1e-4, rel


def test_noalloc_reports_a_wait_that_ran_out():
    import torch
    import hyena_long_convolution_b200 as hy
    lib = hy.lib()
    case = Case(1, 4096, 64, 8, seed=77)  # one chain of 32 units: several groups
    y_ref, S_ref = case.workspace_call()
    ptr, nbytes = ctypes.c_void_p(), ctypes.c_size_t()
    assert lib.hyena_modal_noalloc_scratch(ctypes.byref(ptr), ctypes.byref(nbytes)) == OK
    assert nbytes.value == 24 << 20
    assert _check() == OK
    # header word 0 is the next group ticket: start it at 1, so group 0 never
    # runs and the next group's look-back waits on a flag nothing sets; the
    # wait gives up after its bounded time and the launch ends normally
    torch.cuda.synchronize()
    _device_words(ptr.value, 1)[0] = 1
    torch.cuda.synchronize()
    case.noalloc_call()
    # a following call is unaffected, and the earlier failure is still reported
    y, S = case.noalloc_call()
    assert _check() == TIMEOUT
    assert _check() == OK  # the record was cleared
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(S, S_ref)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    import torch
    import hyena_long_convolution_b200 as hy
    lib = hy.lib()
    limit = 24 << 20
    B, D, N = 1, 64, 16
    while hy.workspace_size(B, D + 64, N) <= limit:
        D += 64
    assert hy.workspace_size(B, D, N) <= limit < hy.workspace_size(B, D + 64, N)
    x = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    rc = lib.hyena_modal_long_conv_noalloc(_p(x), _p(x), _p(x), D + 64, _p(x), _p(x), None, _p(x), D + 64,
                                           None, None, B, 16, D + 64, N, None)
    assert rc == WORKSPACE  # nothing launched
    assert b"limit" in lib.hyena_last_error_message()
