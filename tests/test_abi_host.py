"""The C-ABI library loads on a host without a GPU, exports every entry point
that include/hyena.h declares, and rejects bad arguments on the host before
touching the device (no compute call is made here).
"""
import ctypes
import os
import re

import pytest

import hyena_long_convolution_b200 as hy
from hyena_long_convolution_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hyena.h")

OK, INVALID, ALIGN, UNSUP, CUDA, TIMEOUT, WORKSPACE = range(7)
A = 0x10000  # a 16-byte-aligned fake device address; never dereferenced here


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hyena_[a-z0-9_]+)\s*\(", src)))


def test_header_and_binding_agree():
    names = declared_functions()
    assert names, "no declarations parsed"
    assert sorted(_lib.SIGNATURES) == names


def test_library_exports_every_declared_symbol():
    lib = hy.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings_and_version():
    lib = hy.lib()
    for code, name in _lib.STATUS.items():
        assert lib.hyena_status_string(code).decode() == name
    assert lib.hyena_status_string(99).decode() == "HYENA_ERR_UNKNOWN"
    assert lib.hyena_abi_version() == 100


def test_workspace_size():
    lib = hy.lib()
    assert lib.hyena_modal_long_conv_workspace_size(0, 64, 8) == 0
    assert lib.hyena_modal_long_conv_workspace_size(1, 64, 0) == 0
    assert lib.hyena_modal_long_conv_workspace_size(1, 64, hy.MAX_MODES + 1) == 0
    a = lib.hyena_modal_long_conv_workspace_size(1, 4096, 16)
    b = lib.hyena_modal_long_conv_workspace_size(2, 4096, 16)
    c = lib.hyena_modal_long_conv_workspace_size(1, 4096, 8)
    assert 0 < c < a < b
    assert a % 256 == 0
    # independent of the sequence length by construction: no L argument
    assert a < 64 << 20


def modal(lib, **kw):
    args = dict(x1=A, x2=A, x3=A, ld_x=64, lp=A, res=A, ds=None, y=A + 4096, ld_y=64,
                s_in=None, s_out=None, B=1, L=16, D=64, N=8, ws=None, ws_bytes=0, st=None)
    args.update(kw)
    return lib.hyena_modal_long_conv(args["x1"], args["x2"], args["x3"], args["ld_x"], args["lp"],
                                     args["res"], args["ds"], args["y"], args["ld_y"], args["s_in"],
                                     args["s_out"], args["B"], args["L"], args["D"], args["N"],
                                     args["ws"], args["ws_bytes"], args["st"])


def fir(lib, entry="hyena_short_conv", **kw):
    args = dict(x1=A, x2=A, x3=A, ld_x=64, taps=A, ds=None, y=A + 4096, ld_y=64, h_in=None,
                h_out=None, B=1, L=16, D=64, K=7, st=None)
    args.update(kw)
    return getattr(lib, entry)(args["x1"], args["x2"], args["x3"], args["ld_x"], args["taps"],
                               args["ds"], args["y"], args["ld_y"], args["h_in"], args["h_out"],
                               args["B"], args["L"], args["D"], args["K"], args["st"])


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), INVALID), (dict(L=-1), INVALID), (dict(D=0), INVALID),
    (dict(x1=None), INVALID), (dict(y=None), INVALID), (dict(lp=None), INVALID),
    (dict(res=None), INVALID), (dict(N=0), INVALID), (dict(N=65), UNSUP),
    (dict(ld_x=32), INVALID), (dict(ld_y=60), INVALID), (dict(D=60, ld_x=64, ld_y=64), ALIGN),
    (dict(ld_x=68), ALIGN), (dict(x2=A + 2), ALIGN), (dict(y=A + 8), ALIGN),
    (dict(s_in=A + 4), ALIGN), (dict(ds=A + 4), ALIGN),
    (dict(ws=None), WORKSPACE), (dict(ws=A, ws_bytes=1024), WORKSPACE),
])
def test_modal_rejects_bad_arguments(kw, code):
    assert modal(hy.lib(), **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), INVALID), (dict(L=-5), INVALID), (dict(x3=None), INVALID), (dict(taps=None), INVALID),
    (dict(K=0), INVALID), (dict(K=129), UNSUP), (dict(ld_x=8), INVALID), (dict(x1=A + 6), ALIGN),
    (dict(taps=A + 2), ALIGN), (dict(h_in=A + 4), ALIGN), (dict(D=12, ld_x=16, ld_y=16), ALIGN),
])
@pytest.mark.parametrize("entry", ["hyena_short_conv", "hyena_short_conv_dft"])
def test_short_conv_rejects_bad_arguments(kw, code, entry):
    # the tensor-core FIR takes the same arguments and refuses the same ones
    assert fir(hy.lib(), entry, **kw) == code


def mdec(lib, x1=A, x2=A, x3=A, ld_x=64, a=A, R=A, Ds=None, y=A, ld_y=64, state=A, B=1, D=64, N=8):
    return lib.hyena_modal_decode(x1, x2, x3, ld_x, a, R, Ds, y, ld_y, state, B, D, N, None)


def fdec(lib, x1=A, x2=A, x3=A, ld_x=64, taps=A, Ds=None, y=A, ld_y=64, hist=A, B=1, D=64, K=7):
    return lib.hyena_short_decode(x1, x2, x3, ld_x, taps, Ds, y, ld_y, hist, B, D, K, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), INVALID), (dict(state=None), INVALID), (dict(a=None), INVALID), (dict(R=None), INVALID),
    (dict(y=None), INVALID), (dict(N=0), INVALID), (dict(N=65), UNSUP), (dict(ld_x=32), INVALID),
    (dict(state=A + 4), ALIGN), (dict(x2=A + 2), ALIGN), (dict(Ds=A + 8), ALIGN), (dict(D=12, ld_x=16, ld_y=16), ALIGN),
])
def test_modal_decode_rejects_bad_arguments(kw, code):
    assert mdec(hy.lib(), **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), INVALID), (dict(taps=None), INVALID), (dict(hist=None), INVALID), (dict(K=0), INVALID),
    (dict(K=129), UNSUP), (dict(hist=A + 4), ALIGN), (dict(taps=A + 2), ALIGN), (dict(ld_y=16), INVALID),
])
def test_short_decode_rejects_bad_arguments(kw, code):
    assert fdec(hy.lib(), **kw) == code


def packed_calls(lib, xp=A, ld_x=192, group=1, y=A + 65536, ld_y=64, B=1, L=16, D=64):
    """Status of each packed entry point for one projection-buffer description
    (every other argument valid)."""
    return {
        "modal": lib.hyena_modal_long_conv_packed(xp, ld_x, group, A, A, None, y, ld_y, None, None,
                                                  B, L, D, 8, None, 0, None),
        "fir": lib.hyena_short_conv_packed(xp, ld_x, group, A, None, y, ld_y, None, None, B, L, D, 7, None),
        "mdec": lib.hyena_modal_decode_packed(xp, ld_x, group, A, A, None, y, ld_y, A, B, D, 8, None),
        "fdec": lib.hyena_short_decode_packed(xp, ld_x, group, A, None, y, ld_y, A, B, D, 7, None),
        "cmodal": lib.hyena_modal_long_conv_complex_packed(xp, ld_x, group, A, A, None, y, ld_y, None, None,
                                                           B, L, D, 4, None, 0, None),
        "cdec": lib.hyena_modal_decode_complex_packed(xp, ld_x, group, A, A, None, y, ld_y, A, B, D, 4, None),
    }


@pytest.mark.parametrize("kw,code", [
    (dict(group=0), INVALID), (dict(group=-8), INVALID), (dict(group=7), INVALID),  # 64 % 7 != 0
    (dict(D=48, ld_x=144, ld_y=48, group=12), UNSUP),   # not a multiple of 8
    (dict(D=48, ld_x=144, ld_y=48, group=24), UNSUP),   # neither divides 64 nor is a multiple of 64
    (dict(D=192, ld_x=576, ld_y=192, group=96), UNSUP),
    (dict(ld_x=184), INVALID), (dict(xp=None), INVALID), (dict(y=None), INVALID), (dict(B=0), INVALID),
    (dict(xp=A + 2), ALIGN), (dict(ld_x=196), ALIGN), (dict(D=60, ld_x=180, ld_y=64, group=1), ALIGN),
])
def test_packed_entry_points_reject_bad_arguments(kw, code):
    res = packed_calls(hy.lib(), **kw)
    assert set(res.values()) == {code}, res


def test_packed_entry_points_check_their_own_arguments():
    """A valid buffer description with an invalid filter argument fails the
    same way as the plain entry point."""
    lib = hy.lib()
    assert lib.hyena_modal_long_conv_packed(A, 192, 1, A, A, None, A + 65536, 64, None, None,
                                            1, 16, 64, hy.MAX_MODES + 1, None, 0, None) == UNSUP
    assert lib.hyena_modal_long_conv_packed(A, 192, 64, A, A, None, A + 65536, 64, None, None,
                                            1, 16, 64, 8, None, 0, None) == WORKSPACE
    assert lib.hyena_short_conv_packed(A, 192, 8, A, None, A + 65536, 64, None, None, 1, 16, 64, 129, None) == UNSUP
    assert lib.hyena_modal_decode_packed(A, 192, 16, A, A, None, A + 65536, 64, None, 1, 64, 8, None) == INVALID
    assert lib.hyena_short_decode_packed(A, 192, 32, A, None, A + 65536, 64, None, 1, 64, 7, None) == INVALID


def test_complex_entry_points_reject_bad_arguments():
    lib = hy.lib()

    def conv(**kw):
        a = dict(x1=A, x2=A, x3=A, ld_x=64, p=A, r=A, ds=None, y=A + 4096, ld_y=64, s_in=None, s_out=None,
                 B=1, L=16, D=64, N=4, ws=None, ws_bytes=0)
        a.update(kw)
        return lib.hyena_modal_long_conv_complex(a["x1"], a["x2"], a["x3"], a["ld_x"], a["p"], a["r"], a["ds"],
                                                 a["y"], a["ld_y"], a["s_in"], a["s_out"], a["B"], a["L"],
                                                 a["D"], a["N"], a["ws"], a["ws_bytes"], None)

    def dec(**kw):
        a = dict(x1=A, x2=A, x3=A, ld_x=64, p=A, r=A, ds=None, y=A + 4096, ld_y=64, s=A, B=1, D=64, N=4)
        a.update(kw)
        return lib.hyena_modal_decode_complex(a["x1"], a["x2"], a["x3"], a["ld_x"], a["p"], a["r"], a["ds"],
                                              a["y"], a["ld_y"], a["s"], a["B"], a["D"], a["N"], None)

    assert conv(N=0) == INVALID
    assert conv(N=hy.MAX_COMPLEX_MODES + 1) == UNSUP
    assert conv(p=None) == INVALID
    assert conv(r=A + 4) == ALIGN
    assert conv() == WORKSPACE
    assert conv(ws=A, ws_bytes=lib.hyena_modal_long_conv_workspace_size(1, 64, 4)) == WORKSPACE  # needs 2N slots
    assert dec(N=0) == INVALID
    assert dec(N=hy.MAX_COMPLEX_MODES + 1) == UNSUP
    assert dec(s=None) == INVALID
    assert dec(s=A + 8) == ALIGN
    assert dec(ld_x=32) == INVALID


def test_other_entry_points_reject_bad_arguments():
    lib = hy.lib()
    assert lib.hyena_modal_state_init(None, 1, 64, 8, None) == INVALID
    assert lib.hyena_modal_state_init(A, 0, 64, 8, None) == INVALID
    assert lib.hyena_modal_workspace_init(None, 100, None) == INVALID
    assert lib.hyena_modal_workspace_init(A, 0, None) == INVALID
    assert lib.hyena_workspace_check(None, None) == INVALID


def test_host_buffer_entry_point_sizes_and_bad_arguments():
    lib = hy.lib()
    ws = lib.hyena_modal_host_workspace_size
    assert ws(1, 4096, 16, 100) == 0  # not a multiple of 128
    assert ws(1, 4096, 16, 0) == 0
    assert ws(1, 4096, 16, 2048) > 0
    assert ws(1, 4096, hy.MAX_MODES + 1, 2048) == 0
    # two staging slots of x1, x2, x3, y (8 bytes per channel-token each) on
    # top of the scan's workspace and the carried state
    extra = ws(1, 4096, 16, 2048) - lib.hyena_modal_long_conv_workspace_size(1, 4096, 16)
    assert extra >= 2 * 2048 * 4096 * 8 + 4096 * 16 * 4

    def conv(x=A, L=256, D=64, N=8, chunk=128, w=A, wb=1 << 30, ld_x=None, ld_y=None):
        return lib.hyena_modal_long_conv_host(x, x, x, ld_x or D, A, A, None, x, ld_y or D, None, None,
                                              1, L, D, N, chunk, w, wb, None)
    assert conv(chunk=100) == INVALID
    assert conv(chunk=0) == INVALID
    assert conv(x=None) == INVALID
    assert conv(N=0) == INVALID
    assert conv(N=hy.MAX_MODES + 1) == UNSUP
    assert conv(ld_x=32) == INVALID
    assert conv(D=60) == ALIGN
    assert conv(w=None) == WORKSPACE
    assert conv(wb=1024) == WORKSPACE
    assert conv(w=A + 16) == ALIGN


def test_prepared_entry_points_reject_bad_arguments():
    lib = hy.lib()
    big = 1 << 30

    def prep(a=A, r=A, D=64, N=8, w=A, wb=big):
        return lib.hyena_modal_prepare(a, r, None, 1, D, N, w, wb, None)
    assert prep(a=None) == INVALID
    assert prep(r=None) == INVALID
    assert prep(N=0) == INVALID
    assert prep(N=hy.MAX_MODES + 1) == UNSUP
    assert prep(D=60) == ALIGN
    assert prep(a=A + 4) == ALIGN
    assert prep(w=None) == WORKSPACE
    assert prep(wb=64) == WORKSPACE

    def conv(x=A, L=256, N=8, w=A, wb=big):
        return lib.hyena_modal_long_conv_prepared(x, x, x, 64, x, 64, None, None, 1, L, 64, N, w, wb, None)
    assert conv(x=None) == INVALID
    assert conv(N=0) == INVALID
    assert conv(N=hy.MAX_MODES + 1) == UNSUP
    assert conv(w=None) == WORKSPACE
    assert conv(wb=64) == WORKSPACE


def test_short_host_buffer_entry_point_sizes_and_bad_arguments():
    lib = hy.lib()
    ws = lib.hyena_short_host_workspace_size
    assert ws(1, 4096, 128, 0) == 0
    assert ws(1, 4096, 129, 2048) == 0
    assert ws(2, 4096, 128, 2048) >= 2 * 4 * 2 * 2048 * 4096 * 2 + 2 * 127 * 4096 * 4

    def conv(x=A, L=256, D=64, K=7, chunk=128, w=A, wb=1 << 30, ld_x=None):
        return lib.hyena_short_conv_host(x, x, x, ld_x or D, A, None, x, D, None, None, 1, L, D, K, chunk, w, wb, None)
    assert conv(chunk=0) == INVALID
    assert conv(x=None) == INVALID
    assert conv(K=0) == INVALID
    assert conv(K=129) == UNSUP
    assert conv(ld_x=32) == INVALID
    assert conv(D=60) == ALIGN
    assert conv(w=None) == WORKSPACE
    assert conv(wb=1024) == WORKSPACE
    assert conv(w=A + 16) == ALIGN


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "SO", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.lib()
