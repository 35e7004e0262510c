"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: closed forms
(impulse and step responses, state decay), scipy's textbook IIR/FIR routine
``scipy.signal.lfilter``, a pure-Python brute force, hand-derived golden
fixtures, and invariants the operator must satisfy (chunking, linearity,
causality, gate placement).  Together they are chosen so that a dropped term,
a wrong sign, an off-by-one in a power or a lag, a transposed operand or a
misplaced gate fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
from scipy.signal import lfilter, lfiltic

import oracle
from oracle import brute
from synth import bf16_bits_to_f32, f32_to_bf16_bits, make_fir_inputs, make_modal_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def ones_bits(shape):
    return bits(np.ones(shape, np.float32))


def rel_l2(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def small_modal(B=2, L=96, D=12, N=5, seed=11, with_state=True):
    inp = make_modal_inputs(B, L, D, N, seed, threads=1)
    S = None
    if with_state:
        S = np.random.default_rng(seed + 1).standard_normal((B, D, N))
    return inp, S


# ---------------------------------------------------------------- modal form


def test_direct_equals_recurrence_modal_1k_shape():
    # Two independently coded forms of the same filter (O(L^2) convolution with
    # the synthesised h, versus one recurrence per mode).
    inp = make_modal_inputs(1, 1024, 64, 8, 0, threads=1)
    S = np.random.default_rng(5).standard_normal((1, 64, 8))
    args = (inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"], inp["Dskip"])
    yd, sd = oracle.modal_direct(*args, state_in=S)
    yr, sr = oracle.modal_recurrence(*args, state_in=S)
    assert rel_l2(yr, yd) < 1e-12
    assert rel_l2(sr, sd) < 1e-12


def test_impulse_response_closed_form():
    # x1 = x3 = 1, x2 = delta at t=0, Dskip = 0: y[t] = h[t] = sum_n R_n e^{a_n t}.
    L, D = 200, 3
    a = np.array([[-0.05], [-0.7], [-1e-3]], np.float32)
    R = np.array([[1.5], [-0.25], [2.0]], np.float32)
    x2 = np.zeros((1, L, D), np.float32)
    x2[0, 0, :] = 1.0
    y, s = oracle.modal_recurrence(ones_bits((1, L, D)), bits(x2), ones_bits((1, L, D)), a, R)
    t = np.arange(L)
    for c in range(D):
        ref = float(R[c, 0]) * np.exp(float(a[c, 0]) * t)
        np.testing.assert_allclose(y[0, :, c], ref, rtol=1e-13, atol=0)
        # state after L tokens of an impulse at t=0 is e^{a (L-1)}
        assert math.isclose(s[0, c, 0], math.exp(float(a[c, 0]) * (L - 1)), rel_tol=1e-13)


def test_impulse_superposition_of_modes():
    L, D, N = 64, 2, 4
    a = -np.exp(np.random.default_rng(0).uniform(-6, 0, (D, N))).astype(np.float32)
    R = np.random.default_rng(1).standard_normal((D, N)).astype(np.float32)
    x2 = np.zeros((1, L, D), np.float32)
    x2[0, 0, :] = 1.0
    y, _ = oracle.modal_recurrence(ones_bits((1, L, D)), bits(x2), ones_bits((1, L, D)), a, R)
    t = np.arange(L)
    for c in range(D):
        ref = sum(float(R[c, n]) * np.exp(float(a[c, n]) * t) for n in range(N))
        np.testing.assert_allclose(y[0, :, c], ref, rtol=1e-12, atol=1e-15)


def test_step_response_geometric_sum():
    # v = 1: conv[t] = sum_n R_n (1 - p_n^{t+1}) / (1 - p_n).
    L, D, N = 300, 3, 3
    a = -np.exp(np.random.default_rng(2).uniform(math.log(1e-3), 0, (D, N))).astype(np.float32)
    R = np.random.default_rng(3).standard_normal((D, N)).astype(np.float32)
    y, _ = oracle.modal_recurrence(ones_bits((1, L, D)), ones_bits((1, L, D)),
                                   ones_bits((1, L, D)), a, R)
    t = np.arange(L)
    for c in range(D):
        p = np.exp(a[c].astype(np.float64))
        ref = sum(float(R[c, n]) * (1 - p[n] ** (t + 1)) / (1 - p[n]) for n in range(N))
        np.testing.assert_allclose(y[0, :, c], ref, rtol=1e-11)


def test_each_mode_matches_scipy_lfilter():
    # A single mode is the textbook first-order IIR s[t] = p s[t-1] + v[t];
    # scipy.signal.lfilter([1], [1, -p]) with initial conditions from lfiltic.
    inp, S = small_modal(B=1, L=257, D=4, N=3)
    v = bf16_bits_to_f32(inp["x1"]).astype(np.float64) * bf16_bits_to_f32(inp["x2"])
    x3 = bf16_bits_to_f32(inp["x3"]).astype(np.float64)
    y, s_out = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                       inp["residues"], inp["Dskip"], state_in=S)
    for c in range(4):
        conv = np.zeros(257)
        for n in range(3):
            p = math.exp(float(inp["log_poles"][c, n]))
            zi = lfiltic([1.0], [1.0, -p], y=[S[0, c, n]])
            sn, _ = lfilter([1.0], [1.0, -p], v[0, :, c], zi=zi)
            conv += float(inp["residues"][c, n]) * sn
            assert math.isclose(s_out[0, c, n], sn[-1], rel_tol=1e-12, abs_tol=1e-12)
        ref = x3[0, :, c] * conv + float(inp["Dskip"][c]) * v[0, :, c]
        np.testing.assert_allclose(y[0, :, c], ref, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("omega", [math.pi / 2, math.pi])
def test_steady_state_frequency_response(omega):
    # v[t] = cos(omega t) (exact in bf16 for omega = pi/2, pi), x3 = 1: once the
    # transients p^t have died out, conv[t] = Re(H(e^{j omega}) e^{j omega t})
    # with the transfer function H(z) = sum_n R_n / (1 - p_n z^-1).
    L, D, N = 600, 3, 4
    g = np.random.default_rng(8)
    a = np.log(g.uniform(0.05, 0.9, (D, N))).astype(np.float32)     # |p| <= 0.9: p^300 < 1e-13
    R = g.standard_normal((D, N)).astype(np.float32)
    t = np.arange(L)
    x1 = np.round(np.cos(omega * t)).astype(np.float32)[None, :, None].repeat(D, 2)  # exactly 1, 0, -1
    y, _ = oracle.modal_recurrence(bits(x1), ones_bits((1, L, D)), ones_bits((1, L, D)), a, R)
    for c in range(D):
        p = np.exp(a[c].astype(np.float64))
        H = np.sum(R[c].astype(np.float64) / (1.0 - p * np.exp(-1j * omega)))
        ref = np.real(H * np.exp(1j * omega * t))
        np.testing.assert_allclose(y[0, 300:, c], ref[300:], rtol=1e-10, atol=1e-10)


def test_skip_sits_outside_the_gate():
    # R = 0: y = Dskip * v, whatever x3 is (reading: the skip is not gated by x3).
    inp, S = small_modal()
    R0 = np.zeros_like(inp["residues"])
    y, _ = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], R0,
                                   inp["Dskip"], state_in=S)
    v = bf16_bits_to_f32(inp["x1"]).astype(np.float64) * bf16_bits_to_f32(inp["x2"])
    np.testing.assert_array_equal(y, inp["Dskip"][None, None, :].astype(np.float64) * v)


def test_state_out_closed_form():
    # Impulse at t0 only: state_out = e^{a (L-1-t0)} + e^{a L} S_in.
    L, D, N, t0 = 50, 2, 2, 7
    a = np.array([[-0.1, -0.9], [-0.01, -2.0]], np.float32)
    R = np.ones((D, N), np.float32)
    S = np.array([[[0.5, -1.0], [2.0, 3.0]]])
    x2 = np.zeros((1, L, D), np.float32)
    x2[0, t0] = 1.0
    _, s = oracle.modal_recurrence(ones_bits((1, L, D)), bits(x2), ones_bits((1, L, D)), a, R,
                                   state_in=S)
    for c in range(D):
        for n in range(N):
            ref = math.exp(float(a[c, n]) * (L - 1 - t0)) + math.exp(float(a[c, n]) * L) * S[0, c, n]
            assert math.isclose(s[0, c, n], ref, rel_tol=1e-12)


@pytest.mark.parametrize("chunks", [1, 64, 1024, [5, 0, 300, 1, 718]])
def test_chunked_equals_single_pass(chunks):
    # Fidelity independent of chunk size (turboquant-evo2-int4 card, §"Chunk
    # size"); every position of every chunk is compared (the same card's
    # correctness-fix section describes a chunked path that lost all but the
    # last position).
    inp = make_modal_inputs(2, 1024, 16, 8, 7, threads=1)
    S = np.random.default_rng(9).standard_normal((2, 16, 8))
    args = (inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"], inp["Dskip"])
    y1, s1 = oracle.modal_recurrence(*args, state_in=S)
    yc, sc = oracle.modal_chunked(*args, state_in=S, chunks=chunks)
    assert rel_l2(yc, y1) < 1e-12
    assert rel_l2(sc, s1) < 1e-12
    # the direct form, chunked, must agree as well (state enters via its decay)
    if chunks == 64:
        ys = []
        Sd = S
        for t0 in range(0, 1024, 64):
            sl = slice(t0, t0 + 64)
            y, Sd = oracle.modal_direct(inp["x1"][:, sl], inp["x2"][:, sl], inp["x3"][:, sl],
                                        inp["log_poles"], inp["residues"], inp["Dskip"], Sd)
            ys.append(y)
        assert rel_l2(np.concatenate(ys, 1), y1) < 1e-12


@pytest.mark.parametrize("L", [1, 2, 17, 64])
def test_brute_force_tiny(L):
    inp, S = small_modal(B=2, L=L, D=3, N=4, seed=20 + L)
    y, s = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                   inp["residues"], inp["Dskip"], state_in=S)
    x1 = bf16_bits_to_f32(inp["x1"]).astype(float)
    x2 = bf16_bits_to_f32(inp["x2"]).astype(float)
    x3 = bf16_bits_to_f32(inp["x3"]).astype(float)
    for b in range(2):
        for c in range(3):
            v = [x1[b, t, c] * x2[b, t, c] for t in range(L)]
            yb, sb = brute.modal_channel(v, list(x3[b, :, c]),
                                         [float(q) for q in inp["log_poles"][c]],
                                         [float(q) for q in inp["residues"][c]],
                                         float(inp["Dskip"][c]), list(S[b, c]))
            np.testing.assert_allclose(y[b, :, c], yb, rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(s[b, c], sb, rtol=1e-13, atol=1e-13)


def test_linearity_in_v_and_R():
    inp, _ = small_modal(B=1, L=128, D=6, N=4, with_state=False)
    x1, x2, x3 = inp["x1"], inp["x2"], inp["x3"]
    a, Ds = inp["log_poles"], inp["Dskip"]
    # linear in R (skip off): residues on a 2^-10 grid so R1 + R2 is exact in fp32
    g = np.random.default_rng(4)
    R1 = (np.round(g.uniform(-4, 4, (6, 4)) * 1024) / 1024).astype(np.float32)
    R2 = (np.round(g.uniform(-4, 4, (6, 4)) * 1024) / 1024).astype(np.float32)
    ya, _ = oracle.modal_recurrence(x1, x2, x3, a, R1)
    yb, _ = oracle.modal_recurrence(x1, x2, x3, a, R2)
    yab, _ = oracle.modal_recurrence(x1, x2, x3, a, R1 + R2)
    assert rel_l2(ya + yb, yab) < 1e-13
    # linear in v: scaling x2 by 2 (exact in bf16) doubles the output
    x2d = f32_to_bf16_bits(bf16_bits_to_f32(x2) * 2)
    y1, s1 = oracle.modal_recurrence(x1, x2, x3, a, inp["residues"], Ds)
    y2, s2 = oracle.modal_recurrence(x1, x2d, x3, a, inp["residues"], Ds)
    np.testing.assert_allclose(y2, 2 * y1, rtol=1e-14, atol=0)
    np.testing.assert_allclose(s2, 2 * s1, rtol=1e-14, atol=0)


def test_causality():
    inp, S = small_modal(B=1, L=200, D=4, N=4)
    args = [inp["x1"], inp["x2"].copy(), inp["x3"], inp["log_poles"], inp["residues"], inp["Dskip"]]
    y0, _ = oracle.modal_recurrence(*args, state_in=S)
    args[1][0, 120, :] = bits(np.full(4, 7.0))
    y1, _ = oracle.modal_recurrence(*args, state_in=S)
    np.testing.assert_array_equal(y0[:, :120], y1[:, :120])
    assert np.all(y0[:, 120] != y1[:, 120])


def test_row_stride_and_batch_rows():
    # x given with a row stride ld = 3D (e.g. views of a [B, L, 3D] projection
    # output) gives the same result as contiguous [B, L, D]; batch rows are
    # independent.
    inp, S = small_modal(B=3, L=40, D=8, N=3)
    junk = f32_to_bf16_bits(np.random.default_rng(0).standard_normal((3, 40, 16)).astype(np.float32))
    wide = [np.concatenate([inp[k], junk], axis=2) for k in ("x1", "x2", "x3")]
    y_ref, s_ref = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                           inp["residues"], inp["Dskip"], state_in=S)
    y_w, s_w = oracle.modal_recurrence(*wide, inp["log_poles"], inp["residues"], inp["Dskip"],
                                       state_in=S)
    np.testing.assert_array_equal(y_w, y_ref)
    np.testing.assert_array_equal(s_w, s_ref)
    for b in range(3):
        yb, sb = oracle.modal_recurrence(inp["x1"][b:b + 1], inp["x2"][b:b + 1], inp["x3"][b:b + 1],
                                         inp["log_poles"], inp["residues"], inp["Dskip"],
                                         state_in=S[b:b + 1])
        np.testing.assert_array_equal(yb[0], y_ref[b])
        np.testing.assert_array_equal(sb[0], s_ref[b])


def test_zero_length_passes_state_through():
    inp, S = small_modal(B=1, L=0, D=4, N=2)
    y, s = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                   inp["residues"], inp["Dskip"], state_in=S)
    assert y.shape == (1, 0, 4)
    np.testing.assert_array_equal(s, S)
    _, s0 = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                    inp["residues"], inp["Dskip"])
    np.testing.assert_array_equal(s0, 0)


# ---------------------------------------------------------------- explicit FIR


def test_fir_matches_scipy_lfilter():
    inp = make_fir_inputs(2, 300, 5, 7, 3, with_skip=True, threads=1)
    H = np.random.default_rng(8).standard_normal((2, 6, 5))
    y, h_out = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"], H)
    v = bf16_bits_to_f32(inp["x1"]).astype(np.float64) * bf16_bits_to_f32(inp["x2"])
    x3 = bf16_bits_to_f32(inp["x3"]).astype(np.float64)
    taps = bf16_bits_to_f32(inp["taps"]).astype(np.float64)
    for b in range(2):
        for c in range(5):
            full = np.concatenate([H[b, :, c], v[b, :, c]])
            conv = lfilter(taps[c], [1.0], full)[6:]
            ref = x3[b, :, c] * conv + float(inp["Dskip"][c]) * v[b, :, c]
            np.testing.assert_allclose(y[b, :, c], ref, rtol=1e-12, atol=1e-12)
            np.testing.assert_array_equal(h_out[b, :, c], full[-6:])


def test_fir_delta_tap_is_exact_shift():
    inp = make_fir_inputs(1, 64, 4, 5, 4, threads=1)
    taps = np.zeros((4, 5), np.float32)
    taps[:, 3] = 1.0
    y, _ = oracle.fir(inp["x1"], inp["x2"], inp["x3"], bits(taps))
    v = bf16_bits_to_f32(inp["x1"]).astype(np.float64) * bf16_bits_to_f32(inp["x2"])
    x3 = bf16_bits_to_f32(inp["x3"]).astype(np.float64)
    np.testing.assert_array_equal(y[:, :3], 0)
    np.testing.assert_array_equal(y[:, 3:], x3[:, 3:] * v[:, :-3])


def test_fir_single_tap_pointwise():
    inp = make_fir_inputs(1, 33, 4, 1, 5, with_skip=True, threads=1)
    y, h = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"])
    v = bf16_bits_to_f32(inp["x1"]).astype(np.float64) * bf16_bits_to_f32(inp["x2"])
    x3 = bf16_bits_to_f32(inp["x3"]).astype(np.float64)
    tap = bf16_bits_to_f32(inp["taps"][:, 0]).astype(np.float64)
    np.testing.assert_allclose(y, x3 * tap * v + inp["Dskip"].astype(np.float64) * v, rtol=1e-15)
    assert h.shape == (1, 0, 4)


def test_fir_with_modal_taps_equals_modal_when_short():
    # For L <= K a FIR whose taps are the modal filter's first K values is the
    # modal conv itself; taps must be exact in bf16, so pick p = 1/2 powers.
    L = K = 16
    D = 2
    a = np.full((D, 1), math.log(0.5), np.float32)
    R = np.array([[1.0], [-3.0]], np.float32)
    inp = make_modal_inputs(1, L, D, 1, 6, threads=1)
    ym, _ = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], a, R)
    taps = np.stack([float(R[c, 0]) * 0.5 ** np.arange(K) for c in range(D)]).astype(np.float32)
    yf, _ = oracle.fir(inp["x1"], inp["x2"], inp["x3"], bits(taps))
    np.testing.assert_allclose(yf, ym, rtol=1e-7, atol=1e-9)  # fp32 rounding of ln 0.5


@pytest.mark.parametrize("chunks", [1, 5, 64, [3, 0, 100, 1, 152]])
def test_fir_chunked_equals_single_pass(chunks):
    inp = make_fir_inputs(2, 256, 6, 9, 6, with_skip=True, threads=1)
    H = np.random.default_rng(3).standard_normal((2, 8, 6))
    args = (inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"])
    y1, h1 = oracle.fir(*args, H)
    yc, hc = oracle.fir_chunked(*args, H, chunks=chunks)
    np.testing.assert_array_equal(yc, y1)
    np.testing.assert_array_equal(hc, h1)


def test_fir_brute_force_tiny():
    inp = make_fir_inputs(1, 20, 3, 6, 9, with_skip=True, threads=1)
    H = np.random.default_rng(1).standard_normal((1, 5, 3))
    y, h = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], inp["Dskip"], H)
    x1 = bf16_bits_to_f32(inp["x1"]).astype(float)
    x2 = bf16_bits_to_f32(inp["x2"]).astype(float)
    x3 = bf16_bits_to_f32(inp["x3"]).astype(float)
    taps = bf16_bits_to_f32(inp["taps"]).astype(float)
    for c in range(3):
        v = list(x1[0, :, c] * x2[0, :, c])
        yb, hb = brute.fir_channel(v, list(x3[0, :, c]), list(taps[c]), float(inp["Dskip"][c]),
                                   list(H[0, :, c]))
        np.testing.assert_allclose(y[0, :, c], yb, rtol=1e-14, atol=1e-14)
        np.testing.assert_allclose(h[0, :, c], hb, rtol=0, atol=0)


def test_fir_short_sequence_history_shift():
    # L < K-1: the new history is the old one shifted by L, then the new v.
    inp = make_fir_inputs(1, 3, 2, 8, 2, threads=1)
    H = np.arange(14, dtype=np.float64).reshape(1, 7, 2)
    _, h = oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], None, H)
    v = bf16_bits_to_f32(inp["x1"]).astype(np.float64) * bf16_bits_to_f32(inp["x2"])
    np.testing.assert_array_equal(h[0, :4], H[0, 3:])
    np.testing.assert_array_equal(h[0, 4:], v[0])


# ---------------------------------------------------------------- golden fixtures


def _load_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *rest = line.split()
            vals[k] = [float(r) for r in rest]
    return vals


@pytest.mark.parametrize("name", ["modal_prefix_sum.txt", "modal_half_pole.txt"])
def test_golden_modal(name):
    g = _load_golden(name)
    L, N = int(g["L"][0]), int(g["N"][0])
    sh = (1, L, 1)
    x = [bits(np.array(g[k], np.float32).reshape(sh)) for k in ("x1", "x2", "x3")]
    a = np.array(g["log_poles"], np.float32).reshape(1, N)
    R = np.array(g["residues"], np.float32).reshape(1, N)
    Ds = np.array(g["Dskip"], np.float32)
    S = np.array(g["state_in"]).reshape(1, 1, N) if "state_in" in g else None
    tol = g["tol"][0]
    for fn in (oracle.modal_recurrence, oracle.modal_direct):
        y, s = fn(*x, a, R, Ds, S)
        np.testing.assert_allclose(y.ravel(), g["y"], rtol=tol, atol=tol)
        np.testing.assert_allclose(s.ravel(), g["state_out"], rtol=tol, atol=tol)


def test_golden_fir():
    g = _load_golden("fir_history.txt")
    L, K = int(g["L"][0]), int(g["K"][0])
    sh = (1, L, 1)
    x = [bits(np.array(g[k], np.float32).reshape(sh)) for k in ("x1", "x2", "x3")]
    taps = bits(np.array(g["taps"], np.float32).reshape(1, K))
    H = np.array(g["hist_in"]).reshape(1, K - 1, 1)
    y, h = oracle.fir(*x, taps, np.array(g["Dskip"], np.float32), H)
    np.testing.assert_array_equal(y.ravel(), g["y"])
    np.testing.assert_array_equal(h.ravel(), g["hist_out"])


def test_inputs_are_deterministic_and_bf16():
    a = make_modal_inputs(1, 2048, 32, 4, 3, threads=4)
    b = make_modal_inputs(1, 2048, 32, 4, 3, threads=1)
    for k in ("x1", "x2", "x3", "log_poles", "residues", "Dskip"):
        np.testing.assert_array_equal(a[k], b[k])
    assert np.all(a["log_poles"] < 0) and np.all(a["log_poles"] >= -1.0)
    # rounding is to nearest even: 1 + 2^-8 (a tie) rounds down to 1
    assert f32_to_bf16_bits(np.array([1 + 2 ** -8], np.float32))[0] == 0x3F80
    assert f32_to_bf16_bits(np.array([1 + 3 * 2 ** -8], np.float32))[0] == 0x3F82


def test_oracle_refuses_sizes_it_cannot_hold():
    # The oracle keeps at most 256 modes and a 128-value FIR history per
    # channel; beyond that it must refuse the call, never leave outputs unwritten.
    x = np.zeros((1, 4, 8), np.uint16)
    a = np.full((8, 257), -0.5, np.float32)
    with pytest.raises(ValueError):
        oracle.modal_recurrence(x, x, x, a, np.ones_like(a))
    taps = np.zeros((8, 130), np.uint16)
    with pytest.raises(ValueError):
        oracle.fir(x, x, x, taps)
    # the largest supported sizes still run and fill every output
    y, S = oracle.modal_recurrence(x, x, x, a[:, :256], np.ones_like(a[:, :256]))
    assert np.all(np.isfinite(y)) and np.all(S == 0.0)
    y, H = oracle.fir(x, x, x, taps[:, :129])
    assert np.all(y == 0.0) and H.shape == (1, 128, 8) and np.all(H == 0.0)
