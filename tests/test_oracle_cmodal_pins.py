"""Pins for the complex-mode oracle (CPU only).

The complex modal filter h[k] = Re sum_n R_n p_n^k is checked against things
other than its own recurrence: the independent direct form (polar
coordinates, no complex arithmetic), the polar closed form of an impulse
response, scipy's textbook IIR routine ``scipy.signal.lfilter`` (one complex
mode is a real second-order section), the real-mode oracle when the poles are
real, the conjugate symmetry of the real part, the closed-form state, and
chunking.  A wrong sign of an imaginary part, a conjugated pole or residue, a
dropped cross term or an off-by-one power fails at least one of them.
"""
import cmath
import math
import os

import numpy as np
import pytest
from scipy.signal import lfilter

import oracle
from synth import bf16_bits_to_f32, f32_to_bf16_bits, make_cmodal_inputs


def bits(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def ones_bits(shape):
    return bits(np.ones(shape, np.float32))


def rel_l2(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def cx(pairs):
    """fp32 [..., 2] (re, im) -> complex128."""
    p = np.asarray(pairs, dtype=np.float64)
    return p[..., 0] + 1j * p[..., 1]


@pytest.mark.parametrize("B,L,D,N", [(1, 300, 8, 1), (2, 130, 12, 3), (1, 257, 6, 8)])
def test_direct_equals_recurrence(B, L, D, N):
    inp = make_cmodal_inputs(B, L, D, N, seed=L + N, threads=1)
    S = np.random.default_rng(N).standard_normal((B, D, N, 2))
    args = (inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"], inp["Dskip"])
    yd, sd = oracle.cmodal_direct(*args, state_in=S)
    yr, sr = oracle.cmodal_recurrence(*args, state_in=S)
    assert rel_l2(yr, yd) < 1e-12
    assert rel_l2(sr, sd) < 1e-12


def test_impulse_response_polar_closed_form():
    # x1 = x3 = 1, x2 = delta at t = 0, no skip: y[t] = |R| |p|^t cos(t arg p + arg R).
    L, D = 160, 3
    poles = np.array([[[0.9 * math.cos(0.3), 0.9 * math.sin(0.3)]],
                      [[-0.5, 0.6]],
                      [[0.999, -0.02]]], np.float32)
    res = np.array([[[1.2 * math.cos(-0.7), 1.2 * math.sin(-0.7)]], [[0.25, -1.5]], [[2.0, 0.0]]], np.float32)
    x2 = np.zeros((1, L, D), np.float32)
    x2[0, 0, :] = 1.0
    y, s = oracle.cmodal_recurrence(ones_bits((1, L, D)), bits(x2), ones_bits((1, L, D)), poles, res)
    t = np.arange(L)
    for c in range(D):
        p, R = complex(*map(float, poles[c, 0])), complex(*map(float, res[c, 0]))
        ref = abs(R) * abs(p) ** t * np.cos(t * cmath.phase(p) + cmath.phase(R))
        np.testing.assert_allclose(y[0, :, c], ref, rtol=1e-10, atol=1e-13)
        # state after an impulse at t = 0: p^(L-1)
        st = complex(s[0, c, 0, 0], s[0, c, 0, 1])
        assert cmath.isclose(st, p ** (L - 1), rel_tol=1e-11, abs_tol=1e-300)


def test_each_mode_is_a_second_order_section_scipy():
    # Re(R s_t) with s_t = p s_{t-1} + v_t is the real IIR
    #   b = [Re R, -Re(R conj p)],  a = [1, -2 Re p, |p|^2].
    inp = make_cmodal_inputs(1, 300, 4, 3, seed=9, threads=1)
    v = bf16_bits_to_f32(inp["x1"]).astype(np.float64) * bf16_bits_to_f32(inp["x2"])
    x3 = bf16_bits_to_f32(inp["x3"]).astype(np.float64)
    y, _ = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"], inp["Dskip"])
    P, R = cx(inp["poles"]), cx(inp["residues"])
    for c in range(4):
        conv = np.zeros(300)
        for n in range(3):
            p, r = P[c, n], R[c, n]
            b = [r.real, -(r * np.conj(p)).real]
            a = [1.0, -2.0 * p.real, abs(p) ** 2]
            conv += lfilter(b, a, v[0, :, c])
        ref = x3[0, :, c] * conv + float(inp["Dskip"][c]) * v[0, :, c]
        np.testing.assert_allclose(y[0, :, c], ref, rtol=1e-10, atol=1e-10)


def test_real_poles_reduce_to_the_real_modal_oracle():
    # Imaginary parts zero, real parts in (0, 1): the real-mode oracle with
    # log-poles a = log p gives the same filter (up to the fp32 rounding of a).
    B, L, D, N = 1, 200, 5, 4
    g = np.random.default_rng(4)
    p = g.uniform(0.2, 0.999, (D, N))
    R = g.standard_normal((D, N))
    poles = np.stack([p, np.zeros_like(p)], -1).astype(np.float32)
    res = np.stack([R, np.zeros_like(R)], -1).astype(np.float32)
    inp = make_cmodal_inputs(B, L, D, N, seed=1, threads=1)
    yc, sc = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], poles, res, inp["Dskip"])
    a = np.log(poles[..., 0].astype(np.float64)).astype(np.float32)
    yr, sr = oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], a, res[..., 0], inp["Dskip"])
    assert rel_l2(yc, yr) < 2e-5
    assert rel_l2(sc[..., 0], sr) < 2e-5
    assert np.all(sc[..., 1] == 0.0)


def test_conjugate_modes_give_the_same_real_filter():
    # Re(R p^k) = Re(conj R conj p^k): conjugating every pole and residue
    # leaves y unchanged and conjugates the state.
    inp = make_cmodal_inputs(2, 150, 6, 5, seed=3, threads=1)
    S = np.random.default_rng(2).standard_normal((2, 6, 5, 2))
    conj = np.array([1.0, -1.0], np.float32)
    y1, s1 = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"],
                                      inp["Dskip"], S)
    y2, s2 = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"] * conj,
                                      inp["residues"] * conj, inp["Dskip"], S * conj)
    assert rel_l2(y2, y1) < 1e-13
    assert rel_l2(s2, s1 * conj) < 1e-13


def test_state_out_closed_form():
    # Impulse at t0 only: state_out = p^(L-1-t0) + p^L S_in.
    L, D, t0 = 60, 2, 11
    poles = np.array([[[0.8, 0.5]], [[-0.3, -0.9]]], np.float32)
    res = np.ones((D, 1, 2), np.float32)
    S = np.array([[[[0.5, -1.0]], [[2.0, 3.0]]]])
    x2 = np.zeros((1, L, D), np.float32)
    x2[0, t0] = 1.0
    _, s = oracle.cmodal_recurrence(ones_bits((1, L, D)), bits(x2), ones_bits((1, L, D)), poles, res, state_in=S)
    for c in range(D):
        p = complex(*map(float, poles[c, 0]))
        ref = p ** (L - 1 - t0) + p ** L * complex(*S[0, c, 0])
        assert cmath.isclose(complex(*s[0, c, 0]), ref, rel_tol=1e-12)


@pytest.mark.parametrize("chunks", [1, 64, [5, 0, 300, 1, 206]])
def test_chunked_equals_single_pass(chunks):
    inp = make_cmodal_inputs(1, 512, 8, 4, seed=6, threads=1)
    S = np.random.default_rng(1).standard_normal((1, 8, 4, 2))
    args = (inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"], inp["Dskip"])
    y1, s1 = oracle.cmodal_recurrence(*args, state_in=S)
    y2, s2 = oracle.cmodal_chunked(*args, state_in=S, chunks=chunks)
    assert rel_l2(y2, y1) < 1e-12
    assert rel_l2(s2, s1) < 1e-12


def test_skip_sits_outside_the_gate():
    inp = make_cmodal_inputs(1, 64, 4, 2, seed=2, threads=1)
    y, _ = oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"],
                                    np.zeros_like(inp["residues"]), inp["Dskip"])
    v = bf16_bits_to_f32(inp["x1"]).astype(np.float64) * bf16_bits_to_f32(inp["x2"])
    np.testing.assert_array_equal(y, inp["Dskip"][None, None, :].astype(np.float64) * v)


def test_golden_quarter_turn():
    """Hand-derived fixture tests/golden/cmodal_quarter_turn.txt (derivation in
    its header): both oracle forms reproduce the exact dyadic values."""
    g = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "cmodal_quarter_turn.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, *vals = line.split()
                g[k] = [float(v) for v in vals]
    L, N = int(g["L"][0]), int(g["N"][0])
    sh = (1, L, 1)
    x = [bits(np.array(g[k], np.float32).reshape(sh)) for k in ("x1", "x2", "x3")]
    p = np.array(g["poles"], np.float32).reshape(1, N, 2)
    R = np.array(g["residues"], np.float32).reshape(1, N, 2)
    Ds = np.array(g["Dskip"], np.float32)
    S = np.array(g["state_in"]).reshape(1, 1, N, 2)
    tol = g["tol"][0]
    for fn in (oracle.cmodal_recurrence, oracle.cmodal_direct):
        y, s = fn(*x, p, R, Ds, S)
        np.testing.assert_allclose(y.ravel(), g["y"], rtol=tol, atol=tol)
        np.testing.assert_allclose(s.ravel(), g["state_out"], rtol=tol, atol=tol)


@pytest.mark.parametrize("omega", [math.pi / 2, math.pi])
def test_steady_state_frequency_response(omega):
    # h[k] = Re sum R p^k has the real transfer function
    # H(z) = 1/2 sum_n [R_n / (1 - p_n z^-1) + conj(R_n) / (1 - conj(p_n) z^-1)];
    # for v[t] = cos(omega t) the steady state is Re(H(e^{j omega}) e^{j omega t}).
    L, D, N = 600, 3, 3
    g = np.random.default_rng(9)
    rho = g.uniform(0.05, 0.9, (D, N))
    th = g.uniform(0.0, math.pi, (D, N))
    poles = np.stack([rho * np.cos(th), rho * np.sin(th)], -1).astype(np.float32)
    res = g.standard_normal((D, N, 2)).astype(np.float32)
    t = np.arange(L)
    x1 = np.round(np.cos(omega * t)).astype(np.float32)[None, :, None].repeat(D, 2)  # exactly 1, 0, -1
    y, _ = oracle.cmodal_recurrence(bits(x1), ones_bits((1, L, D)), ones_bits((1, L, D)), poles, res)
    z1 = np.exp(-1j * omega)
    for c in range(D):
        P, R = cx(poles[c]), cx(res[c])
        H = 0.5 * np.sum(R / (1.0 - P * z1) + np.conj(R) / (1.0 - np.conj(P) * z1))
        ref = np.real(H * np.exp(1j * omega * t))
        np.testing.assert_allclose(y[0, 300:, c], ref[300:], rtol=1e-10, atol=1e-10)
