"""Pure-Python brute force for tiny inputs -- TEST INFRASTRUCTURE.

Independent of hyena_oracle.c: plain Python floats (IEEE double), math.exp,
double loops over output and input positions.  Used only to pin the C oracle on
L <= 64.  Same operator and readings as the C oracle: the modal filter
h[k] = sum_n R_n exp(a_n k) (Evo2-7B-262K model card, §Implementation Notes),
a carried state that enters with decay exp(a_n (t+1)), explicit FIR in lag
order with a K-1 history (Evo2-7B-262K model card, "Block dispatch" and
"Custom cache"), y = x3 * conv + Dskip * v.
"""
from __future__ import annotations

import math


def modal_channel(v, x3, a, R, dskip=0.0, s_in=None):
    """One channel: v, x3 lists of floats; a, R lists of length N."""
    L = len(v)
    N = len(a)
    y = []
    for t in range(L):
        conv = 0.0
        for s in range(t + 1):
            h = 0.0
            for n in range(N):
                h += R[n] * math.exp(a[n] * (t - s))
            conv += h * v[s]
        if s_in is not None:
            for n in range(N):
                conv += R[n] * math.exp(a[n] * (t + 1)) * s_in[n]
        y.append(x3[t] * conv + dskip * v[t])
    s_out = []
    for n in range(N):
        acc = 0.0 if s_in is None else math.exp(a[n] * L) * s_in[n]
        for s in range(L):
            acc += math.exp(a[n] * (L - 1 - s)) * v[s]
        s_out.append(acc)
    return y, s_out


def fir_channel(v, x3, taps, dskip=0.0, hist=None):
    """One channel: taps in lag order; hist = the K-1 earlier values of v, oldest first."""
    K = len(taps)
    H = K - 1
    past = list(hist) if hist is not None else [0.0] * H
    full = past + list(v)  # full[H + t] = v[t]
    y = []
    for t in range(len(v)):
        conv = 0.0
        for k in range(K):
            conv += taps[k] * full[H + t - k]
        y.append(x3[t] * conv + dskip * v[t])
    hist_out = full[len(full) - H:] if H > 0 else []
    return y, hist_out
