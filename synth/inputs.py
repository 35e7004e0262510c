"""Deterministic synthetic workloads for the gated Hyena cascade operator.

The pages measure only on genomic data that is not available here, so these
seeded draws stand in for it with the pages' shapes: D = 4096 channels
(Evo2-7B-262K model card, §Architecture), 8K to 262K tokens of context and
1024-token prefill chunks (turboquant-evo2-int4 model card, §"Chunk size").

Recipe (every config):
  * x1, x2, x3: iid N(0, 1) fp32 draws, rounded to bf16 (round to nearest
    even).  Tensor k (0, 1, 2 for x1, x2, x3) is drawn in blocks of
    ``ROW_BLOCK`` flattened (b, t) rows; block j uses
    ``numpy.random.default_rng([seed, k, j])``, so blocks can be drawn in
    parallel and any block can be regenerated alone.
  * modal parameters from ``default_rng([seed, 100])``, in this order:
    log-poles a = -exp(U(ln 1e-3, 0)) as fp32 [D, N]; residues R ~ N(0, 1/N)
    as fp32 [D, N]; skip Dskip ~ N(0, 1) as fp32 [D].
  * wide-dynamic-range option: after the parameters, the same generator draws
    per-(tensor, channel) factors 10^U(-2, 2) [3, D]; each x tensor is
    multiplied by its factor in fp32 before rounding to bf16.
  * FIR taps from ``default_rng([seed, 101])``: N(0, 1/K) fp32 [D, K] rounded
    to bf16; FIR skip (when requested) from the same generator, N(0, 1).
  * complex modal parameters from ``default_rng([seed, 102])``, in this order:
    pole moduli r = exp(-exp(U(ln 1e-3, 0))) [D, N] (the real log-pole draw,
    exponentiated), pole angles U(0, pi) [D, N], residues (N(0, 1) + i N(0, 1))
    / sqrt(2N) [D, N], skip N(0, 1) [D]; poles r (cos, sin) and residues are
    stored as fp32 [D, N, 2] (real, imaginary).

All integer bit patterns are numpy uint16 arrays so the oracle and the GPU read
identical bits.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ROW_BLOCK = 1024

# The five acceptance workloads, by name: shapes and distributions; each
# name's seed is fixed here and used for every draw of that workload.
WORKLOAD_SHAPES = {
    "modal_1k": dict(kind="modal", B=1, L=1024, D=64, N=8, seed=0, wide_range=False,
                     name="modal B1 L1024 D64 N8"),
    "fir_8k": dict(kind="fir", B=2, L=8192, D=4096, K=(7, 128), seed=1,
                   name="short FIR B2 L8192 D4096 K7/K128"),
    "modal_32k": dict(kind="modal", B=1, L=32768, D=4096, N=16, seed=2, wide_range=False,
                      name="modal B1 L32768 D4096 N16"),
    "modal_131k_chunked": dict(kind="modal", B=1, L=131072, D=4096, N=16, seed=3, wide_range=False,
                               chunk=1024, name="modal B1 L131072 D4096 N16, 128 chunks of 1024"),
    "modal_262k_wide": dict(kind="modal", B=1, L=262144, D=4096, N=16, seed=4, wide_range=True,
                            name="modal B1 L262144 D4096 N16, wide dynamic range"),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits.

    Inputs are finite draws, so no NaN handling is needed here.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _draw_tensor(seed: int, k: int, rows: int, D: int, scale: np.ndarray | None,
                 out: np.ndarray, threads: int) -> None:
    nblk = (rows + ROW_BLOCK - 1) // ROW_BLOCK

    def one(j: int) -> None:
        r0 = j * ROW_BLOCK
        r1 = min(rows, r0 + ROW_BLOCK)
        g = np.random.default_rng([seed, k, j])
        blk = g.standard_normal((r1 - r0, D), dtype=np.float32)
        if scale is not None:
            blk *= scale[None, :]
        out[r0:r1] = f32_to_bf16_bits(blk)

    if threads <= 1 or nblk == 1:
        for j in range(nblk):
            one(j)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, range(nblk)))


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(32, os.cpu_count() or 1))


def make_x(seed: int, B: int, L: int, D: int, scales: np.ndarray | None = None,
           threads: int | None = None):
    """Draw x1, x2, x3 as uint16 bf16 bits, shape [B, L, D]."""
    threads = _threads() if threads is None else threads
    xs = []
    for k in range(3):
        out = np.empty((B * L, D), dtype=np.uint16)
        _draw_tensor(seed, k, B * L, D, None if scales is None else scales[k], out, threads)
        xs.append(out.reshape(B, L, D))
    return xs


def make_modal_params(seed: int, D: int, N: int, wide_range: bool = False):
    g = np.random.default_rng([seed, 100])
    a = (-np.exp(g.uniform(math.log(1e-3), 0.0, size=(D, N)))).astype(np.float32)
    R = (g.standard_normal((D, N)) / math.sqrt(N)).astype(np.float32)
    Dskip = g.standard_normal(D).astype(np.float32)
    scales = None
    if wide_range:
        scales = (10.0 ** g.uniform(-2.0, 2.0, size=(3, D))).astype(np.float32)
    return a, R, Dskip, scales


def make_cmodal_params(seed: int, D: int, N: int):
    g = np.random.default_rng([seed, 102])
    r = np.exp(-np.exp(g.uniform(math.log(1e-3), 0.0, size=(D, N))))
    theta = g.uniform(0.0, math.pi, size=(D, N))
    Rre = g.standard_normal((D, N))
    Rim = g.standard_normal((D, N))
    Dskip = g.standard_normal(D).astype(np.float32)
    poles = np.stack([r * np.cos(theta), r * np.sin(theta)], axis=-1).astype(np.float32)
    residues = (np.stack([Rre, Rim], axis=-1) / math.sqrt(2 * N)).astype(np.float32)
    return poles, residues, Dskip


def make_cmodal_inputs(B: int, L: int, D: int, N: int, seed: int, threads: int | None = None) -> dict:
    """x1, x2, x3 as for the real modal filter; N complex modes (poles and
    residues fp32 [D, N, 2])."""
    poles, residues, Dskip = make_cmodal_params(seed, D, N)
    x1, x2, x3 = make_x(seed, B, L, D, None, threads)
    return dict(x1=x1, x2=x2, x3=x3, poles=poles, residues=residues, Dskip=Dskip, B=B, L=L, D=D, N=N)


def make_modal_inputs(B: int, L: int, D: int, N: int, seed: int,
                      wide_range: bool = False, threads: int | None = None) -> dict:
    a, R, Dskip, scales = make_modal_params(seed, D, N, wide_range)
    x1, x2, x3 = make_x(seed, B, L, D, scales, threads)
    return dict(x1=x1, x2=x2, x3=x3, log_poles=a, residues=R, Dskip=Dskip,
                scales=scales, B=B, L=L, D=D, N=N)


def make_fir_inputs(B: int, L: int, D: int, K: int, seed: int, with_skip: bool = False,
                    threads: int | None = None) -> dict:
    g = np.random.default_rng([seed, 101])
    taps = f32_to_bf16_bits((g.standard_normal((D, K)) / math.sqrt(K)).astype(np.float32))
    Dskip = g.standard_normal(D).astype(np.float32) if with_skip else None
    x1, x2, x3 = make_x(seed, B, L, D, None, threads)
    return dict(x1=x1, x2=x2, x3=x3, taps=taps, Dskip=Dskip, B=B, L=L, D=D, K=K)


def make_workload_inputs(name: str, K: int | None = None, threads: int | None = None) -> dict:
    cfg = WORKLOAD_SHAPES[name]
    if cfg["kind"] == "fir":
        K = cfg["K"][0] if K is None else K
        return make_fir_inputs(cfg["B"], cfg["L"], cfg["D"], K, cfg["seed"], threads=threads)
    return make_modal_inputs(cfg["B"], cfg["L"], cfg["D"], cfg["N"], cfg["seed"],
                             cfg["wide_range"], threads)
