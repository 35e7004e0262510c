#!/usr/bin/env python3
"""Benchmark of the gated Hyena long convolution on B200.

Default workload: the long modal filter (hcl) over B=1, L=32768, D=4096, N=16
real modes, bf16 x1/x2/x3 ~ N(0, 1), single pass.  One step = one call of
hyena_modal_long_conv (coefficient synthesis + the scan kernel: every stage of
the path, from loading x1/x2/x3 to storing y and the final state).

Prints ONE JSON line (rank 0).  Metric: channel-tokens/s (one channel-token =
one (b, t, c) output element); the roofline object reports the dominant
kernel's achieved HBM bandwidth counted at 8 algorithmic bytes per
channel-token (x1, x2, x3 read, y written, bf16 each) against the measured HBM
peak.  Inputs (768 MB) are larger than L2 (126 MB), so no L2 flush is needed
between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Multi-GPU (torchrun): the operator has no cross-GPU step on this path, so each
rank runs an independent replica of the workload on its own GPU (weak
scaling); ranks only meet for the barriers and the max-over-ranks timing.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "hcl long-conv channel-tokens/s at L=32K D=4096; achieved HBM GB/s vs peak"
UNIT = "channel-tokens/s"
BYTES_PER_CHTOK = 8  # 3 bf16 reads + 1 bf16 write

WORKLOADS = {
    "modal32k": dict(kind="modal", B=1, L=32768, D=4096, N=16, seed=2, chunk=None,
                     desc="hcl modal long conv, B=1 L=32768 D=4096 N=16, single pass"),
    "chunked131k": dict(kind="modal", B=1, L=131072, D=4096, N=16, seed=3, chunk=1024,
                        desc="hcl modal long conv, B=1 L=131072 D=4096 N=16, 128 chunks of 1024 with carried state"),
    "long262k": dict(kind="modal", B=1, L=262144, D=4096, N=16, seed=4, chunk=None, wide=True,
                     desc="hcl modal long conv, B=1 L=262144 D=4096 N=16, wide dynamic range, single pass"),
    "fir7": dict(kind="fir", B=2, L=8192, D=4096, K=7, seed=1,
                 desc="hcs explicit FIR K=7, B=2 L=8192 D=4096"),
    "fir128": dict(kind="fir", B=2, L=8192, D=4096, K=128, seed=1,
                   desc="hcm explicit FIR K=128, B=2 L=8192 D=4096"),
    # the same operator as overlap-save DFT-as-GEMM on the tensor cores (tf32)
    "fir128_dft": dict(kind="fir", B=2, L=8192, D=4096, K=128, seed=1, dft=True,
                       desc="hcm explicit FIR K=128, B=2 L=8192 D=4096, tensor-core DFT-as-GEMM (tf32)"),
    # inputs read from one projection buffer interleaved per channel triple
    # (x1_c, x2_c, x3_c adjacent), the in_proj output layout
    "modal32k_triples": dict(kind="modal", B=1, L=32768, D=4096, N=16, seed=2, chunk=None, group=1,
                             desc="hcl modal long conv, B=1 L=32768 D=4096 N=16, single pass, "
                                  "inputs interleaved per channel triple"),
    "fir7_triples": dict(kind="fir", B=2, L=8192, D=4096, K=7, seed=1, group=1,
                         desc="hcs explicit FIR K=7, B=2 L=8192 D=4096, inputs interleaved per channel triple"),
    "fir128_triples": dict(kind="fir", B=2, L=8192, D=4096, K=128, seed=1, group=1,
                           desc="hcm explicit FIR K=128, B=2 L=8192 D=4096, inputs interleaved per channel triple"),
    # more than 16 real modes (two or four lanes per channel pair)
    "modal32k_n32": dict(kind="modal", B=1, L=32768, D=4096, N=32, seed=11, chunk=None,
                         desc="hcl modal long conv, B=1 L=32768 D=4096 N=32, single pass"),
    "modal32k_n64": dict(kind="modal", B=1, L=32768, D=4096, N=64, seed=12, chunk=None,
                         desc="hcl modal long conv, B=1 L=32768 D=4096 N=64, single pass"),
    # complex modes, h[t] = Re sum R p^t (the Evo 1 modal form; state size 8)
    "cmodal8k": dict(kind="modal", cx=True, B=1, L=8192, D=4096, N=8, seed=9, chunk=None,
                     desc="complex-mode modal long conv, B=1 L=8192 D=4096 N=8, single pass"),
    "cmodal32k": dict(kind="modal", cx=True, B=1, L=32768, D=4096, N=8, seed=10, chunk=None,
                      desc="complex-mode modal long conv, B=1 L=32768 D=4096 N=8, single pass"),
    # generation: one step = L one-token decode calls (state / window carried)
    "decode_modal": dict(kind="modal", decode=True, B=1, L=256, D=4096, N=16, seed=5, chunk=None,
                         desc="hcl decode, B=1 D=4096 N=16, 256 one-token steps"),
    "decode_modal_b64": dict(kind="modal", decode=True, B=64, L=64, D=4096, N=16, seed=6, chunk=None,
                             desc="hcl decode, B=64 D=4096 N=16, 64 one-token steps"),
    "decode_fir128": dict(kind="fir", decode=True, B=1, L=256, D=4096, K=128, seed=7,
                          desc="hcm decode, B=1 D=4096 K=128, 256 one-token steps"),
}


def alu_peak_tflops():
    """FP32 SIMT peak of the GPU: SMs x 128 FMA lanes x 2 flops x max SM
    clock (the measured-peaks file's clock when present, else the device's)."""
    import torch
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    mhz = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mhz = float(json.load(f)["sm_max_mhz"])
    except Exception:
        mhz = props.clock_rate / 1e3 if hasattr(props, "clock_rate") else 1965.0
    return props.multi_processor_count * 128 * 2 * mhz * 1e6 / 1e12


def algorithmic_bytes(wl):
    """Bytes a step must move at least: 8 per channel-token (x1, x2, x3 read,
    y written) for prefill; a decode call also reads and writes the carried
    state (N floats) or window (K-1 floats) and reads the filter parameters."""
    chtok = wl["B"] * wl["L"] * wl["D"]
    if not wl.get("decode"):
        return BYTES_PER_CHTOK * chtok
    if wl["kind"] == "modal":
        per_call = wl["B"] * wl["D"] * (8 + 8 * wl["N"]) + wl["D"] * (8 * wl["N"] + 4)
    else:
        per_call = wl["B"] * wl["D"] * (8 + 8 * (wl["K"] - 1)) + wl["D"] * (2 * wl["K"] + 4)
    return per_call * wl["L"]


# Tensor-core work of the DFT-as-GEMM FIR per channel-token: per 64 channels x
# 128 outputs, the taps' spectrum (2 x 128 x 64 x 128 MACs), the window's
# (2 x 128 x 64 x 256) and the inverse (128 x 64 x 256): 1024 MACs.
DFT_FLOPS_PER_CHTOK = 2 * 1024
# Nominal dense tf32 / bf16 tensor rates of a B200 (1.1 and 2.25 PFLOP/s).
TF32_PER_BF16 = 1.1 / 2.25


def tensor_peak_tflops_tf32():
    """Dense tf32 tensor peak: the measured bf16 GEMM rate (burst) when the
    measured-peaks file is present, else a fallback of 1590 TFLOP/s (an
    earlier cuBLAS bf16 measurement on a B200), times the nominal tf32 / bf16
    ratio."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]) * TF32_PER_BF16, "measured bf16_tflops x nominal tf32/bf16"
    except Exception:
        return 1590.0 * TF32_PER_BF16, "fallback bf16 1590 TFLOP/s x nominal tf32/bf16"


def flops_per_chtok(wl):
    """Algorithmic flops per channel-token: the recurrence form's 2N FMAs
    (hcl; complex modes: 6N, four for p s + v and two for Re(R s)) or K FMAs
    (explicit FIR), plus v = x1 x2, the gate and the skip."""
    if wl["kind"] == "modal":
        return (12 if wl.get("cx") else 4) * wl["N"] + 4
    return 2 * wl["K"] + 4


def kernel_fma_per_chtok(wl):
    """FP32 FMA-pipe operations per channel-token that the kernels issue at
    the least: the modal scan sweeps every unit twice (the aggregate, N FMAs
    per real mode slot, then the outputs, 2N), forms v = x1 x2 in both sweeps
    and applies the gate and the skip (3N + 4; complex modes: 4 per mode in
    the aggregate, 6 in the output sweep); the FIR kernels K FMAs plus v, the
    gate and the skip."""
    if wl["kind"] == "modal":
        return (10 * wl["N"] if wl.get("cx") else 3 * wl["N"]) + 4
    if wl.get("dft"):
        return None  # the arithmetic is on the tensor cores
    return wl["K"] + 3


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


KERNEL_SOURCES = {
    "modal": ("hyena_long_convolution_b200/csrc/modal_scan.cu",
              "hyena_long_convolution_b200/csrc/modal_scan_wide.cu",
              "hyena_long_convolution_b200/csrc/modal_synth.cu",
              "hyena_long_convolution_b200/csrc/hyena_device.cuh",
              "hyena_long_convolution_b200/csrc/hyena_internal.h"),
    "fir": ("hyena_long_convolution_b200/csrc/short_conv.cu",
            "hyena_long_convolution_b200/csrc/hyena_device.cuh",
            "hyena_long_convolution_b200/csrc/hyena_internal.h"),
    "fir_dft": ("hyena_long_convolution_b200/csrc/fir_dft.cu",
                "hyena_long_convolution_b200/csrc/hyena_device.cuh",
                "hyena_long_convolution_b200/csrc/hyena_internal.h"),
}


def kernel_source_hash(kind="modal"):
    """sha256/16 of the sources of one kernel family (modal scan or FIR)."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(workload)
    except Exception:
        return None
    wl = WORKLOADS[workload]
    kind = "fir_dft" if wl.get("dft") else wl["kind"]
    if not rec or rec.get("kernel_sources_sha256_16") != kernel_source_hash(kind):
        return None
    return rec.get("dram_bytes_per_launch")


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def workload_config(wl):
    """The workload part of the JSON line's config (shared by both arms)."""
    return {"workload": wl["desc"], "B": wl["B"], "L": wl["L"], "D": wl["D"],
            **({"N": wl["N"], "modes": "complex" if wl.get("cx") else "real"} if wl["kind"] == "modal"
               else {"K": wl["K"]}),
            "mode": "decode (one-token calls)" if wl.get("decode") else "prefill",
            "input_layout": (f"packed projection, channel groups of {wl['group']}" if wl.get("group")
                             else "three [B, L, D] tensors")}


def max_over_ranks(pg, values, device):
    """Element-wise maximum over all ranks of per-rank timings (the slowest
    replica bounds the job); the values themselves without a process group.
    Every rank calls it at the same point with the same number of values."""
    if pg is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_rate(world, units_per_step, steps, total_ms):
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time."""
    return world * units_per_step * steps / (total_ms / 1e3)


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons during the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)  # let the sampler start before the timed region opens
        except Exception:
            self.proc = None
        return self

    def mark(self, which):
        setattr(self, which, time.time())

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        import datetime
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0 = getattr(self, "start", None)
        t1 = getattr(self, "end", None)
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            # a short timed region can fall between two 50 ms samples: then the
            # samples within 0.3 s of it stand in (counted in "samples")
            slack = 0.05 if t0 is None or t1 is None or t1 - t0 > 0.5 else 0.3
            if ts is not None and t0 is not None and t1 is not None and not (t0 - slack <= ts <= t1 + slack):
                continue
            try:
                sm.append(float(parts[2]))
                smax = float(parts[3])
            except ValueError:
                continue
            for nm, val in zip(names, parts[6:10]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle leg


def oracle_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def oracle_single_thread_rate(workload, target_s=2.0):
    """The oracle's rate on one host thread (OpenMP fixed to 1 thread in a child
    process, since the thread count is read when the oracle library loads)."""
    import subprocess
    code = ("import bench, json, os; os.environ['OMP_NUM_THREADS'] = '1'; "
            f"r, smp, th = bench.oracle_sample_rate(bench.WORKLOADS[{workload!r}], {target_s!r}); "
            "print(json.dumps([r, smp, th]))")
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                             timeout=120, check=True).stdout.strip().splitlines()[-1]
        rate, sample, _ = json.loads(out)
        return rate, sample
    except Exception as e:  # a baseline detail: report why it is missing instead of failing the bench
        return None, f"not measured: {type(e).__name__}"


def oracle_sample_rate(wl, target_s=10.0):
    """Times the fp64 oracle (as it stands) on a bounded sample of the workload.

    The sample keeps all L tokens (so long-range decays are exercised) and a
    subset of channels sized for roughly `target_s` seconds of CPU work.
    Returns (channel-tokens/s, sample description, threads).
    """
    import oracle
    from synth import make_cmodal_inputs, make_fir_inputs, make_modal_inputs
    threads = oracle_threads()
    os.environ.setdefault("OMP_NUM_THREADS", str(threads))
    L = wl["L"]
    B = wl["B"]

    def run(D):
        if wl.get("cx"):
            inp = make_cmodal_inputs(B, L, D, wl["N"], wl["seed"])
            t = time.perf_counter()
            oracle.cmodal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["poles"], inp["residues"],
                                     inp["Dskip"])
            return time.perf_counter() - t
        if wl["kind"] == "modal":
            inp = make_modal_inputs(B, L, D, wl["N"], wl["seed"], wl.get("wide", False))
            t = time.perf_counter()
            if wl.get("chunk") or wl.get("decode"):
                oracle.modal_chunked(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"], inp["residues"],
                                     inp["Dskip"], None, chunks=1 if wl.get("decode") else wl["chunk"])
            else:
                oracle.modal_recurrence(inp["x1"], inp["x2"], inp["x3"], inp["log_poles"],
                                        inp["residues"], inp["Dskip"])
            return time.perf_counter() - t
        inp = make_fir_inputs(B, L, D, wl["K"], wl["seed"])
        t = time.perf_counter()
        if wl.get("decode"):
            oracle.fir_chunked(inp["x1"], inp["x2"], inp["x3"], inp["taps"], None, None, chunks=1)
        else:
            oracle.fir(inp["x1"], inp["x2"], inp["x3"], inp["taps"], None, None)
        return time.perf_counter() - t

    oracle.build()
    D0 = max(8, min(wl["D"], 8 * threads))
    dt = run(D0)
    rate = B * L * D0 / max(dt, 1e-9)
    D1 = int(min(wl["D"], max(D0, rate * target_s / (B * L))))
    D1 = max(8, D1 - D1 % 8)
    if D1 > D0:
        dt = run(D1)
        rate = B * L * D1 / max(dt, 1e-9)
    else:
        D1 = D0
    sample = f"B={B} L={L} D={D1} of {wl['D']} channels ({B * L * D1:.3g} channel-tokens), {dt:.1f} s"
    return rate, sample, threads


# ------------------------------------------------------------------ GPU leg


def make_device_inputs(wl, device):
    import torch
    from synth import make_cmodal_inputs, make_fir_inputs, make_modal_inputs

    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)

    if wl.get("cx"):
        inp = make_cmodal_inputs(wl["B"], wl["L"], wl["D"], wl["N"], wl["seed"])
        host = dict(x1=inp["x1"], x2=inp["x2"], x3=inp["x3"], a=inp["poles"], R=inp["residues"], Ds=inp["Dskip"])
        dev = dict(x1=up(inp["x1"]), x2=up(inp["x2"]), x3=up(inp["x3"]),
                   a=torch.from_numpy(inp["poles"]).to(device),
                   R=torch.from_numpy(inp["residues"]).to(device),
                   Ds=torch.from_numpy(inp["Dskip"]).to(device))
    elif wl["kind"] == "modal":
        inp = make_modal_inputs(wl["B"], wl["L"], wl["D"], wl["N"], wl["seed"], wl.get("wide", False))
        host = dict(x1=inp["x1"], x2=inp["x2"], x3=inp["x3"])
        dev = dict(x1=up(inp["x1"]), x2=up(inp["x2"]), x3=up(inp["x3"]),
                   a=torch.from_numpy(inp["log_poles"]).to(device),
                   R=torch.from_numpy(inp["residues"]).to(device),
                   Ds=torch.from_numpy(inp["Dskip"]).to(device))
        host.update(a=inp["log_poles"], R=inp["residues"], Ds=inp["Dskip"])
    else:
        inp = make_fir_inputs(wl["B"], wl["L"], wl["D"], wl["K"], wl["seed"])
        host = dict(x1=inp["x1"], x2=inp["x2"], x3=inp["x3"], taps=inp["taps"])
        dev = dict(x1=up(inp["x1"]), x2=up(inp["x2"]), x3=up(inp["x3"]), taps=up(inp["taps"]))
    if wl.get("group"):
        # one [B, L, 3D] projection buffer, channel groups of `group` as [x1 | x2 | x3]
        G = wl["group"]
        B, L, D = wl["B"], wl["L"], wl["D"]
        xp = np.stack([host.pop(k).reshape(B, L, D // G, G) for k in ("x1", "x2", "x3")], axis=3)
        host["xp"] = np.ascontiguousarray(xp.reshape(B, L, 3 * D))
        for k in ("x1", "x2", "x3"):
            del dev[k]
        dev["xp"] = up(host["xp"])
    return host, dev


class Step:
    """One pass of the hot path over the resident inputs, via the C ABI."""

    def __init__(self, wl, dev, device, graph=False):
        import torch
        import hyena_long_convolution_b200 as hy
        self.hy = hy
        self.wl = wl
        self.dev = dev
        B, L, D = wl["B"], wl["L"], wl["D"]
        self.y = torch.empty((B, L, D), dtype=torch.bfloat16, device=device)
        self.launches = 0
        if wl["kind"] == "modal":
            cx = bool(wl.get("cx"))
            self.ws = hy.ModalWorkspace(B, D, (2 if cx else 1) * wl["N"], device=device)
            self.S = torch.zeros((B, D, wl["N"], 2) if cx else (B, D, wl["N"]), device=device)
        elif wl.get("decode"):
            self.H = torch.zeros((B, wl["K"] - 1, D), device=device)
        self.graph = None
        if graph:
            s = torch.cuda.Stream(device=device)
            s.wait_stream(torch.cuda.current_stream(device))
            with torch.cuda.stream(s):
                self._run()  # warm the per-device kernel attributes outside capture
            torch.cuda.current_stream(device).wait_stream(s)
            torch.cuda.synchronize(device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._run()
            self.graph = g

    def _run(self):
        hy, wl, d = self.hy, self.wl, self.dev
        n = 0
        if wl.get("decode"):
            # a generation loop: the state / window starts empty, one call per token
            if wl["kind"] == "modal":
                hy.modal_state_init(self.S)
            else:
                self.H.zero_()
            n += 1
            for t in range(wl["L"]):
                sl = slice(t, t + 1)
                if wl["kind"] == "modal":
                    hy.modal_decode(d["x1"][:, sl], d["x2"][:, sl], d["x3"][:, sl], d["a"], d["R"], d["Ds"], self.S,
                                    y=self.y[:, sl])
                else:
                    hy.short_decode(d["x1"][:, sl], d["x2"][:, sl], d["x3"][:, sl], d["taps"], None, self.H,
                                    y=self.y[:, sl])
                n += hy.last_launch_count()
            self.launches = n
            return
        if wl.get("cx"):
            hy.modal_long_conv_complex(d["x1"], d["x2"], d["x3"], d["a"], d["R"], d["Ds"], y=self.y,
                                       state_out=self.S, workspace=self.ws)
            self.launches = hy.last_launch_count()
            return
        if wl.get("group"):
            if wl["kind"] == "modal":
                hy.modal_long_conv_packed(d["xp"], wl["group"], d["a"], d["R"], d["Ds"], y=self.y,
                                          state_out=self.S, workspace=self.ws)
            else:
                hy.short_conv_packed(d["xp"], wl["group"], d["taps"], None, y=self.y)
            self.launches = hy.last_launch_count()
            return
        if wl["kind"] == "modal":
            if wl.get("chunk"):
                # chunked prefill of one sequence: the filter is synthesised
                # once, then every chunk runs with the carried state
                hy.modal_state_init(self.S)
                n += hy.last_launch_count()
                hy.modal_prepare(d["a"], d["R"], d["Ds"], self.ws, B=wl["B"])
                n += hy.last_launch_count()
                c = wl["chunk"]
                for t0 in range(0, wl["L"], c):
                    sl = slice(t0, t0 + c)
                    hy.modal_long_conv_prepared(d["x1"][:, sl], d["x2"][:, sl], d["x3"][:, sl], wl["N"], self.ws,
                                                y=self.y[:, sl], state_in=self.S, state_out=self.S)
                    n += hy.last_launch_count()
            else:
                hy.modal_long_conv(d["x1"], d["x2"], d["x3"], d["a"], d["R"], d["Ds"], y=self.y,
                                   state_out=self.S, workspace=self.ws)
                n += hy.last_launch_count()
        else:
            conv = hy.short_conv_dft if wl.get("dft") else hy.short_conv
            conv(d["x1"], d["x2"], d["x3"], d["taps"], None, y=self.y)
            n += hy.last_launch_count()
        self.launches = n

    def __call__(self):
        if self.graph is not None:
            self.graph.replay()
        else:
            self._run()

    def check(self):
        """Raises if a bounded wait inside a modal launch gave up (the timed
        launches would then have produced wrong results quickly)."""
        if getattr(self, "ws", None) is not None:
            self.hy.workspace_check(self.ws)


def time_steps(step, steps, warmup, device):
    import torch
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    stream = torch.cuda.current_stream(device)
    for i in range(steps):
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(device)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return per


E2E_CHUNK = 2048  # tokens per chunk of the host-buffer entry point (16 units)


def e2e_leg(wl, host, dev, device, steps, warmup):
    """Same metric through the public binding with pinned host buffers: every
    step copies x1/x2/x3 (and the filter parameters) host->device, runs the
    operator and copies y device->host, all inside the timed region."""
    import torch
    import hyena_long_convolution_b200 as hy

    def pin(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else a)
        return t.pin_memory()

    hx = {k: pin(v) for k, v in host.items()}
    # Prefill with separate inputs (real modes, FIR) streams its host buffers
    # through the library's host-buffer entry points (chunks, copies in both
    # directions overlapping the computation); everything else copies here.
    streamed = not (wl.get("cx") or wl.get("group") or wl.get("decode") or wl.get("dft"))
    on_host = ("x1", "x2", "x3") if streamed else ()
    dx = {k: torch.empty(v.shape, dtype=v.dtype, device=device) for k, v in hx.items() if k not in on_host}
    y_host = torch.empty((wl["B"], wl["L"], wl["D"]), dtype=torch.int16).pin_memory()
    B, L, D = wl["B"], wl["L"], wl["D"]
    y = torch.empty((B, L, D), dtype=torch.bfloat16, device=device)
    if streamed and wl["kind"] == "modal":
        hws = hy.HostWorkspace(B, D, wl["N"], chunk=E2E_CHUNK, device=device)
    elif streamed:
        hws_fir = torch.empty(int(hy.lib().hyena_short_host_workspace_size(B, D, wl["K"], E2E_CHUNK)),
                              dtype=torch.uint8, device=device)
    if wl["kind"] == "modal":
        cx = bool(wl.get("cx"))
        ws = hy.ModalWorkspace(B, D, (2 if cx else 1) * wl["N"], device=device)
        S = torch.zeros((B, D, wl["N"], 2) if cx else (B, D, wl["N"]), device=device)
    elif wl.get("decode"):
        H = torch.zeros((B, wl["K"] - 1, D), device=device)

    def step():
        for k in dx:
            dx[k].copy_(hx[k], non_blocking=True)
        if streamed:
            xh = [hx[k].view(torch.bfloat16) for k in ("x1", "x2", "x3")]
            if wl["kind"] == "modal":
                hy.modal_long_conv_host(*xh, dx["a"], dx["R"], dx["Ds"], y=y_host, workspace=hws)
            else:
                hy.short_conv_host(*xh, dx["taps"].view(torch.bfloat16), None, y=y_host, chunk=E2E_CHUNK,
                                   workspace=hws_fir)
            return
        bf = {k: dx[k].view(torch.bfloat16) for k in ("x1", "x2", "x3", "xp") if k in dx}
        if wl.get("cx"):
            hy.modal_long_conv_complex(bf["x1"], bf["x2"], bf["x3"], dx["a"], dx["R"], dx["Ds"], y=y, workspace=ws)
        elif wl.get("group"):
            if wl["kind"] == "modal":
                hy.modal_long_conv_packed(bf["xp"], wl["group"], dx["a"], dx["R"], dx["Ds"], y=y, workspace=ws)
            else:
                hy.short_conv_packed(bf["xp"], wl["group"], dx["taps"].view(torch.bfloat16), None, y=y)
        elif wl.get("decode"):
            (S.zero_() if wl["kind"] == "modal" else H.zero_())
            for t in range(L):
                sl = slice(t, t + 1)
                if wl["kind"] == "modal":
                    hy.modal_decode(bf["x1"][:, sl], bf["x2"][:, sl], bf["x3"][:, sl], dx["a"], dx["R"], dx["Ds"],
                                    S, y=y[:, sl])
                else:
                    hy.short_decode(bf["x1"][:, sl], bf["x2"][:, sl], bf["x3"][:, sl],
                                    dx["taps"].view(torch.bfloat16), None, H, y=y[:, sl])
        elif wl["kind"] == "modal":
            hy.modal_long_conv(bf["x1"], bf["x2"], bf["x3"], dx["a"], dx["R"], dx["Ds"], y=y, workspace=ws)
        else:
            conv = hy.short_conv_dft if wl.get("dft") else hy.short_conv
            conv(bf["x1"], bf["x2"], bf["x3"], dx["taps"].view(torch.bfloat16), None, y=y)
        y_host.copy_(y.view(torch.int16), non_blocking=True)

    per = time_steps(step, steps, warmup, device)
    if streamed and wl["kind"] == "modal":
        hy.workspace_check(hws)  # a launch whose bounded wait gave up is an error, not a timing
    elif wl["kind"] == "modal":
        hy.workspace_check(ws)
    h2d = sum(v.numel() * v.element_size() for v in hx.values())
    d2h = y_host.numel() * y_host.element_size()
    return per, h2d, d2h


def run_gpu(args, wl):
    import torch
    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        pg = dist
    import hyena_long_convolution_b200 as hy
    hy.lib()  # fail loudly if the library is missing

    host, dev = make_device_inputs(wl, device)
    step = Step(wl, dev, device, graph=args.graph)
    chtok = wl["B"] * wl["L"] * wl["D"]

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize(device)

    for _ in range(args.warmup):
        step()
    barrier()
    with ClockSampler(local) as clk:
        clk.mark("start")
        per = time_steps(step, args.steps, 0, device)
        clk.mark("end")
    step.check()
    barrier()
    t_total_ms = max_over_ranks(pg, [sum(per)], device)[0]
    ms_step = t_total_ms / args.steps
    value = job_rate(world, chtok, args.steps, t_total_ms)

    # e2e through the binding with host buffers (fewer steps: PCIe-bound)
    e_steps = max(3, min(args.steps, 5))
    eper, h2d, d2h = e2e_leg(wl, host, dev, device, e_steps, 3)
    e_total = max_over_ranks(pg, [sum(eper)], device)[0]
    e_value = job_rate(world, chtok, e_steps, e_total)

    peak, peak_kind = measured_peaks()
    per_sorted = sorted(per)
    avg_ms = statistics.mean(per)
    step_bytes = algorithmic_bytes(wl)
    achieved = step_bytes / (avg_ms / 1e3) / 1e9
    traffic = recorded_traffic(args.workload)
    # The roofline that bounds the path: HBM (8 B per channel-token) unless
    # the algorithmic flops take longer at the SIMT peak (long explicit FIRs).
    alu_peak = alu_peak_tflops()
    flops = flops_per_chtok(wl) * chtok
    if wl.get("dft"):
        # the DFT path's own arithmetic on the tensor cores bounds it
        tc_peak, tc_src = tensor_peak_tflops_tf32()
        mma_flops = DFT_FLOPS_PER_CHTOK * chtok
        roof = {"bound": "tensor", "achieved": mma_flops / (avg_ms / 1e3) / 1e12, "peak": tc_peak,
                "unit": "TFLOP/s", "peak_source": tc_src, "algorithmic_flops_per_launch": mma_flops}
    elif flops / (alu_peak * 1e12) > step_bytes / (peak * 1e9):
        roof = {"bound": "alu", "achieved": flops / (avg_ms / 1e3) / 1e12, "peak": alu_peak, "unit": "TFLOP/s",
                "peak_source": "derived: SMs x 128 FP32 lanes x 2 flops x max SM clock",
                "algorithmic_flops_per_launch": flops}
    else:
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "peak_source": f"{peak_kind} hbm_gbs (copy)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    # The kernels' own arithmetic floor: their FMA-pipe work at the SIMT peak
    # (a step cannot beat it however well its memory traffic is hidden).
    fma_pc = kernel_fma_per_chtok(wl)
    fma_floor_ms = fma_pc * chtok / (alu_peak * 1e12 / 2) * 1e3 if fma_pc and not wl.get("decode") else None
    roof.update({"traffic": traffic, "algorithmic_bytes_per_step": step_bytes,
                 "hbm_frac": achieved / peak, "kernel_ms_min": per_sorted[0], "kernel_ms_avg": avg_ms,
                 "fma_floor_ms": fma_floor_ms,
                 "fma_floor_frac": (fma_floor_ms / avg_ms) if fma_floor_ms else None})

    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "io_dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 inputs, pages' shapes)",
        "config": {**workload_config(wl),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "cache": "inputs larger than L2 (no flush)", "graph": bool(args.graph)},
        "roofline": roof,
        "e2e": {"value": e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e_total / e_steps},
        "gpu_launches": step.launches * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, sample, threads = oracle_sample_rate(wl, args.cpu_seconds)
        rate1, sample1 = oracle_single_thread_rate(args.workload)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": sample, "cpu_model": cpu_model(),
                                "single_thread": {"value": rate1, "sample": sample1}}
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, wl):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    rate_samples = []
    sample = ""
    threads = oracle_threads()
    per_step = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        rate, sample, threads = oracle_sample_rate(wl, per_step)
        if i >= args.warmup:
            rate_samples.append(rate)
    value = statistics.mean(rate_samples)
    chtok = wl["B"] * wl["L"] * wl["D"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": chtok / value * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**workload_config(wl), "parallelism": "host cores (fp64 oracle)"},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"per step: {sample}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="modal32k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--graph", action="store_true", help="replay each step as a captured CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()
