#!/usr/bin/env python
"""Throughput of block-scaled NVFP4 quantization on B200.

One step quantizes the tensors of one Llama-style MLP up-projection training
step (X 16384x4096, W 14336x4096, dY 16384x14336, bf16) the way a fully-NVFP4
linear layer needs them: RTN on X and W along d_model (forward), MS-EDEN with
a 128-point random Hadamard rotation on dY row-wise and transposed, and on X
and W transposed (backward) -- six quantize calls through the library's C
ABI, each tensor's two tensor amaxes first, from one read of the tensor
(nvfp4_amax_dual).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  value = algorithmic bytes (2 B read + 0.5 B
codes + 0.0625 B scales per element of every call) / device time, all ranks
summed (weak scaling: each rank quantizes its own step's tensors, no data-path
collective).  The K timed steps are captured once as a CUDA graph of the
C-ABI launches and replayed once, with CUDA events between the launches, so
host enqueue time stays out of the device timeline; L2 is flushed (a 256 MiB
write) before every timed step, outside the marks.  --impl reference times the
CPU oracle, run over ranges of view rows on every host core, on a bounded
sample of the same workload.
"""
import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

METRIC = "NVFP4 quantize GB/s and % of B200 HBM peak per mode (Gelem/s), 1 GPU"
UNIT = "GB/s"
BYTES_PER_ELEMENT = 2.0 + 0.5 + 0.0625   # bf16 in, E2M1 codes out, E4M3 scales out
PREPASS_BYTES_PER_ELEMENT = 2.0          # the amax pre-pass reads the tensor once more
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20

# DRAM bytes per launch measured by ncu for the dominant kernel, keyed by the
# hash of the kernel sources they were taken with.  A changed kernel reports
# traffic = null until it is captured again.
NCU_TRAFFIC = {
    # the ncu capture of the dominant launch at full size (one pass):
    # dram__bytes_read.sum + dram__bytes_write.sum, one launch
    ("fa43c9f0070e72b0", "quantize_dual dy (dy.rowwise.ms_eden.g128 + dy.transposed.ms_eden.g128)"):
        472454400 + 224126976,
    ("65a6a919a9ff92ea", "quantize_dual dy (dy.rowwise.ms_eden.g128 + dy.transposed.ms_eden.g128)"):
        472376576 + 223989760,
    ("e67268332ab8fc9f", "quantize_dual dy (dy.rowwise.ms_eden.g128 + dy.transposed.ms_eden.g128)"):
        472720896 + 224553728,
    ("7abb43885c7454fa", "quantize_dual dy (dy.rowwise.ms_eden.g128 + dy.transposed.ms_eden.g128)"):
        472767744 + 224883968,
    ("8d52fa3e473e5908", "quantize_dual dy (dy.rowwise.ms_eden.g128 + dy.transposed.ms_eden.g128)"):
        472467456 + 224157952,
    ("159b0bcef2cc77d9", "quantize_dual dy (dy.rowwise.ms_eden.g128 + dy.transposed.ms_eden.g128)"):
        472862976 + 224496384,
    ("3bbcfdfa5970de20", "quantize_dual dy (dy.rowwise.ms_eden.g128 + dy.transposed.ms_eden.g128)"):
        472672000 + 224679936,
    ("886b5cad3ef870ce", "quantize_dual dy (dy.rowwise.ms_eden.g128 + dy.transposed.ms_eden.g128)"):
        472838144 + 224669440,
}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=None,
                   help="steps of the end-to-end measurement (default: --steps)")
    p.add_argument("--cpu-sample-fraction", type=float, default=1.0 / 8,
                   help="fraction of each call's view rows the CPU baseline quantizes")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-gemm", action="store_true",
                   help="skip the NVFP4 GEMMs of the step (measured after the quantization step)")
    p.add_argument("--no-per-mode", action="store_true",
                   help="skip the per-mode table (every mode on dY, quantize kernel alone)")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workloads' calls (256x256, weight, gradient, activation)")
    p.add_argument("--profile-case", default=None, metavar="ROWSxCOLS",
                   help="profiling run: only one gradient-like tensor of this shape through the step's launches "
                        "(dual pre-pass, dual quantize, single-layout MS-EDEN and RTN quantizes), --steps times; "
                        "prints the per-launch times, not the benchmark line")
    p.add_argument("--profile-modes", default="", metavar="MODES",
                   help="with --profile-case: also quantize row-wise in these modes (comma-separated names, "
                        "e.g. sr,if4,4over6), without rotation and with g = 128")
    p.add_argument("--no-unfused", action="store_true",
                   help="skip the comparison step with one quantize launch per call")
    p.add_argument("--no-eager", action="store_true",
                   help="skip the eager (host-launched) run reported beside the graph-timed value")
    return p.parse_args(argv)


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world, device=None):
    if world > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value over all ranks (every rank takes part)."""
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(bytes_per_rank_step: float, steps: int, world: int, max_seconds: float) -> float:
    """GB/s of the whole job: every rank's bytes over the slowest rank's time."""
    return bytes_per_rank_step * steps * world / max_seconds / 1e9


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.path:
            self.out.close()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak_bf16():
    """Measured dense bf16 tensor throughput (TFLOP/s, burst), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback"


def kernel_source_hash():
    """Hash of the dominant kernel's sources: the tensor-core translation unit
    and every header (the other translation units do not reach it)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nvfp4_microscaling_quantization_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith(".cu") and name != "rotate_mma.cu":
            continue
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------- our CUDA path
class Call:
    """One quantization call bound to device buffers, issued through the raw C ABI."""

    def __init__(self, N, call, x, seed, stream_handle):
        self.N, self.call, self.x, self.seed = N, call, x, seed
        rows, cols = x.shape
        self.rows, self.cols, self.ld = rows, cols, x.stride(0)
        self.elements = rows * cols
        self.codes, self.scales, self.gscale = N.alloc_outputs(rows, cols, call.layout, x.device)
        self.amax = torch.empty(1, dtype=torch.float32, device=x.device)
        P = ctypes.c_void_p
        self.p = dict(x=P(x.data_ptr()), codes=P(self.codes.data_ptr()), scales=P(self.scales.data_ptr()),
                      gscale=P(self.gscale.data_ptr()), amax=P(self.amax.data_ptr()))
        self.stream = stream_handle

    def amax_pass(self):
        st = self.N.nvfp4_amax(self.p["x"], self.rows, self.cols, self.ld, self.call.layout,
                               self.call.rht_group, self.seed, self.p["amax"], self.stream)
        if st:
            raise self.N.Nvfp4Error(st, "nvfp4_amax")

    def quantize(self):
        st = self.N.nvfp4_quantize(self.p["x"], self.rows, self.cols, self.ld, self.call.layout, self.call.mode,
                                   self.call.rht_group, self.seed, self.p["amax"], self.p["codes"],
                                   self.p["scales"], self.p["gscale"], None, 0, self.stream)
        if st:
            raise self.N.Nvfp4Error(st, "nvfp4_quantize")

    def output_bytes(self):
        return self.codes.numel() + self.scales.numel() + 4


class TensorCalls:
    """The calls on one tensor.  A tensor quantized in both layouts gets its
    two tensor amaxes from one nvfp4_amax_dual pre-pass (one read of the
    tensor); any other set of calls runs one pre-pass per call."""

    def __init__(self, N, calls):
        self.N, self.calls = N, calls
        layouts = sorted(c.call.layout for c in calls)
        self.dual = len(calls) == 2 and layouts == [0, 1]
        if self.dual:
            self.row = next(c for c in calls if c.call.layout == 0)
            self.col = next(c for c in calls if c.call.layout == 1)

    def amax_passes(self):
        if not self.dual:
            for c in self.calls:
                c.amax_pass()
            return
        r, c = self.row, self.col
        st = self.N.nvfp4_amax_dual(r.p["x"], r.rows, r.cols, r.ld, r.call.rht_group, c.call.rht_group, r.seed,
                                    r.p["amax"], c.p["amax"], r.stream)
        if st:
            raise self.N.Nvfp4Error(st, "nvfp4_amax_dual")

    def quantize_dual(self):
        """Both layouts' codes and scales from one read (nvfp4_quantize_dual)."""
        r, c = self.row, self.col
        st = self.N.nvfp4_quantize_dual(r.p["x"], r.rows, r.cols, r.ld, r.call.mode, r.call.rht_group, c.call.mode,
                                        c.call.rht_group, r.seed, r.p["amax"], c.p["amax"], r.p["codes"],
                                        r.p["scales"], r.p["gscale"], c.p["codes"], c.p["scales"], c.p["gscale"],
                                        r.stream)
        if st:
            raise self.N.Nvfp4Error(st, "nvfp4_quantize_dual")

    def body(self, fused):
        """The launches of this tensor's part of a step: its pre-pass(es), then
        one dual quantize (fused) or one quantize per call."""
        out = [(self.amax_passes, "amax", self)]
        if fused and self.dual:
            out.append((self.quantize_dual, "dual", self))
        else:
            out += [(c.quantize, "quant", c) for c in self.calls]
        return out

    def launches(self, fused=True):
        pre = 1 if self.dual else len(self.calls)
        return pre + (1 if fused and self.dual else len(self.calls))

    def label(self):
        return self.calls[0].call.tensor

    def prepass_elements(self):
        """Elements the pre-pass launch(es) read."""
        return self.calls[0].elements if self.dual else sum(c.elements for c in self.calls)

    def dual_calls(self):
        return [self.row, self.col]


class DualGroupCalls:
    """Several tensors quantized in both layouts with the same modes and
    rotation groups (the linear layer's forward operands X and W): one
    both-layout pre-pass launch and one both-layout quantize launch for all
    of them (nvfp4_amax_dual_group, nvfp4_quantize_dual_group), each walking
    all their tiles with one persistent grid."""

    def __init__(self, N, members):
        self.N, self.members, self.dual = N, members, True
        self.calls = [c for m in members for c in m.calls]
        rows, cols = [m.row for m in members], [m.col for m in members]
        self.n = len(members)
        r0, c0 = rows[0], cols[0]
        self.modes = (r0.call.mode, r0.call.rht_group, c0.call.mode, c0.call.rht_group)
        self.seed, self.stream = r0.seed, r0.stream
        ptrs = lambda vals: (ctypes.c_void_p * self.n)(*vals)  # noqa: E731
        i64s = lambda vals: (ctypes.c_int64 * self.n)(*vals)  # noqa: E731
        self.a = dict(x=ptrs([r.p["x"] for r in rows]), rows=i64s([r.rows for r in rows]),
                      cols=i64s([r.cols for r in rows]), ld=i64s([r.ld for r in rows]),
                      amax_r=ptrs([r.p["amax"] for r in rows]), amax_c=ptrs([c.p["amax"] for c in cols]),
                      codes_r=ptrs([r.p["codes"] for r in rows]), scales_r=ptrs([r.p["scales"] for r in rows]),
                      gscale_r=ptrs([r.p["gscale"] for r in rows]), codes_c=ptrs([c.p["codes"] for c in cols]),
                      scales_c=ptrs([c.p["scales"] for c in cols]), gscale_c=ptrs([c.p["gscale"] for c in cols]))

    def amax_passes(self):
        a, (_, g_r, _, g_c) = self.a, self.modes
        st = self.N.nvfp4_amax_dual_group(self.n, a["x"], a["rows"], a["cols"], a["ld"], g_r, g_c, self.seed,
                                          a["amax_r"], a["amax_c"], self.stream)
        if st:
            raise self.N.Nvfp4Error(st, "nvfp4_amax_dual_group")

    def quantize_dual(self):
        a, (m_r, g_r, m_c, g_c) = self.a, self.modes
        st = self.N.nvfp4_quantize_dual_group(self.n, a["x"], a["rows"], a["cols"], a["ld"], m_r, g_r, m_c, g_c,
                                              self.seed, a["amax_r"], a["amax_c"], a["codes_r"], a["scales_r"],
                                              a["gscale_r"], a["codes_c"], a["scales_c"], a["gscale_c"],
                                              self.stream)
        if st:
            raise self.N.Nvfp4Error(st, "nvfp4_quantize_dual_group")

    def body(self, fused=True):
        return [(self.amax_passes, "amax", self), (self.quantize_dual, "dual", self)]

    def launches(self, fused=True):
        return 2

    def label(self):
        return "+".join(m.label() for m in self.members)

    def prepass_elements(self):
        return sum(m.row.elements for m in self.members)

    def dual_calls(self):
        return [c for m in self.members for c in (m.row, m.col)]


def group_step_parts(parts):
    """The step's launch groups: tensors quantized in both layouts with the
    same modes and rotation groups share a DualGroupCalls (in order of first
    appearance); the others keep their own."""
    out, by_modes = [], {}
    for p in parts:
        if not p.dual:
            out.append([p])
            continue
        key = (p.row.call.mode, p.row.call.rht_group, p.col.call.mode, p.col.call.rht_group)
        if key in by_modes:
            by_modes[key].append(p)
        else:
            by_modes[key] = [p]
            out.append(by_modes[key])
    return [ms[0] if len(ms) == 1 else DualGroupCalls(ms[0].N, ms) for ms in out]


def dist_us(seconds):
    """mean, median, p10 and p90 of a list of durations, in microseconds."""
    a = np.asarray(seconds, dtype=np.float64) * 1e6
    return {"mean": round(float(a.mean()), 2), "median": round(float(np.median(a)), 2),
            "p10": round(float(np.percentile(a, 10)), 2), "p90": round(float(np.percentile(a, 90)), 2)}


class GraphTimer:
    """Times launch sequences inside one CUDA graph.

    Each of `reps` repetitions is: an L2 flush (a write of L2_FLUSH_BYTES,
    outside the marks), then the callables of `body` with a CUDA event
    recorded before the first, between each two and after the last.  The
    repetitions are captured once on `stream` (the callables launch on it
    through the C ABI) and the graph is replayed once, so the host takes no
    part while the marks are being recorded: the device runs every launch
    back to back.  durations()[r][i] is callable i of repetition r, seconds.
    With per_launch=False only the repetition's first and last marks are
    recorded, so consecutive launches are adjacent graph nodes (a kernel
    launched with programmatic stream serialization can then start its
    prologue during its predecessor's tail); totals() only."""

    def __init__(self, stream, body, reps, flush, per_launch=True):
        self.stream, self.body, self.reps, self.flush = stream, body, reps, flush
        self.per_launch = per_launch
        mk = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
        n_marks = len(body) + 1 if per_launch else 2
        self.ev = [[mk() for _ in range(n_marks)] for _ in range(reps)]
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=stream, capture_error_mode="thread_local"):
            for r in range(reps):
                if flush is not None:
                    flush.zero_()
                self.ev[r][0].record()
                for i, fn in enumerate(body):
                    fn()
                    if per_launch:
                        self.ev[r][i + 1].record()
                if not per_launch:
                    self.ev[r][1].record()

    def replay(self):
        self.graph.replay()

    def durations(self):
        return [[self.ev[r][i].elapsed_time(self.ev[r][i + 1]) / 1e3 for i in range(len(self.body))]
                for r in range(self.reps)]

    def totals(self):
        return [self.ev[r][0].elapsed_time(self.ev[r][-1]) / 1e3 for r in range(self.reps)]

    def release(self):
        self.graph.reset()
        self.graph = None


def timed_in_graph(stream, body, reps, flush, device, per_launch=True):
    """Capture, replay once, and return (per-callable durations or None, per-rep totals)."""
    t = GraphTimer(stream, body, reps, flush, per_launch=per_launch)
    torch.cuda.synchronize(device)
    t.replay()
    torch.cuda.synchronize(device)
    out = (t.durations() if per_launch else None), t.totals()
    t.release()
    return out


def call_line(name, elements, secs, peak):
    d = dist_us(secs)
    t = d["mean"] / 1e6
    gbs = BYTES_PER_ELEMENT * elements / t / 1e9
    return {"call": name, "elements": elements, "us": d, "gbs": round(gbs, 1), "gelem_s": round(elements / t / 1e9, 1),
            "frac_of_hbm_peak": round(gbs / peak, 4)}


def per_mode_table(N, W, x, seed, stream, sh, device, flush, peak, reps=5):
    """Every mode on one tensor (the headline gradient dY), both layouts, with
    and without the 128-point rotation: the quantize kernel alone with the
    tensor amax supplied (from its own pre-pass), L2 flushed before each
    launch, timed inside a CUDA graph.  MS-EDEN is defined with the rotation only."""
    from nvfp4_microscaling_quantization_b200.workloads import Call as WCall
    out = []
    for layout in (W.ROWWISE, W.TRANSPOSED):
        for mode in (W.RTN, W.SR, W.MS_EDEN, W.IF4, W.FOUR_OVER_SIX, W.SCALE_SEARCH, W.MXFP4, W.NVINT4,
                     W.NVFP3, W.NVINT3, W.IF3, W.MXFP3):
            for g in (0, 128):
                if mode == W.MS_EDEN and g == 0:
                    continue
                c = Call(N, WCall("dy", layout, mode, g), x, seed, sh)
                with torch.cuda.stream(stream):
                    c.amax_pass()
                    c.quantize()
                durs, _ = timed_in_graph(stream, [c.quantize], reps, flush, device)
                out.append(call_line(c.call.name, c.elements, [d[0] for d in durs], peak))
                del c
    torch.cuda.synchronize(device)
    return out


def workload_table(N, W, stream, sh, device, flush, peak, reps=10):
    """The other configurations' calls, each on its own tensor: the quantize
    kernel with the tensor amax supplied (`quantize`), and the two-pass path
    that computes the amax first (`two_pass`: pre-pass + quantize).  L2 is
    flushed before each repetition; CUDA graph timing."""
    out = []
    for make in (W.small, W.weight, W.gradient, W.activation):
        wl = make()
        tensors = wl.tensors(device)
        lines = []
        for wc in wl.calls:
            c = Call(N, wc, tensors[wc.tensor], wl.seed, sh)
            with torch.cuda.stream(stream):
                c.amax_pass()
                c.quantize()
            durs, _ = timed_in_graph(stream, [c.amax_pass, c.quantize], reps, flush, device)
            q = call_line(wc.name, c.elements, [d[1] for d in durs], peak)
            two = call_line(wc.name, c.elements, [d[0] + d[1] for d in durs], peak)
            lines.append({"call": wc.name, "elements": c.elements,
                          "quantize": {k: q[k] for k in ("us", "gbs", "gelem_s", "frac_of_hbm_peak")},
                          "two_pass": {k: two[k] for k in ("us", "gbs", "gelem_s", "frac_of_hbm_peak")}})
            del c
        out.append({"workload": wl.name, "description": wl.description,
                    "shapes": {k: list(v) for k, v in wl.shapes.items()}, "seed": wl.seed, "calls": lines})
        del tensors
        torch.cuda.synchronize(device)
    return out


def gemm_table(N, calls, stream, device, reps=10):
    """The three GEMMs of the linear layer's training step on the step's own
    quantized outputs (nvfp4_gemm, bf16 D): Y = X W^T (RTN X and W row-wise),
    dX = dY W (MS-EDEN dY row-wise, W transposed), dW = dY^T X (MS-EDEN dY and
    X transposed).  Timed inside a CUDA graph (no L2 flush: the operands are
    re-read from L2 within a launch anyway); the fp4 dense tensor peak is the
    measured bf16 peak x 4 (nominal 9 / 2.25 PF)."""
    by = {c.call.name: c for c in calls}
    q = lambda name: (by[name].codes, by[name].scales, by[name].gscale)  # noqa: E731
    cases = [("Y = X W^T", "x.rowwise.rtn.norht", "w.rowwise.rtn.norht"),
             ("dX = dY W", "dy.rowwise.ms_eden.g128", "w.transposed.ms_eden.g128"),
             ("dW = dY^T X", "dy.transposed.ms_eden.g128", "x.transposed.ms_eden.g128")]
    peak_bf16, kind = tensor_peak_bf16()
    peak = 4.0 * peak_bf16
    out = []
    for name, an, bn in cases:
        a, b = q(an), q(bn)
        m, k, n = a[0].shape[0], 2 * a[0].shape[1], b[0].shape[0]
        d = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        with torch.cuda.stream(stream):
            for _ in range(3):
                N.gemm(a, b, out=d)
        durs, _ = timed_in_graph(stream, [lambda: N.gemm(a, b, out=d)], reps, None, device)
        ts = dist_us([x[0] for x in durs])
        tf = 2.0 * m * n * k / (ts["mean"] / 1e6) / 1e12
        out.append({"gemm": name, "a": an, "b": bn, "m": m, "n": n, "k": k, "out": "bf16",
                    "us": ts, "tflops": round(tf, 1),
                    "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": round(peak, 1),
                                 "peak_kind": f"fp4 dense = 4 x {kind} bf16", "unit": "TFLOP/s",
                                 "frac": round(tf / peak, 4)}})
        del d
    torch.cuda.synchronize(device)
    return out


def linear_layer_table(N, groups, stream, device, flush, tensors, reps=10):
    """The Quartet II linear layer of the MLP up-projection, fully NVFP4, as
    one forward and one backward pass:
      forward : X and W's both-layout pre-pass and both-layout quantize, one
                launch each for the two operands (row-wise RTN for Y,
                transposed MS-EDEN kept for the backward pass), then
                Y = X W^T (nvfp4_gemm, bf16 out);
      backward: dY's dual pre-pass and dual quantize (MS-EDEN both ways),
                then dX = dY W and dW = dY^T X (nvfp4_gemm, bf16 out).
    Timed inside CUDA graphs (L2 flushed before each repetition), beside the
    same three GEMMs in bf16 through torch.matmul (cuBLAS) on the unquantized
    tensors -- the comparison behind the pages' "up to 4.2x faster than BF16"
    for their Blackwell kernels (context, not a target)."""
    by = {g.calls[0].call.tensor: g for g in groups}
    gx, gw, gdy = by["x"], by["w"], by["dy"]
    q = lambda c: (c.codes, c.scales, c.gscale)  # noqa: E731
    x, w, dy = tensors["x"], tensors["w"], tensors["dy"]
    y = torch.empty(x.shape[0], w.shape[0], dtype=torch.bfloat16, device=device)
    dx = torch.empty(dy.shape[0], w.shape[1], dtype=torch.bfloat16, device=device)
    dw = torch.empty(dy.shape[1], x.shape[1], dtype=torch.bfloat16, device=device)
    gxw = DualGroupCalls(N, [gx, gw])
    fwd = [gxw.amax_passes, gxw.quantize_dual, lambda: N.gemm(q(gx.row), q(gw.row), out=y)]
    bwd = [gdy.amax_passes, gdy.quantize_dual,
           lambda: N.gemm(q(gdy.row), q(gw.col), out=dx),
           lambda: N.gemm(q(gdy.col), q(gx.col), out=dw)]
    with torch.cuda.stream(stream):
        for fn in fwd + bwd:
            fn()
    # pass times with marks at the pass boundaries only; the per-launch split
    # from a second, instrumented replay
    _, t_fwd = timed_in_graph(stream, fwd, reps, flush, device, per_launch=False)
    _, t_bwd = timed_in_graph(stream, bwd, reps, flush, device, per_launch=False)
    d_fwd, _ = timed_in_graph(stream, fwd, reps, flush, device)
    d_bwd, _ = timed_in_graph(stream, bwd, reps, flush, device)
    bf = [lambda: torch.matmul(x, w.t(), out=y), lambda: torch.matmul(dy, w, out=dx),
          lambda: torch.matmul(dy.t(), x, out=dw)]
    with torch.cuda.stream(stream):
        for fn in bf:
            fn()
    _, t_bf = timed_in_graph(stream, bf, reps, flush, device, per_launch=False)
    d_bf, _ = timed_in_graph(stream, bf, reps, flush, device)
    torch.cuda.synchronize(device)
    f, b, r = dist_us(t_fwd), dist_us(t_bwd), dist_us(t_bf)
    m, k, n = x.shape[0], x.shape[1], w.shape[0]
    flops = 3 * 2.0 * m * n * k
    names_f = ["amax_dual x+w", "quantize_dual x+w", "gemm Y = X W^T"]
    names_b = ["amax_dual dy", "quantize_dual dy", "gemm dX = dY W", "gemm dW = dY^T X"]
    step_us = f["median"] + b["median"]
    return {
        "shapes": {"x": list(x.shape), "w": list(w.shape), "dy": list(dy.shape)},
        "forward_us": f, "backward_us": b, "step_us": round(step_us, 2),
        "forward_launches": {nm: dist_us([d[i] for d in d_fwd]) for i, nm in enumerate(names_f)},
        "backward_launches": {nm: dist_us([d[i] for d in d_bwd]) for i, nm in enumerate(names_b)},
        "gemm_tflops_effective": round(flops / (step_us / 1e6) / 1e12, 1),
        "bf16_cublas_step_us": r,
        "bf16_gemms_us": {nm: dist_us([d[i] for d in d_bf]) for i, nm in
                          enumerate(["Y = X W^T", "dX = dY W", "dW = dY^T X"])},
        "speedup_over_bf16": round(r["median"] / step_us, 3),
        "note": "quantization of all three operands in both layouts included in the NVFP4 step; the bf16 step "
                "is the three GEMMs alone",
    }


def run_ours(args, world, rank, local):
    from nvfp4_microscaling_quantization_b200 import binding as N
    from nvfp4_microscaling_quantization_b200 import workloads as W

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    N.lib()
    wl = W.mlp_up(seed=4 + 1000 * rank)
    tensors = wl.tensors(device)
    stream = torch.cuda.Stream(device)
    sh = ctypes.c_void_p(stream.cuda_stream)
    calls = [Call(N, c, tensors[c.tensor], wl.seed, sh) for c in wl.calls]
    per_tensor = [TensorCalls(N, [c for c in calls if c.call.tensor == name])
                  for name in dict.fromkeys(c.tensor for c in wl.calls)]
    groups = group_step_parts(per_tensor)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    bytes_per_step = sum(BYTES_PER_ELEMENT * c.elements for c in calls)
    elems_per_step = sum(c.elements for c in calls)
    # one step = per launch group (X and W together, dY alone) its both-layout
    # pre-pass, then its both-layout quantize (both layouts from one read): 4
    # launches; the unfused step (per tensor a pre-pass, one quantize per call,
    # 9 launches) is timed too, for comparison
    body, body_names = [], []
    for grp in groups:
        for fn, kind, obj in grp.body(fused=True):
            body.append(fn)
            body_names.append((kind, obj))
    body_unfused = [fn for grp in per_tensor for fn, _, _ in grp.body(fused=False)]

    def step():
        for fn in body:
            fn()

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 0)):
            flush.zero_()
            step()
    torch.cuda.synchronize(device)
    K = args.steps

    # eager reference run (host enqueues every launch; reported, not the value)
    eager = None
    if not args.no_eager:
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        marks = [[ev() for _ in range(len(body) + 1)] for _ in range(K)]
        with torch.cuda.stream(stream):
            for k in range(K):
                flush.zero_()
                marks[k][0].record()
                for i, fn in enumerate(body):
                    fn()
                    marks[k][i + 1].record()
        torch.cuda.synchronize(device)
        e_steps = [marks[k][0].elapsed_time(marks[k][-1]) / 1e3 for k in range(K)]
        e_calls = [[marks[k][i].elapsed_time(marks[k][i + 1]) / 1e3 for k in range(K)] for i in range(len(body))]

    # the timed region: the K steps as one CUDA graph of the same C-ABI
    # launches, marks at the step boundaries only (value); then the same K
    # steps with a mark between every two launches (per-launch times, roofline)
    timer = GraphTimer(stream, body, K, flush, per_launch=False)
    inst = GraphTimer(stream, body, K, flush, per_launch=True)
    with ClockSampler(local) as clocks:
        barrier(world, local)
        torch.cuda.synchronize(device)
        timer.replay()
        torch.cuda.synchronize(device)
        barrier(world, local)
        inst.replay()
        torch.cuda.synchronize(device)
        barrier(world, local)
    clock = clocks.summary()
    totals = timer.totals()
    durs, inst_totals = inst.durations(), inst.totals()
    timer.release()
    inst.release()

    total_s = max_over_ranks(sum(totals), world, device)
    per_fn = [[durs[k][i] for k in range(K)] for i in range(len(body))]
    quant_idx = [i for i, (kind, _) in enumerate(body_names) if kind in ("quant", "dual")]
    quant_total_s = max_over_ranks(sum(sum(per_fn[i]) for i in quant_idx), world, device)
    value = weak_scaling_value(bytes_per_step, K, world, total_s)
    value_supplied = weak_scaling_value(bytes_per_step, K, world, quant_total_s)
    peak, peak_kind = hbm_peak()

    def moved_bytes(kind, obj):
        """Bytes a launch must move: a quantize reads 2 B and writes 0.5625 B
        per element; a dual quantize reads once and writes both views."""
        if kind == "quant":
            return BYTES_PER_ELEMENT * obj.elements
        if kind == "dual":
            return (PREPASS_BYTES_PER_ELEMENT + 2 * (BYTES_PER_ELEMENT - 2.0)) * obj.prepass_elements()
        return PREPASS_BYTES_PER_ELEMENT * obj.prepass_elements()

    def launch_name(kind, obj):
        if kind == "quant":
            return f"quantize {obj.call.name}"
        t = obj.label()
        return (f"quantize_dual {t} ({' + '.join(c.call.name for c in obj.dual_calls())})" if kind == "dual"
                else f"amax_{'dual' if obj.dual else 'single'} {t}")

    # dominant kernel: the quantize launch with the largest mean duration in the step
    dom_i = max(quant_idx, key=lambda i: statistics.mean(per_fn[i]))
    dom_kind, dom = body_names[dom_i]
    dom_stats = dist_us(per_fn[dom_i])
    # algorithmic bytes: 2.5625 B per element of every call the launch serves
    # (two calls for a both-layout launch); moved bytes: what it must transfer
    dom_calls = [dom] if dom_kind == "quant" else dom.dual_calls()
    dom_bytes = sum(BYTES_PER_ELEMENT * c.elements for c in dom_calls)
    dom_moved = moved_bytes(dom_kind, dom)
    achieved = dom_bytes / (dom_stats["mean"] / 1e6) / 1e9
    achieved_moved = dom_moved / (dom_stats["mean"] / 1e6) / 1e9
    src_hash = kernel_source_hash()
    traffic = NCU_TRAFFIC.get((src_hash, launch_name(dom_kind, dom)))

    per_launch = []
    for i, (kind, obj) in enumerate(body_names):
        d = dist_us(per_fn[i])
        t = d["mean"] / 1e6
        line = {"launch": launch_name(kind, obj), "us": d}
        if kind == "amax":
            line["read_gbs"] = round(moved_bytes(kind, obj) / t / 1e9, 1)
        else:
            calls_of = [obj] if kind == "quant" else obj.dual_calls()
            metric_bytes = sum(BYTES_PER_ELEMENT * c.elements for c in calls_of)
            line.update({"for_calls": [c.call.name for c in calls_of],
                         "gbs": round(metric_bytes / t / 1e9, 1),
                         "gelem_s": round(sum(c.elements for c in calls_of) / t / 1e9, 1),
                         "moved_gbs": round(moved_bytes(kind, obj) / t / 1e9, 1),
                         "frac_of_hbm_peak": round(moved_bytes(kind, obj) / t / 1e9 / peak, 4)})
        per_launch.append(line)

    unfused = None
    if not args.no_unfused:
        _, u_tot = timed_in_graph(stream, body_unfused, K, flush, device, per_launch=False)
        u_s = sum(u_tot)
        unfused = {"note": "the same step with one quantize launch per call (9 launches), CUDA graph timing",
                   "ms_per_step": {k: round(v / 1e3, 4) for k, v in dist_us(u_tot).items()},
                   "value": round(weak_scaling_value(bytes_per_step, K, 1, u_s), 1)}
    if not args.no_eager:
        eager = {"note": "the same K steps launched eagerly from Python (host enqueue in the device timeline); "
                         "not the value",
                 "ms_per_step": dist_us(e_steps), "dominant_launch_us": dist_us(e_calls[dom_i])}
        eager["ms_per_step"] = {k: round(v / 1e3, 4) for k, v in eager["ms_per_step"].items()}

    # the quantization tables first, the GEMM tables (about 1 kW) after them,
    # each with the clocks sampled while it runs
    table_clocks = {}
    per_mode = None
    if not args.no_per_mode:
        with ClockSampler(local) as ck:
            per_mode = per_mode_table(N, W, tensors["dy"], wl.seed, stream, sh, device, flush, peak)
        table_clocks["per_mode_dy"] = ck.summary()

    configs = None
    if not args.no_configs:
        with ClockSampler(local) as ck:
            configs = workload_table(N, W, stream, sh, device, flush, peak)
        table_clocks["configs"] = ck.summary()

    gemms = layer = None
    if not args.no_gemm:
        with ClockSampler(local) as ck:
            gemms = gemm_table(N, calls, stream, device)
            layer = linear_layer_table(N, per_tensor, stream, device, flush, tensors)
        table_clocks["nvfp4_gemm+linear_layer"] = ck.summary()

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, calls, tensors, stream, device, world, bytes_per_step)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = {k: v.cpu() for k, v in tensors.items()}
        cpu = cpu_baseline(wl, host, args.cpu_sample_fraction)

    step_stats = {k: round(v / 1e3, 4) for k, v in dist_us(totals).items()}
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(total_s * 1e3 / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {
            "workload": "mlp_up: one Llama-style MLP up-projection training step's tensors, "
                        "X 16384x4096 N(0,1), W 14336x4096 N(0,0.02^2), dY 16384x14336 Student-t3 std 1e-4",
            "calls": [c.call.name for c in calls],
            "path": "X and W together, then dY: one tensor-amax pre-pass for both layouts of every tensor of "
                    "the group (nvfp4_amax_dual_group), then both layouts' codes and scales from one read of each "
                    "(nvfp4_quantize_dual_group); 4 launches, C ABI, one stream",
            "timing": "the K steps captured once as one CUDA graph of the C-ABI launches (consecutive launches "
                      "adjacent, CUDA events at the step boundaries) and replayed once; per-launch times from a "
                      "second replay with an event between every two launches",
            "input_dtype": "bf16", "l2": "flushed before every timed step (256 MiB write, outside the marks)",
            "parallelism": f"replicas x{world} (independent tensors per rank)",
        },
        "gelem_per_s": round(elems_per_step * K * world / total_s / 1e9, 1),
        "frac_of_hbm_peak": round(value / world / peak, 4),
        "step_ms": step_stats,
        "step_ms_with_launch_marks": {k: round(v / 1e3, 4) for k, v in dist_us(inst_totals).items()},
        "value_amax_supplied": round(value_supplied, 1),
        "frac_of_hbm_peak_amax_supplied": round(value_supplied / world / peak, 4),
        "roofline": {"bound": "hbm", "kernel": launch_name(dom_kind, dom),
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes": int(dom_bytes),
                     "algorithmic_bytes_note": "2.5625 B per element of each call the launch serves",
                     "calls": [c.call.name for c in dom_calls],
                     "moved_bytes": int(dom_moved),
                     "moved_gbs": round(achieved_moved, 1), "frac_of_moved": round(achieved_moved / peak, 4),
                     "avg_launch_us": dom_stats["mean"], "launch_us": dom_stats},
        "per_launch": per_launch,
        "gpu_launches": sum(g.launches(fused=True) for g in groups) * K,
        "clocks": clock,
        "kernel_source": src_hash,
    }
    if eager is not None:
        result["eager"] = eager
    if unfused is not None:
        result["unfused"] = unfused
    if gemms is not None:
        result["nvfp4_gemm"] = gemms
    if layer is not None:
        result["linear_layer"] = layer
    if table_clocks:
        result["table_clocks"] = table_clocks
    if per_mode is not None:
        result["per_mode_dy"] = per_mode
    if configs is not None:
        result["configs"] = configs
    if e2e is not None:
        result["e2e"] = e2e
    if cpu is not None:
        result["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_e2e(args, calls, tensors, stream, device, world, bytes_per_step):
    """Same step through the public API with host buffers: pinned H2D of the step's
    inputs, the six calls, D2H of every output, all inside the timed region.

    Steps are pipelined the way a caller streaming tensors would run them: the
    host-to-device copies (one stream) of step i overlap the kernels (a second
    stream) of step i-1 and the device-to-host copies (a third) of step i-1;
    inputs and outputs are double-buffered, so a step's copies never overwrite
    what the previous step's kernels still read or its outputs still hold."""
    N = calls[0].N
    s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    sh = ctypes.c_void_p(s_comp.cuda_stream)
    inputs = [tensors, {k: torch.empty_like(v) for k, v in tensors.items()}]
    sets = [[Call(N, c.call, inputs[b][c.call.tensor], c.seed, sh) for c in calls] for b in range(2)]
    group_sets = [group_step_parts([TensorCalls(N, [c for c in cs if c.call.tensor == name])
                                    for name in dict.fromkeys(c.call.tensor for c in cs)]) for cs in sets]
    host_in = {k: v.cpu().pin_memory() for k, v in tensors.items()}
    host_out = [(torch.empty(c.codes.shape, dtype=torch.uint8).pin_memory(),
                 torch.empty(c.scales.shape, dtype=torch.uint8).pin_memory(),
                 torch.empty(1, dtype=torch.float32).pin_memory()) for c in calls]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(c.output_bytes() for c in calls)

    def run(K):
        ev = {k: [torch.cuda.Event() for _ in range(K)] for k in ("in", "comp", "out")}
        for i in range(K):
            b = i % 2
            if i >= 2:
                s_in.wait_event(ev["comp"][i - 2])   # input set b is free once step i-2's kernels are done
            with torch.cuda.stream(s_in):
                for k, t in inputs[b].items():
                    t.copy_(host_in[k], non_blocking=True)
            ev["in"][i].record(s_in)
            s_comp.wait_event(ev["in"][i])
            if i >= 2:
                s_comp.wait_event(ev["out"][i - 2])  # output set b copied out
            for grp in group_sets[b]:
                for fn, _, _ in grp.body(fused=True):
                    fn()
            ev["comp"][i].record(s_comp)
            s_out.wait_event(ev["comp"][i])
            with torch.cuda.stream(s_out):
                for c, (hc, hs, hg) in zip(sets[b], host_out):
                    hc.copy_(c.codes, non_blocking=True)
                    hs.copy_(c.scales, non_blocking=True)
                    hg.copy_(c.gscale, non_blocking=True)
            ev["out"][i].record(s_out)

    run(2)
    torch.cuda.synchronize(device)
    K = max(args.e2e_steps if args.e2e_steps is not None else args.steps, 1)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device.index)
    torch.cuda.synchronize(device)
    start.record(s_in)
    run(K)
    end.record(s_out)
    torch.cuda.synchronize(device)
    barrier(world, device.index)
    secs = max_over_ranks(start.elapsed_time(end) / 1e3, world, device)
    return {"value": round(weak_scaling_value(bytes_per_step, K, world, secs), 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K,
            "ms_per_step": round(secs * 1e3 / K, 3),
            "pipeline": "H2D of step i || kernels and D2H of step i-1, inputs and outputs double-buffered"}


# ------------------------------------------------------------------------ CPU oracle
def _sample_calls(wl, host, fraction):
    """For every call, the sub-tensor holding the first `fraction` of its view rows."""
    from nvfp4_microscaling_quantization_b200 import workloads as W
    out = []
    for c in wl.calls:
        x = host[c.tensor]
        rows, cols = x.shape
        if c.layout == W.ROWWISE:
            n = max(1, int(rows * fraction))
            sub = x[:n]
        else:
            n = max(8, int(cols * fraction) // 8 * 8)
            sub = x[:, :n]
        out.append((c, W.bf16_bits(sub.contiguous())))
    return out


def time_oracle_sample(wl, samples, pool):
    """The oracle on every sampled call: its amax pre-pass, then the quantization,
    each split over the pool's worker processes by view rows."""
    elements = 0
    t0 = time.perf_counter()
    for c, xb in samples:
        a = pool.amax(xb, c.layout, c.rht_group, wl.seed)
        pool.quantize(xb, c.layout, c.mode, c.rht_group, wl.seed, a)
        elements += xb.size
    return elements, time.perf_counter() - t0


def cpu_baseline(wl, host, fraction):
    from oracle.pool import OraclePool
    samples = _sample_calls(wl, host, fraction)
    with OraclePool() as pool:
        elements, secs = time_oracle_sample(wl, samples, pool)
        cores = pool.workers
    return {"value": round(BYTES_PER_ELEMENT * elements / secs / 1e9, 4), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"first {fraction:.4g} of the view rows of each of the {len(samples)} calls "
                      f"({elements} elements, amax pre-pass + quantize), the single-threaded C oracle run on "
                      f"ranges of view rows in {cores} processes (one per host core), {secs:.1f} s"}


def run_reference(args, world, rank, wl=None, fraction=1.0 / 64):
    """The CPU oracle as the reference arm, on rank 0 only (the other ranks return at once)."""
    if rank != 0:
        return None
    from oracle.pool import OraclePool
    from nvfp4_microscaling_quantization_b200 import workloads as W
    wl = W.mlp_up(seed=4) if wl is None else wl
    # the worker processes start (spawn) before this process touches a GPU
    with OraclePool() as pool:
        device = "cuda" if torch.cuda.is_available() else "cpu"
        full = wl.tensors(device)
        host = {k: v.cpu() for k, v in full.items()}
        del full
        samples = _sample_calls(wl, host, fraction)
        for _ in range(max(args.warmup, 0)):
            time_oracle_sample(wl, samples, pool)
        total_e, total_s = 0, 0.0
        for _ in range(args.steps):
            e, s = time_oracle_sample(wl, samples, pool)
            total_e += e
            total_s += s
        cores = pool.workers
    value = BYTES_PER_ELEMENT * total_e / total_s / 1e9
    sample = (f"each step: first {fraction:.4g} of the view rows of each of the {wl.name} calls "
              f"({total_e // max(args.steps, 1)} elements, amax pre-pass + quantize), the single-threaded C "
              f"oracle on ranges of view rows in {cores} processes")
    line = json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_s * 1e3 / max(args.steps, 1), 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{wl.name} (bounded sample per step)", "input_dtype": "bf16"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    })
    print(line, flush=True)
    return line


def run_profile_case(args):
    """A small, self-contained run of the step's kernels on one tensor, for ncu
    captures that must stay within a few GB: a Student-t3 (std 1e-4) tensor of
    the given shape, and per iteration its dual pre-pass, its dual quantize
    (MS-EDEN both ways, and RTN rows + MS-EDEN columns), the single-layout
    quantizes (MS-EDEN g = 128 both layouts, RTN row-wise, and row-wise in the
    modes of --profile-modes without rotation and with g = 128), and the NVFP4
    GEMM of the RTN row-wise quantization with itself."""
    from nvfp4_microscaling_quantization_b200 import binding as N
    from nvfp4_microscaling_quantization_b200 import workloads as W
    rows, cols = (int(v) for v in args.profile_case.lower().split("x"))
    device = torch.device("cuda", 0)
    g = torch.Generator(device=device)
    g.manual_seed(11)
    x = W.student_t3((rows, cols), 1e-4, g)
    stream = torch.cuda.Stream(device)
    sh = ctypes.c_void_p(stream.cuda_stream)
    calls = {(lay, mode, grp): Call(N, W.Call("p", lay, mode, grp), x, 11, sh)
             for lay, mode, grp in [(W.ROWWISE, W.MS_EDEN, 128), (W.TRANSPOSED, W.MS_EDEN, 128),
                                    (W.ROWWISE, W.RTN, 0)]}
    by_name = {name: mode for mode, name in W.MODE_NAMES.items()}
    for name in filter(None, args.profile_modes.split(",")):
        for grp in (0, 128):
            calls[(W.ROWWISE, by_name[name], grp)] = Call(N, W.Call("p", W.ROWWISE, by_name[name], grp), x, 11, sh)
    eden = TensorCalls(N, [calls[(W.ROWWISE, W.MS_EDEN, 128)], calls[(W.TRANSPOSED, W.MS_EDEN, 128)]])
    mixed = TensorCalls(N, [calls[(W.ROWWISE, W.RTN, 0)], calls[(W.TRANSPOSED, W.MS_EDEN, 128)]])
    body = [("amax_dual eden", eden.amax_passes), ("quantize_dual eden", eden.quantize_dual),
            ("amax_dual mixed", mixed.amax_passes), ("quantize_dual mixed", mixed.quantize_dual)]
    body += [(f"quantize {c.call.name}", c.quantize) for c in calls.values()]
    # one NVFP4 GEMM of the RTN row-wise quantization with itself (P P^T)
    rq = calls[(W.ROWWISE, W.RTN, 0)]
    d = torch.empty(rows, rows, dtype=torch.bfloat16, device=device)
    body.append(("gemm P P^T", lambda: N.gemm((rq.codes, rq.scales, rq.gscale), (rq.codes, rq.scales, rq.gscale),
                                               out=d, stream=stream)))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    times = {name: [] for name, _ in body}
    with torch.cuda.stream(stream):
        for c in calls.values():  # every call's own tensor amax (the extra modes have no dual pre-pass)
            c.amax_pass()
        for _, fn in body:        # first launches (module loading) outside the timing
            fn()
        torch.cuda.synchronize(device)
        for _ in range(max(args.steps, 1)):
            for name, fn in body:
                flush.zero_()
                a, b = ev(), ev()
                a.record()
                fn()
                b.record()
                b.synchronize()
                times[name].append(a.elapsed_time(b) * 1e3)
    torch.cuda.synchronize(device)
    print(json.dumps({"profile_case": [rows, cols], "launch_us_median": {k: round(statistics.median(v), 2)
                                                                         for k, v in times.items()}}), flush=True)


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_env()
    if args.profile_case:
        run_profile_case(args)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl ours needs a CUDA GPU")
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
