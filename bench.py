"""Benchmark of the SmoothQuant W8A8 int8 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill]
                    [--path smoothquant|forward|forward-prologue|per-tensor|ste-train|weight-only]
                    [--serial]
                    [--impl ours|reference] [--no-e2e] [--no-cpu-baseline]

A step is one pass of the whole path over one batch of seeded synthetic input:
calibration (column max-abs of the calibration batch and of W, smoothing
factor s), weight fold + int8 quantisation, per-token activation quantisation
and the int8 tcgen05 GEMM with its dequant + bias epilogue.  The default
workload is the largest layer, the prefill GEMM: X[8192x8192] bf16 with 41
outlier channels x100, W[28672x8192] bf16 ~N(0,0.01), no bias, alpha 0.5,
calibration batch of 512 rows.  `--workload tiny|proj|mlp|decode` selects the
other layer shapes.

Paths (`--path`):
  smoothquant  the whole path above (default, except for decode);
  forward      the per-call path once the weight is prepared: sq_forward on
               pre-quantised weights (default for decode: every call streams
               the 64 MiB of int8 W from HBM -- the calls rotate over enough
               prepared weight copies, >= 256 MiB, that L2 cannot serve them);
  forward-prologue
               the same per-call forward through sq_forward_prologue, whose
               GEMM quantises X itself (codes written straight into the
               tensor core's shared-memory operand after a scale pre-pass);
  per-tensor   one scale per tensor for W and X, then the int8 GEMM;
  ste-train    s from the running max, the forward, and the straight-through
               backward to X, W, bias and eta_alpha of a seeded dL/dY;
  weight-only  W quantised per output channel with s = 1, bf16 activations.

Timing.  Whole steps (all paths but forward): every step is preceded by an L2
flush (a 256 MiB write, then a 512 MiB read, so that L2 holds neither the
step's inputs nor dirty lines whose write-back would land inside the timed
step); the step's calls are captured as one CUDA graph with timing-event
nodes before and after it; the kernels overlap each other's launch through
programmatic dependent launch, and calls that depend only on earlier calls
(the weight prep and the activation quantiser both need s alone) run on
forked streams (`--serial` captures them in order).  The forward path captures
the K timed calls as one graph between two event nodes (the span / K is the
step time), each call on the next weight copy of the rotation.

Per call (the roofline and the `kernels` breakdown): a graph of back-to-back
launches of that call between two event nodes, replayed after the L2 flush;
consecutive launches take their inputs from different copies (a rotation whose
copies add up to at least 256 MiB, twice the L2), so every launch reads its
inputs from HBM.  The span / launches is the call's duration; a graph with
event nodes between single calls gives `ms_single_launch`.  On the forward
paths the timed region is itself such a run of the call (K launches on the
rotation), so its mean launch duration is the call's duration there
(`ms_short_run` keeps the REPS-launch figure).  With N > 1 (one
process per GPU under torchrun) every rank runs an independent replica (the
layer shards by tokens with no exchange): the value is the tokens all ranks
processed divided by the slowest rank's time.

The JSON line adds: `e2e` (the same step through the Python binding with the
inputs copied from pinned host memory and Y copied back, every step),
`roofline` of the dominant call, `cpu_baseline` (the CPU oracle timed on a
bounded sample, rank 0 only), sampled `clocks`, and per-call `kernels` times.
`--impl reference` times the CPU oracle itself as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "W8A8 linear int8 TOPS & tokens/s at 1 B200; % of INT8 tensor peak / HBM roofline"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20        # written before each step
FLUSH_READ_BYTES = 512 << 20   # then read, leaving L2 clean
L2_BYTES = 126 << 20
ROTATE_BYTES = 256 << 20       # inputs of a rotation add up to at least this (2x L2)
MAX_ROTATION = 128             # copies at most (tiny inputs stay partly L2-resident)
# fallback peaks (only if MEASURED_PEAKS.json is absent)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_OVER_BF16 = 2.0  # nominal dense int8 / bf16 ratio (4.5 / 2.25 PFLOP/s)
# fp32 multiply-add peak of the CUDA cores: 148 SMs x 128 lanes x 2 flops x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
PATHS = ["smoothquant", "forward", "forward-prologue", "per-tensor", "ste-train", "weight-only"]
# the per-call forward paths and the call each one times
FORWARD_CALLS = {"forward": "sq_forward", "forward-prologue": "sq_forward_prologue"}
# sq_forward fuses the activation quantisation into the weight-streaming
# kernel up to this many tokens (one launch), else runs the quantiser first
FORWARD_FUSED_MAX_M = 8


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default=None, choices=PATHS,
                    help="smoothquant: the whole path (default); forward: sq_forward on prepared weights "
                         "(default for decode); forward-prologue: sq_forward_prologue (the GEMM quantises "
                         "X itself) on prepared weights; per-tensor: the baseline W8A8 path (one scale per tensor); "
                         "ste-train: a learnable-alpha training step (s from the running max, forward, "
                         "straight-through backward); weight-only: the int8 weight-only comparison")
    ap.add_argument("--serial", action="store_true",
                    help="capture the step's calls strictly in order (by default calls that depend only on "
                         "earlier stages run on forked streams)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--settle-s", type=float, default=1.0,
                    help="untimed replays after warm-up until this much wall time has passed (clock sampling)")
    args = ap.parse_args(argv)
    if args.path is None:
        args.path = default_path(args.workload)
    return args


def default_path(workload_name):
    """The decode layer is timed as a per-call layer on prepared weights."""
    return "forward" if workload_name == "decode" else "smoothquant"


def metric_for(path):
    if path == "ste-train":
        return ("learnable-alpha W8A8 training step (forward + relative-MSE auxiliary loss + straight-through "
                "backward) tokens/s at 1 B200")
    return METRIC


def workload_config(wl, path="smoothquant"):
    c = {
        "workload": f"{wl.name}: X[{wl.M}x{wl.K}] W[{wl.N}x{wl.K}] bf16, alpha {wl.alpha_f32:g}, "
                    f"{wl.outliers} outlier channels x{wl.outlier_scale:g}, calibration {wl.R} rows, "
                    f"{'bias' if wl.has_bias else 'no bias'}",
        "M": wl.M, "N": wl.N, "K": wl.K, "R": wl.R,
        "l2": "flushed before every timed step (256 MiB write, then 512 MiB read)",
    }
    if path == "per-tensor":
        c["workload"] = "per-tensor W8A8 baseline (one scale per tensor), " + c["workload"]
    elif path == "weight-only":
        c["workload"] = ("int8 weight-only comparison (W quantised per output channel with s = 1, activations "
                         "bf16), " + c["workload"])
    elif path == "ste-train":
        c["workload"] = ("learnable-alpha training step (s from the running max of the calibration batch, "
                         "forward, relative-MSE auxiliary loss against the unquantised output with weight "
                         f"{AUX_WEIGHT:g} folded into a seeded bf16 dL/dY, straight-through backward), "
                         + c["workload"])
    elif path in FORWARD_CALLS:
        what = ("sq_forward: activation quantisation + int8 GEMM + epilogue" if path == "forward" else
                "sq_forward_prologue: scale pre-pass + int8 GEMM that quantises X in its prologue + epilogue")
        c["workload"] = (f"per-call forward on pre-quantised weights ({what}; calibration and weight prep done "
                         "once, untimed), " + c["workload"])
        c["l2"] = (f"calls rotate over {forward_rotation(wl)} prepared weight copies "
                   f"({forward_rotation(wl) * wl.N * wl.K / 2**20:.0f} MiB of int8 W), so every call streams "
                   f"its weight from HBM")
    return c


def forward_rotation(wl):
    """Prepared weight copies the forward path rotates over (>= 4, >= 256 MiB)."""
    return max(4, min(MAX_ROTATION, -(-ROTATE_BYTES // (wl.N * wl.K + 4 * wl.N))))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, None, "fallback"


def algorithmic_work(wl):
    """Per call: (minimum HBM bytes per launch, tensor ops per launch or 0,
    their operand type)."""
    M, N, K, R = wl.M, wl.N, wl.K, wl.R
    work = {
        "sq_calibrate": (2 * R * K + 2 * N * K + 8 * K, 0),
        "sq_prepare_weight": (3 * N * K + 4 * N + 4 * K, 0),
        "sq_quantize_act": (3 * M * K + 4 * M + 4 * K, 0),
        "sq_linear": (M * K + N * K + 2 * M * N + 4 * M + 4 * N, 2 * M * N * K),
        # X in (bf16), s, the codes and scales of W in, Y out; the codes of X
        # need not leave the chip
        "sq_forward": (2 * M * K + 4 * K + N * K + 4 * N + 2 * M * N, 2 * M * N * K),
        "sq_forward_prologue": (2 * M * K + 4 * K + N * K + 4 * N + 2 * M * N, 2 * M * N * K),
        # one scale per tensor: the data once in, the codes and the scale row out
        "sq_quantize_per_tensor(W)": (3 * N * K + 4 * N, 0),
        "sq_quantize_per_tensor(X)": (3 * M * K + 4 * M, 0),
        # s from the running max alone: W read, mx read, s written
        "sq_calibrate(mx)": (2 * N * K + 8 * K, 0),
        # G, X, W, Xq, Wq and the scales in; dX, dW (fp32), db, ds out; two
        # contractions of 2MNK each (counted once, whatever the kernel's split)
        "sq_ste_backward": (2 * M * N + 7 * M * K + 7 * N * K + 8 * M + 12 * N + 12 * K, 4 * M * N * K),
        # two passes: Y_fp and Y_q for the sums, then Y_fp, Y_q and G in, G out
        "sq_rel_mse": (12 * M * N + 8, 0),
        # X (bf16) and the codes in, Y out; 2MNK multiply-add operations on the fp32 CUDA cores
        "sq_linear_weight_only": (2 * M * K + N * K + 4 * N + 2 * M * N, 2 * M * N * K),
    }
    typ = {"sq_ste_backward": "bf16", "sq_linear_weight_only": "fp32-alu"}
    return {n: (b, o, typ.get(n, "int8")) for n, (b, o) in work.items()}


# Per-call kernel durations are spans over at least this many back-to-back launches.
REPS = 8

# A kernel running this long sits in a power-capped stretch of work: its
# tensor roofline is the sustained cuBLAS figure rather than the burst one.
SUSTAINED_AFTER_MS = 0.5


def source_sha(files=None):
    """Hash of the kernel sources (all of csrc/, or the listed files of it)."""
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "w8a8_smoothquant_int8_sq_b200", "csrc")
    for f in sorted(files if files else os.listdir(cs)):
        h.update(open(os.path.join(cs, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_call, wl_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
    except Exception:
        return None
    e = d.get(wl_name, {}).get(kernel_call)
    if not e or e.get("source_sha") != source_sha(e.get("sources")):
        return None
    return e.get("dram_bytes_per_launch")


def rotation_count(footprint_bytes):
    """Input copies that make back-to-back launches read from HBM: their
    inputs add up to at least ROTATE_BYTES (at most MAX_ROTATION copies)."""
    if footprint_bytes <= 0:
        return 1
    return int(max(1, min(MAX_ROTATION, -(-ROTATE_BYTES // footprint_bytes))))


# ------------------------------------------------------------- multi-rank
def max_over_ranks(x: float, world: int, device) -> float:
    """The largest value of x over all ranks (for times: the slowest rank).
    With one process per GPU the replicas run independently; this is the only
    collective, and it carries a single number."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def step_stats(times_ms):
    """(mean, median) of the timed steps' device times in ms."""
    t = np.asarray(times_ms, dtype=np.float64)
    return float(t.mean()), float(np.median(t))


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units processed by all ranks per second, over the slowest rank's time."""
    return units_per_rank * world / (ms * 1e-3)


# ------------------------------------------------------------------- clocks
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                rows.append(dict(sm=float(f[1]), max=float(f[2]), power=float(f[3]), util=float(f[4]),
                                 hw=f[6], hwt=f[7], swt=f[8], pcap=f[9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [r for r in rows if r["util"] > 0] or rows
        reasons = set()
        for r in load:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                            ("pcap", "sw_power_cap")):
                if r[k].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r["sm"] for r in load])), "sm_max_mhz": load[0]["max"],
                "reasons": sorted(reasons), "samples": len(load),
                "power_w_max": max(r["power"] for r in load)}


# --------------------------------------------------------------- CPU oracle
# Largest whole step the CPU legs run; beyond it the smoothquant step is timed
# on a sample of rows and extrapolated phase by phase.
WHOLE_STEP_MAX_MNK = 1.0e11
WHOLE_STEP_MAX_NK = 64 << 20
SAMPLE_X_ROWS = 256
SAMPLE_W_ROWS = 4096


def sample_plan(wl, path):
    """(rows of X, rows of W) the oracle's step runs on: all of them for the
    smaller layers, a seeded-input prefix for the prefill layer (whole path
    and per-call forward)."""
    if (path != "smoothquant" and path not in FORWARD_CALLS) or (wl.M * wl.N * wl.K <= WHOLE_STEP_MAX_MNK and
                                                                   wl.N * wl.K <= WHOLE_STEP_MAX_NK):
        return wl.M, wl.N
    return min(wl.M, SAMPLE_X_ROWS), min(wl.N, SAMPLE_W_ROWS)


def oracle_inputs(wl, path, inp=None):
    """The seeded inputs of `wl` (or a copy of `inp`) plus what the path's
    untimed set-up needs."""
    inp = dict(workloads.make_inputs(wl) if inp is None else inp)
    if path == "ste-train":
        inp["G"] = train_gradient(wl)
        inp["Yfp"] = unquantised_output(wl, inp)
    if path in FORWARD_CALLS:
        # the weight is prepared once, outside the timed calls (as on the GPU)
        from oracle import smoothquant as O
        s, _ = O.calibrate(inp["C"], inp["W"], wl.alpha_f32)
        inp["s"] = s
        # the rows of W the (possibly sampled) forward multiplies by
        inp["Wq"], inp["ws"] = O.fold_and_quantize_weight(inp["W"][:sample_plan(wl, path)[1]], s)
    return inp


def oracle_step_seconds(inp, wl, path="smoothquant"):
    """Seconds the oracle takes for one whole step of `path` on `wl`.

    For the prefill layer the smoothquant step is timed on a sample and
    extrapolated per phase, each phase linear in what it processes:
    calibration in full (it reads all of C and W); the weight fold +
    quantisation on the first m_w rows of W (x N / m_w); the activation
    quantisation on the first m_x rows of X (x M / m_x); the int8 product and
    the epilogue on that m_x x m_w block (x M N / (m_x m_w))."""
    from oracle import smoothquant as O
    pc = time.perf_counter
    if path == "ste-train":
        from oracle import ste_backward as STE
        t0 = pc()
        mx = O.column_max_abs(O.widen_bf16(inp["C"]))
        s, _ = O.calibrate(inp["C"][:0], inp["W"], wl.alpha_f32, mx_prev=mx)
        Wq, ws = O.fold_and_quantize_weight(inp["W"], s)
        Yq = O.forward(inp["X"], s, Wq, ws, inp["bias"])[0]
        from oracle import aux_loss as AUX
        AUX.rel_mse(inp["Yfp"], Yq)
        Gt = AUX.add_aux_grad(inp["G"], inp["Yfp"], Yq, AUX_WEIGHT)
        STE.ste_backward(Gt, inp["X"], inp["W"], mx, wl.alpha_f32)
        return pc() - t0
    if path == "weight-only":
        from oracle import weight_only as WO
        t0 = pc()
        Wq, ws = O.fold_and_quantize_weight(inp["W"], np.ones(wl.K, np.float32))
        WO.weight_only_linear(inp["X"], Wq, ws, inp["bias"])
        return pc() - t0
    if path == "per-tensor":
        from oracle import per_tensor as PT
        t0 = pc()
        PT.linear_per_tensor(inp["X"], inp["W"], inp["bias"])
        return pc() - t0
    if path in FORWARD_CALLS:
        # quantisation of X, then product + epilogue (on the sampled block for
        # the prefill layer, each phase scaled by what it covers)
        mx_rows, mw_rows = sample_plan(wl, path)
        b = inp["bias"]
        t0 = pc()
        Xq, xs = O.quantize_activation(inp["X"][:mx_rows], inp["s"])
        t1 = pc()
        acc = O.int8_gemm(Xq, inp["Wq"][:mw_rows])
        O.dequant_epilogue(acc, xs, inp["ws"][:mw_rows], None if b is None else b[:mw_rows])
        t2 = pc()
        return (t1 - t0) * wl.M / mx_rows + (t2 - t1) * (wl.M * wl.N) / (mx_rows * mw_rows)
    mx_rows, mw_rows = sample_plan(wl, path)
    b = inp["bias"]
    t0 = pc()
    s, _ = O.calibrate(inp["C"], inp["W"], wl.alpha_f32)
    t1 = pc()
    Wq, ws = O.fold_and_quantize_weight(inp["W"][:mw_rows], s)
    t2 = pc()
    Xq, xs = O.quantize_activation(inp["X"][:mx_rows], s)
    t3 = pc()
    acc = O.int8_gemm(Xq, Wq)
    O.dequant_epilogue(acc, xs, ws, None if b is None else b[:mw_rows])
    t4 = pc()
    return ((t1 - t0) + (t2 - t1) * wl.N / mw_rows + (t3 - t2) * wl.M / mx_rows
            + (t4 - t3) * (wl.M * wl.N) / (mx_rows * mw_rows))


def oracle_sample_text(wl, path):
    mx_rows, mw_rows = sample_plan(wl, path)
    what = {"per-tensor": "quantise W and X per tensor, product",
            "weight-only": "quantise W per output channel, bf16 x int8 product",
            "ste-train": "s from the running max, fold+quantise W, forward, auxiliary loss, straight-through backward",
            "forward": "forward on the prepared weight: quantise X, int8 product, epilogue",
            "forward-prologue": "forward on the prepared weight: quantise X, int8 product, epilogue",
            "smoothquant": "calibrate, fold+quantise W, quantise X, int8 product, epilogue"}[path]
    if (mx_rows, mw_rows) == (wl.M, wl.N):
        return f"whole {wl.name} steps ({what})"
    if path in FORWARD_CALLS:
        return (f"{wl.name} calls ({what}) timed on a sample and extrapolated per phase: activation quantisation "
                f"on {mx_rows} of {wl.M} X rows, product + epilogue on the {mx_rows}x{mw_rows} block (each phase "
                f"scaled by the rows it covers)")
    return (f"{wl.name} steps ({what}) timed on a sample and extrapolated per phase: calibration in full, "
            f"weight prep on {mw_rows} of {wl.N} W rows, activation quantisation on {mx_rows} of {wl.M} X rows, "
            f"product + epilogue on the {mx_rows}x{mw_rows} block (each phase scaled by the rows it covers)")


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def train_gradient(wl):
    """Seeded synthetic dL/dY [M, N] (bf16 bits) for the training step."""
    return workloads.random_bf16((wl.M, wl.N), seed=1000 * wl.index + 9, scale=1e-3)


# weight of the relative-MSE auxiliary loss in the training step's total loss
AUX_WEIGHT = 1.0


def unquantised_output(wl, inp):
    """Y_fp = X W^T + b of the unquantised layer (bf16 bits, one rounding from
    float64): the reference output the auxiliary loss compares with."""
    from oracle import smoothquant as O
    return O.bf16_round(O.reference_linear_f64(inp["X"], inp["W"], inp["bias"]))


def cpu_oracle_rate(wl, seconds, path="smoothquant", inp=None):
    """Tokens/s of the oracle on (extrapolated) whole steps, run until `seconds`
    of CPU work have passed.  Returns (rate, steps, seconds of work)."""
    inp = oracle_inputs(wl, path, inp)
    oracle_step_seconds(inp, wl, path)  # warm (page-in, BLAS threads)
    n, work, t0 = 0, 0.0, time.perf_counter()
    ext = 0.0
    while True:
        ext += oracle_step_seconds(inp, wl, path)
        n += 1
        work = time.perf_counter() - t0
        if work >= seconds:
            break
    return wl.M * n / ext, n, work


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    path = getattr(args, "path", "smoothquant") or default_path(wl.name)
    inp = oracle_inputs(wl, path)
    for _ in range(args.warmup):
        oracle_step_seconds(inp, wl, path)
    ext, t0 = 0.0, time.perf_counter()
    for _ in range(args.steps):
        ext += oracle_step_seconds(inp, wl, path)
    work = time.perf_counter() - t0
    v = wl.M * args.steps / ext
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": metric_for(path), "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * ext / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64+fp32 (numpy)",
        "data": "synthetic", "config": workload_config(wl, path),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} {oracle_sample_text(wl, path)}; {work:.1f} s of CPU work"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------------- GPU arm
def kernel_report(wl, names, per_call, per_call_single, launches_per_call, rotations=None):
    """Per-call roofline figures and the roofline object of the longest call."""
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_kind = peaks()
    work = algorithmic_work(wl)
    kernels = {}
    for n in names:
        nbytes, ops, op_type = work[n]
        ms = per_call[n]
        sustained = ms >= SUSTAINED_AFTER_MS and bf16_tf_sus is not None
        int8_peak_tops = (bf16_tf_sus if sustained else bf16_tf) * (INT8_OVER_BF16 if op_type == "int8" else 1.0)
        if op_type == "fp32-alu":
            int8_peak_tops = FP32_ALU_TFLOPS
        # the bound is whichever roofline takes longer for this call's work
        t_hbm = nbytes / (hbm_gbs * 1e9)
        t_tensor = ops / (int8_peak_tops * 1e12)
        if t_hbm >= t_tensor:
            ach = nbytes / (ms * 1e-3) / 1e9
            kernels[n] = {"ms": ms, "ms_single_launch": per_call_single[n], "bound": "hbm",
                          "algorithmic_bytes": nbytes, "achieved_gbs": ach,
                          "frac_of_measured_hbm": ach / hbm_gbs, "launches": launches_per_call[n]}
        else:
            ach = ops / (ms * 1e-3) / 1e12
            kernels[n] = {"ms": ms, "ms_single_launch": per_call_single[n], "bound": "tensor", "int8_ops": ops,
                          "achieved_tops": ach,
                          "int8_peak_tops": int8_peak_tops, "frac_of_int8_peak": ach / int8_peak_tops,
                          "peak": "sustained" if sustained else "burst", "launches": launches_per_call[n]}
            if op_type != "int8":
                kernels[n]["operands"] = op_type
            if op_type == "fp32-alu":
                kernels[n]["bound"] = "alu"
        if rotations is not None and n in rotations:
            kernels[n]["input_copies"], kernels[n]["l2_cold"] = rotations[n]
    dom = max(names, key=lambda n: per_call[n])
    kd = kernels[dom]
    if kd["bound"] == "alu":
        roof = {"bound": "alu", "achieved": kd["achieved_tops"], "peak": kd["int8_peak_tops"], "unit": "TFLOP/s",
                "frac": kd["achieved_tops"] / kd["int8_peak_tops"],
                "peak_source": "fp32 FMA peak of the CUDA cores from unit counts and the 1965 MHz clock"}
    elif kd["bound"] == "hbm":
        roof = {"bound": "hbm", "achieved": kd["achieved_gbs"], "peak": hbm_gbs, "unit": "GB/s",
                "frac": kd["achieved_gbs"] / hbm_gbs}
        roof["peak_source"] = f"{peak_kind} HBM copy"
    else:
        roof = {"bound": "tensor", "achieved": kd["achieved_tops"], "peak": kd["int8_peak_tops"], "unit": "TFLOP/s",
                "frac": kd["achieved_tops"] / kd["int8_peak_tops"]}
        roof["peak_source"] = (f"{peak_kind} cuBLAS bf16 {kd['peak']}" if kd.get("operands") == "bf16" else
                               f"{peak_kind} cuBLAS bf16 {kd['peak']} x2 (nominal dense int8/bf16 ratio)")
    roof["kernel"] = dom
    roof["traffic"] = ncu_traffic(dom, wl.name)
    return kernels, roof


class Call:
    """One library call of the step: fn(T) enqueues it with the tensors of T;
    `reads` names the tensors of T it reads from HBM (copied for the rotation
    of the per-call timing); `launches` is its number of kernels."""

    def __init__(self, fn, reads, launches):
        self.fn, self.reads, self.launches = fn, reads, launches


def nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def run_ours(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import w8a8_smoothquant_int8_sq_b200 as sq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    inp = workloads.make_inputs(wl)

    def d(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    K, N, M = wl.K, wl.N, wl.M
    T = {"C": d(inp["C"]), "W": d(inp["W"]), "X": d(inp["X"]),
         "b": d(inp["bias"]) if inp["bias"] is not None else None,
         "s": torch.empty(K, dtype=torch.float32, device=dev),
         "Wq": torch.empty(N, K, dtype=torch.int8, device=dev),
         "w_scale": torch.empty(N, dtype=torch.float32, device=dev),
         "Xq": torch.empty(M, K, dtype=torch.int8, device=dev),
         "x_scale": torch.empty(M, dtype=torch.float32, device=dev),
         "Y": torch.empty(M, N, dtype=torch.bfloat16, device=dev),
         "ws_cal": torch.empty(sq.sq_calibrate_workspace_bytes(K), dtype=torch.uint8, device=dev),
         "ws_fwd": torch.empty(max(sq.sq_forward_workspace_bytes(M, N, K), 16), dtype=torch.uint8, device=dev),
         "ws_pro": torch.empty(max(sq.sq_forward_prologue_workspace_bytes(M, K), 16), dtype=torch.uint8,
                               device=dev),
         "ws_lin": torch.empty(max(sq.sq_workspace_bytes(M, N, K), 16), dtype=torch.uint8, device=dev)}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_read = torch.ones(FLUSH_READ_BYTES // 4, dtype=torch.int32, device=dev)
    a = wl.alpha_f32
    fwd_launches = 1 if M <= FORWARD_FUSED_MAX_M else 2

    if args.path == "weight-only":
        T["ones"] = torch.ones(K, dtype=torch.float32, device=dev)
        calls = {
            "sq_prepare_weight": Call(lambda T: sq.sq_prepare_weight(T["W"], T["ones"], Wq=T["Wq"],
                                                                     w_scale=T["w_scale"]), ["W"], 1),
            "sq_linear_weight_only": Call(lambda T: sq.sq_linear_weight_only(T["X"], T["Wq"], T["w_scale"], T["b"],
                                                                             Y=T["Y"]),
                                          ["X", "Wq", "w_scale", "b"], 1),
        }
        stages = [["sq_prepare_weight"], ["sq_linear_weight_only"]]
    elif args.path == "ste-train":
        # the training step of the learnable-alpha layer: s recomputed from the
        # running activation max (taken once from the calibration batch) and
        # the weight, the forward, the relative-MSE auxiliary loss against the
        # unquantised output folded into dL/dY, and the straight-through
        # backward.  Y_fp (the unquantised layer, an input of the step like G)
        # is formed once by the set-up.
        T["G"] = d(train_gradient(wl))
        T["Yfp"] = d(unquantised_output(wl, inp))
        T["Gt"] = torch.empty_like(T["G"])
        T["aux_loss"] = torch.empty(1, dtype=torch.float64, device=dev)
        T["ws_aux"] = torch.empty(sq.sq_rel_mse_workspace_bytes(), dtype=torch.uint8, device=dev)
        T["mx"] = torch.zeros(K, dtype=torch.float32, device=dev)
        sq.sq_calibrate(T["C"], T["W"], a, s=T["s"], mx_inout=T["mx"], workspace=T["ws_cal"])
        T.update(dXg=torch.empty(M, K, dtype=torch.float32, device=dev),
                 dWg=torch.empty(N, K, dtype=torch.float32, device=dev),
                 dbg=torch.empty(N, dtype=torch.float32, device=dev) if T["b"] is not None else None,
                 dsg=torch.empty(K, dtype=torch.float32, device=dev),
                 d_eta=torch.empty(1, dtype=torch.float32, device=dev),
                 ws_bwd=torch.empty(sq.sq_ste_backward_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev))

        def bwd(T):
            sq.sq_ste_backward(T["Gt"], T["X"], T["W"], T["s"], T["mx"], a, T["Xq"], T["x_scale"], T["Wq"],
                               T["w_scale"], with_db=T["b"] is not None, dX=T["dXg"], dW=T["dWg"], db=T["dbg"],
                               ds=T["dsg"], d_eta=T["d_eta"], workspace=T["ws_bwd"])
        calls = {
            "sq_calibrate(mx)": Call(lambda T: sq.sq_calibrate(None, T["W"], a, s=T["s"], mx_inout=T["mx"],
                                                               workspace=T["ws_cal"]), ["W", "mx"], 2),
            "sq_prepare_weight": Call(lambda T: sq.sq_prepare_weight(T["W"], T["s"], Wq=T["Wq"],
                                                                     w_scale=T["w_scale"]), ["W"], 1),
            "sq_quantize_act": Call(lambda T: sq.sq_quantize_act(T["X"], T["s"], Xq=T["Xq"], x_scale=T["x_scale"]),
                                    ["X"], 1),
            "sq_linear": Call(lambda T: sq.sq_linear(T["Xq"], T["x_scale"], T["Wq"], T["w_scale"], T["b"], Y=T["Y"],
                                                     workspace=T["ws_lin"]), ["Xq", "Wq", "x_scale", "w_scale"], 1),
            "sq_rel_mse": Call(lambda T: sq.sq_rel_mse(T["Yfp"], T["Y"], AUX_WEIGHT, G_in=T["G"], G_out=T["Gt"],
                                                       loss=T["aux_loss"], workspace=T["ws_aux"]),
                               ["Yfp", "Y", "G"], 2),
            "sq_ste_backward": Call(bwd, ["Gt", "X", "W", "Xq", "Wq"], 6),
        }
        stages = [["sq_calibrate(mx)"], ["sq_prepare_weight", "sq_quantize_act"], ["sq_linear"], ["sq_rel_mse"],
                  ["sq_ste_backward"]]
    elif args.path == "per-tensor":
        T["ws_pt"] = torch.empty(sq.sq_quantize_per_tensor_workspace_bytes(), dtype=torch.uint8, device=dev)
        T["ws_pt2"] = torch.empty_like(T["ws_pt"])
        calls = {
            "sq_quantize_per_tensor(W)": Call(lambda T: sq.sq_quantize_per_tensor(
                T["W"], Aq=T["Wq"], scale_rows=T["w_scale"], workspace=T["ws_pt"]), ["W"], 2),
            "sq_quantize_per_tensor(X)": Call(lambda T: sq.sq_quantize_per_tensor(
                T["X"], Aq=T["Xq"], scale_rows=T["x_scale"], workspace=T["ws_pt2"]), ["X"], 2),
            "sq_linear": Call(lambda T: sq.sq_linear(T["Xq"], T["x_scale"], T["Wq"], T["w_scale"], T["b"], Y=T["Y"],
                                                     workspace=T["ws_lin"]), ["Xq", "Wq", "x_scale", "w_scale"], 1),
        }
        # measured slower side by side (41.4 against 40.5 us on proj): in order
        stages = [["sq_quantize_per_tensor(W)"], ["sq_quantize_per_tensor(X)"], ["sq_linear"]]
    elif args.path == "forward":
        # weights prepared once; the timed calls are sq_forward alone
        sq.sq_calibrate(T["C"], T["W"], a, s=T["s"], workspace=T["ws_cal"])
        sq.sq_prepare_weight(T["W"], T["s"], Wq=T["Wq"], w_scale=T["w_scale"])
        calls = {
            "sq_forward": Call(lambda T: sq.sq_forward(T["X"], T["s"], T["Wq"], T["w_scale"], T["b"], Y=T["Y"],
                                                       workspace=T["ws_fwd"]), ["Wq", "w_scale"], fwd_launches),
        }
        stages = [["sq_forward"]]
    elif args.path == "forward-prologue":
        sq.sq_calibrate(T["C"], T["W"], a, s=T["s"], workspace=T["ws_cal"])
        sq.sq_prepare_weight(T["W"], T["s"], Wq=T["Wq"], w_scale=T["w_scale"])
        calls = {  # the scale pre-pass and the GEMM
            "sq_forward_prologue": Call(lambda T: sq.sq_forward_prologue(T["X"], T["s"], T["Wq"], T["w_scale"],
                                                                         T["b"], Y=T["Y"], workspace=T["ws_pro"]),
                                        ["Wq", "w_scale"], 2),
        }
        stages = [["sq_forward_prologue"]]
    else:
        calls = {
            "sq_calibrate": Call(lambda T: sq.sq_calibrate(T["C"], T["W"], a, s=T["s"], workspace=T["ws_cal"]),
                                 ["C", "W"], 2),  # a small kernel clears the workspace first
            "sq_prepare_weight": Call(lambda T: sq.sq_prepare_weight(T["W"], T["s"], Wq=T["Wq"],
                                                                     w_scale=T["w_scale"]), ["W"], 1),
            "sq_quantize_act": Call(lambda T: sq.sq_quantize_act(T["X"], T["s"], Xq=T["Xq"], x_scale=T["x_scale"]),
                                    ["X"], 1),
            "sq_linear": Call(lambda T: sq.sq_linear(T["Xq"], T["x_scale"], T["Wq"], T["w_scale"], T["b"], Y=T["Y"],
                                                     workspace=T["ws_lin"]), ["Xq", "Wq", "x_scale", "w_scale"], 1),
        }
        stages = [["sq_calibrate"], ["sq_prepare_weight", "sq_quantize_act"], ["sq_linear"]]
    names = list(calls)
    launches_per_call = {n: calls[n].launches for n in names}
    assert sorted(n for st in stages for n in st) == sorted(names)
    side = [torch.cuda.Stream(device=dev) for _ in range(max(len(st) for st in stages) - 1)]

    def run_step(T):
        main = torch.cuda.current_stream()
        for st in stages:
            if len(st) == 1 or args.serial:
                for n in st:
                    calls[n].fn(T)
                continue
            fork = torch.cuda.Event()
            fork.record(main)
            for k, n in enumerate(st[1:]):
                side[k].wait_event(fork)
                with torch.cuda.stream(side[k]):
                    calls[n].fn(T)
            calls[st[0]].fn(T)
            for k in range(len(st) - 1):
                join = torch.cuda.Event()
                join.record(side[k])
                main.wait_event(join)

    # initialise library caches and the intermediate tensors outside capture
    for n in names:
        calls[n].fn(T)
    torch.cuda.synchronize()

    # input copies for the L2-cold per-call timing: consecutive launches read
    # different copies, whose inputs add up to >= ROTATE_BYTES
    sets, rotations = {}, {}
    for n in names:
        foot = sum(nbytes(T[k]) for k in calls[n].reads)
        r = rotation_count(foot)
        lst = [T]
        for _ in range(r - 1):
            Ti = dict(T)
            for k in calls[n].reads:
                Ti[k] = None if T[k] is None else T[k].clone()
            lst.append(Ti)
        sets[n] = lst
        rotations[n] = (r, r * foot >= ROTATE_BYTES)
    torch.cuda.synchronize()

    forward_path = args.path in FORWARD_CALLS
    fwd_call = FORWARD_CALLS.get(args.path)
    step_evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    g_step = torch.cuda.CUDAGraph()
    if forward_path:
        # the K timed calls in one graph, each on the next prepared weight copy
        fsets = sets[fwd_call]
        with torch.cuda.graph(g_step):
            step_evs[0].record()
            for k in range(args.steps):
                calls[fwd_call].fn(fsets[k % len(fsets)])
            step_evs[1].record()
        g_warm = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_warm):
            for k in range(max(args.warmup, 1)):
                calls[fwd_call].fn(fsets[k % len(fsets)])
    else:
        with torch.cuda.graph(g_step):
            step_evs[0].record()
            run_step(T)
            step_evs[1].record()
    call_evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(names) + 1)]
    g_calls = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_calls):
        call_evs[0].record()
        for i, n in enumerate(names):
            calls[n].fn(T)
            call_evs[i + 1].record()
    # each call back to back between two event nodes over its rotation: the
    # span / launches is that call's kernel duration with the event node's
    # launch latency amortised, every launch reading its inputs from HBM
    rep_evs = {n: [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for n in names}
    reps = {n: max(REPS, len(sets[n])) for n in names}
    g_reps = {}
    for n in names:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            rep_evs[n][0].record()
            for i in range(reps[n]):
                calls[n].fn(sets[n][i % len(sets[n])])
            rep_evs[n][1].record()
        g_reps[n] = g
    torch.cuda.synchronize()

    def flush_l2():
        flush.fill_(1)
        flush_read.max()

    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
    t_settle = time.perf_counter()
    for _ in range(1 if forward_path else args.warmup):
        flush_l2()
        (g_warm if forward_path else g_step).replay()
        flush_l2()
        g_calls.replay()
    torch.cuda.synchronize()
    # keep the GPU under load briefly so the clock sampler sees steady clocks
    while time.perf_counter() - t_settle < args.settle_s:
        for _ in range(20):
            flush_l2()
            (g_warm if forward_path else g_step).replay()
        torch.cuda.synchronize()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_times = []
    t_wall = time.perf_counter()
    if forward_path:
        flush_l2()
        g_step.replay()
        torch.cuda.synchronize()
        step_times.append(step_evs[0].elapsed_time(step_evs[1]) / args.steps)
    else:
        for k in range(args.steps):
            flush_l2()
            g_step.replay()
            torch.cuda.synchronize()  # the events are read before the next replay re-records them
            step_times.append(step_evs[0].elapsed_time(step_evs[1]))
    wall = time.perf_counter() - t_wall
    if world > 1:
        dist.barrier()
    # per-call device times (same flush, inputs rotated), for the roofline and the breakdown
    per_call_single = {n: 0.0 for n in names}
    per_call = {n: 0.0 for n in names}
    rep_steps = max(1, min(args.steps, 20))
    for k in range(rep_steps):
        flush_l2()
        g_calls.replay()
        torch.cuda.synchronize()
        for i, n in enumerate(names):
            per_call_single[n] += call_evs[i].elapsed_time(call_evs[i + 1])
        for n in names:
            flush_l2()
            g_reps[n].replay()
            torch.cuda.synchronize()
            per_call[n] += rep_evs[n][0].elapsed_time(rep_evs[n][1]) / reps[n]
    clocks = sampler.stop() if sampler else None

    mean_ms, median_ms = step_stats(step_times)
    step_ms = max_over_ranks(mean_ms, world, dev)
    step_median_ms = max_over_ranks(median_ms, world, dev)
    per_call = {n: v / rep_steps for n, v in per_call.items()}
    per_call_single = {n: v / rep_steps for n, v in per_call_single.items()}
    per_call_short = dict(per_call)
    if forward_path:
        # the timed region is itself the call back to back on rotating cold
        # weights: its mean launch duration is the call's (the short graph of
        # REPS launches also carries its first launch's start-up)
        per_call[fwd_call] = mean_ms

    # no bounded device wait may have run out during the timed work
    assert sq.sq_device_status() == 0, "device-side timeout flagged"

    # ------------------------------------------------------------- e2e leg
    # Through the Python binding, every step's inputs copied in from pinned
    # host memory and its Y (and d eta) copied out.  Two device buffer sets
    # and three streams pipeline the steps: the copy-in of step i+1 and the
    # copy-out of step i-1 overlap the kernels of step i (the copy engines and
    # the SMs work side by side, as a serving loop would run them).
    e2e = None
    if not args.no_e2e:
        def pinned(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()

        hX = pinned(inp["X"])
        hW = pinned(inp["W"]) if not forward_path else None
        hC = pinned(inp["C"]) if args.path == "smoothquant" else None
        hb = pinned(inp["bias"]) if (T["b"] is not None and not forward_path) else None
        hG = pinned(train_gradient(wl)) if args.path == "ste-train" else None
        hYfp = pinned(unquantised_output(wl, inp)) if args.path == "ste-train" else None
        hmx = T["mx"].cpu().pin_memory() if args.path == "ste-train" else None
        host_in = {"X": hX, "W": hW, "C": hC, "b": hb, "G": hG, "Yfp": hYfp, "mx": hmx}
        host_in = {k: v for k, v in host_in.items() if v is not None}
        bufs, h_out = [], []
        for _ in range(2):
            D = dict(T)
            for k in host_in:
                D[k] = torch.empty_like(T[k])
            D["Y"] = torch.empty_like(T["Y"])
            if args.path == "ste-train":
                D["d_eta"] = torch.empty_like(T["d_eta"])
                D["Gt"] = torch.empty_like(T["Gt"])
                D["aux_loss"] = torch.empty_like(T["aux_loss"])
            bufs.append(D)
            h_out.append({"Y": torch.empty(M, N, dtype=torch.bfloat16).pin_memory(),
                          "d_eta": torch.empty(1, dtype=torch.float32).pin_memory()})
        s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for b_ in range(2):  # nothing pending on either buffer set at the start
            ev_comp[b_].record(s_comp)
            ev_out[b_].record(s_out)

        def compute(D, i):
            if args.path == "weight-only":
                sq.sq_prepare_weight(D["W"], D["ones"], Wq=D["Wq"], w_scale=D["w_scale"])
                sq.sq_linear_weight_only(D["X"], D["Wq"], D["w_scale"], D["b"], Y=D["Y"])
            elif args.path == "ste-train":
                sq.sq_calibrate(None, D["W"], a, s=D["s"], mx_inout=D["mx"], workspace=D["ws_cal"])
                sq.sq_prepare_weight(D["W"], D["s"], Wq=D["Wq"], w_scale=D["w_scale"])
                sq.sq_quantize_act(D["X"], D["s"], Xq=D["Xq"], x_scale=D["x_scale"])
                sq.sq_linear(D["Xq"], D["x_scale"], D["Wq"], D["w_scale"], D["b"], Y=D["Y"], workspace=D["ws_lin"])
                sq.sq_rel_mse(D["Yfp"], D["Y"], AUX_WEIGHT, G_in=D["G"], G_out=D["Gt"], loss=D["aux_loss"],
                              workspace=D["ws_aux"])
                sq.sq_ste_backward(D["Gt"], D["X"], D["W"], D["s"], D["mx"], a, D["Xq"], D["x_scale"], D["Wq"],
                                   D["w_scale"], with_db=D["b"] is not None, dX=D["dXg"], dW=D["dWg"], db=D["dbg"],
                                   ds=D["dsg"], d_eta=D["d_eta"], workspace=D["ws_bwd"])
            elif args.path == "per-tensor":
                sq.sq_quantize_per_tensor(D["W"], Aq=D["Wq"], scale_rows=D["w_scale"], workspace=D["ws_pt"])
                sq.sq_quantize_per_tensor(D["X"], Aq=D["Xq"], scale_rows=D["x_scale"], workspace=D["ws_pt2"])
                sq.sq_linear(D["Xq"], D["x_scale"], D["Wq"], D["w_scale"], D["b"], Y=D["Y"], workspace=D["ws_lin"])
            elif args.path == "forward":
                F = sets["sq_forward"][i % len(sets["sq_forward"])]
                sq.sq_forward(D["X"], F["s"], F["Wq"], F["w_scale"], F["b"], Y=D["Y"], workspace=D["ws_fwd"])
            elif args.path == "forward-prologue":
                F = sets["sq_forward_prologue"][i % len(sets["sq_forward_prologue"])]
                sq.sq_forward_prologue(D["X"], F["s"], F["Wq"], F["w_scale"], F["b"], Y=D["Y"],
                                       workspace=D["ws_pro"])
            else:
                sq.sq_calibrate(D["C"], D["W"], a, s=D["s"], workspace=D["ws_cal"])
                sq.sq_prepare_weight(D["W"], D["s"], Wq=D["Wq"], w_scale=D["w_scale"])
                sq.sq_forward(D["X"], D["s"], D["Wq"], D["w_scale"], D["b"], Y=D["Y"], workspace=D["ws_fwd"])

        def e2e_step(i):
            b_ = i % 2
            D, H = bufs[b_], h_out[b_]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[b_])      # step i-2 has finished reading these inputs
                for k, h in host_in.items():
                    D[k].copy_(h, non_blocking=True)
                ev_in[b_].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[b_])
                s_comp.wait_event(ev_out[b_])     # step i-2's Y has been copied out
                compute(D, i)
                ev_comp[b_].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b_])
                H["Y"].copy_(D["Y"], non_blocking=True)
                if args.path == "ste-train":
                    H["d_eta"].copy_(D["d_eta"], non_blocking=True)
                ev_out[b_].record(s_out)

        for i in range(3):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(3 + i)
        for b_ in range(2):
            s_out.wait_event(ev_out[b_])
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
        # the copies of the last step agree with the device result
        assert torch.equal(h_out[(2 + args.e2e_steps) % 2]["Y"].view(torch.int16),
                           bufs[(2 + args.e2e_steps) % 2]["Y"].cpu().view(torch.int16))
        call = {"ste-train": "sq_calibrate(mx) + sq_prepare_weight + sq_quantize_act + sq_linear + sq_rel_mse + "
                             "sq_ste_backward, Y and d eta read back",
                "weight-only": "sq_prepare_weight (s = 1) + sq_linear_weight_only",
                "per-tensor": "sq_quantize_per_tensor(W) + sq_quantize_per_tensor(X) + sq_linear",
                "forward": "sq_forward on a prepared weight (X in, Y out)",
                "forward-prologue": "sq_forward_prologue on a prepared weight (X in, Y out)",
                "smoothquant": "sq_calibrate + sq_prepare_weight + sq_forward"}[args.path]
        outs = [h_out[0]["Y"]] + ([h_out[0]["d_eta"]] if args.path == "ste-train" else [])
        e2e = {"value": whole_job_rate(wl.M, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": sum(nbytes(t) for t in host_in.values()),
               "d2h_bytes_per_step": sum(nbytes(t) for t in outs), "ms_per_step": e2e_ms, "call": call,
               "pipelined": "two buffer sets, three streams: copy-in of step i+1 and copy-out of step i-1 "
                            "overlap the kernels of step i"}

    if rank != 0:
        return

    kernels, roof = kernel_report(wl, names, per_call, per_call_single, launches_per_call, rotations)
    if forward_path:
        kernels[fwd_call]["ms_timed_region"] = per_call[fwd_call]
        kernels[fwd_call]["ms_short_run"] = per_call_short[fwd_call]

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        v, n, el = cpu_oracle_rate(wl, args.cpu_seconds, path=args.path, inp=inp)
        cpu = {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{n} {oracle_sample_text(wl, args.path)}; {el:.1f} s of CPU work"}

    value = whole_job_rate(wl.M, world, step_ms)
    cfg = workload_config(wl, args.path)
    if not forward_path:
        cfg["schedule"] = ("serial" if args.serial else
                           " -> ".join("(" + " | ".join(st) + ")" if len(st) > 1 else st[0] for st in stages))
    gemm_call = next((n for n in ("sq_linear", "sq_forward", "sq_forward_prologue", "sq_linear_weight_only")
                      if n in per_call), None)
    line = {
        "metric": metric_for(args.path), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "ms_per_step_median": step_median_ms,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": cfg,
        "tops_per_step": 2.0 * wl.M * wl.N * wl.K * world / (step_ms * 1e-3) / 1e12,
        "gemm_tops": 2 * wl.M * wl.N * wl.K / (per_call[gemm_call] * 1e-3) / 1e12 if gemm_call else None,
        "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": args.steps * sum(launches_per_call.values()),  # the timed steps
        "clocks": clocks, "wall_s_timed": wall,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    wl = workloads.get(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
