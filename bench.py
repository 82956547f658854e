"""Benchmark of the ternary-g128 linear layer (signed block-Hadamard rotation
folded into the weights) on B200.

The workload is the decode GEMV (M=1, K=5120, N=17408, ternary codes with
P(0)=0.33, fp16 g128 scales, bf16 activations with 1% outliers).  One call of
tb_ternary_linear is one pass of the hot path: the inverse rotation of the
activations and the packed-weight GEMV.  A step is a fixed batch of
CALLS_PER_STEP such calls, back to back in one CUDA graph, successive calls on
successive copies of the weights (together larger than L2, so every call
streams its weights from HBM).  `--steps K` times exactly K steps.  The metric
is packed-weight GB/s (codes + scales read once per call).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--fmt 2bit|base3]
  python bench.py --impl reference ...   (the CPU oracle on the same workload)

One JSON line on stdout (rank 0).
"""
from __future__ import annotations

import argparse
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "gemv_gateup_k5120_n17408"
METRIC = "ternary-g128 GEMV packed-weight GB/s vs HBM peak (M=1); prefill GEMM tok/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
CALLS_PER_STEP = 1000   # decode calls per step (rounded up to whole rounds of the weight copies)
PREFILL_CALLS_PER_STEP = 24  # prefill calls per step (a multiple of its 6 weight copies)


def _barrier(world):
    """All ranks meet here (no-op on one GPU)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x, dev, world):
    """The largest of the ranks' values of x: a job takes as long as its
    slowest rank.  x itself on one GPU."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def _workload_bytes(fmt, n, k):
    from oracle import ternary_oracle as orc  # sizes only
    return orc.packed_bytes(fmt, n, k) + n * (k // 128) * 2


def _packed_bytes(fmt, n, k):
    from ternary_weight_signed_b200 import binding as tb
    return tb.tb_packed_bytes(fmt, n, k) + n * (k // 128) * 2


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.split(",") for r in self.tmp.read().strip().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = max(smax, float(r[2]))
                for nm, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def _kernel_src_sha():
    h = hashlib.sha256()
    for name in ("gemv_m1.cuh", "gemv.cuh", "hadamard.cuh", "tb_device.cuh"):
        with open(os.path.join(ROOT, "ternary_weight_signed_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(fmt):
    """DRAM bytes per launch of the GEMV kernel from the committed ncu capture,
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "gemv_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(fmt)
        if e and e.get("kernel_src_sha") == _kernel_src_sha():
            return e["dram_bytes_per_launch"]
    except (OSError, ValueError):
        pass
    return None


# ---------------------------------------------------------------------------- ours
def _launches_per_call(tb, fmt, m, n, k):
    """Kernels one tb_ternary_linear call launches on the path it takes: the
    one-token 2-bit decode kernel rotates x itself up to K = 8192 (one launch);
    the other float paths run an activation prep kernel and one main kernel."""
    path = tb.tb_ternary_linear_path(tb.TB_BF16, fmt, m, n, k, True, True)
    if path == tb.TB_PATH_GEMV and fmt in ("2bit", "1bit") and m == 1 and k // 1024 <= 8:
        return 1
    if path == tb.TB_PATH_GEMV and fmt == "base3":
        return 2 * ((m + 3) // 4)
    return 2


def _upload_problem(tb, inputs, dev, fmt, m, n, k, seed, p0, scale_kind, outlier, copies):
    import torch
    p = inputs.make_linear_inputs(seed, m, n, k, p0, scale_kind, outlier)
    codes = torch.from_numpy(p.codes).to(dev)
    packed0 = torch.empty(tb.tb_packed_bytes(fmt, n, k), dtype=torch.uint8, device=dev)
    tb.tb_pack_ternary(fmt, codes, n, k, packed0)
    del codes
    scales0 = torch.from_numpy(p.scales.view(np.int16)).to(dev)
    packs = [packed0] + [packed0.clone() for _ in range(copies - 1)]
    scls = [scales0] + [scales0.clone() for _ in range(copies - 1)]
    x = torch.from_numpy(p.x_bf16.view(np.int16)).to(dev).view(torch.bfloat16)
    signs = torch.from_numpy(p.signs).to(dev)
    return p, packs, scls, x, signs


def _timed_replays(graph, steps, stream, dev, world):
    """Replays `graph` exactly `steps` times between a barrier and a device
    synchronisation on both sides; CUDA events on the launching stream give
    the total (max over ranks) and each replay's own time."""
    import torch
    _barrier(world)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    with torch.cuda.stream(stream):
        ev[0].record(stream)
        for i in range(steps):
            graph.replay()
            ev[i + 1].record(stream)
    ev[-1].synchronize()
    torch.cuda.synchronize()
    _barrier(world)
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total = _max_over_ranks(ev[0].elapsed_time(ev[-1]), dev, world)
    return total, per


def _spread(per, calls):
    """Median, p10 and p90 of the per-call time over the timed steps (ms)."""
    v = sorted(x / calls for x in per)
    q = lambda f: v[min(len(v) - 1, int(round(f * (len(v) - 1))))]
    return {"median": round(q(0.5), 6), "p10": round(q(0.1), 6), "p90": round(q(0.9), 6)}


def measure_decode(args, tb, inputs, dev, stream, fmt, m, n, k, seed, p0, scale_kind, outlier, world, sample=True):
    """Device time of `args.steps` steps of back-to-back tb_ternary_linear
    calls on the decode workload: a step is one replay of a CUDA graph of
    about CALLS_PER_STEP calls, successive calls on successive weight copies
    (together larger than L2, so every call streams its weights from HBM)."""
    import torch
    step_bytes = _packed_bytes(fmt, n, k)
    copies = max(2, int(np.ceil(2.2 * L2_BYTES / step_bytes)))
    p, packs, scls, x, signs = _upload_problem(tb, inputs, dev, fmt, m, n, k, seed, p0, scale_kind, outlier,
                                               copies)
    y = torch.empty(m, n, dtype=torch.float32, device=dev)
    ws_bytes = tb.tb_ternary_linear_workspace(fmt, m, n, k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    sh = stream.cuda_stream

    def call(i):
        j = i % copies
        tb.tb_ternary_linear(x, tb.TB_BF16, packs[j], scls[j], fmt, m, n, k, signs, y, tb.TB_FP32, ws, ws_bytes,
                             stream=sh)

    calls = copies * int(np.ceil(CALLS_PER_STEP / copies))
    with torch.cuda.stream(stream):
        for i in range(copies):
            call(i)
    stream.synchronize()
    g_main = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g_main, stream=stream):
            for i in range(calls):
                call(i)
        for _ in range(args.warmup):  # warm-up steps (untimed)
            g_main.replay()
    stream.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()) if sample else None
    if sampler:
        sampler.start()
    ms, per = _timed_replays(g_main, args.steps, stream, dev, world)
    clocks = sampler.stop() if sampler else None
    del g_main
    return {"ms_per_call": ms / (args.steps * calls), "ms_per_step": ms / args.steps, "steps": args.steps,
            "calls_per_step": calls, "per_call_spread": _spread(per, calls), "step_bytes": step_bytes,
            "copies": copies, "path": tb.tb_ternary_linear_path(tb.TB_BF16, fmt, m, n, k, True, True),
            "launches": _launches_per_call(tb, fmt, m, n, k) * calls * args.steps, "clocks": clocks,
            "problem": (p, packs, scls, x, signs, ws, ws_bytes, copies)}


def measure_e2e(args, tb, dev, stream, fmt, m, n, k, prob, world):
    """The same metric through the public call with host buffers: every step
    copies x from pinned host memory, runs tb_ternary_linear and copies y back
    to pinned host memory.  Consecutive steps are pipelined over three streams
    (host->device copy, compute, device->host copy) with two buffer sets, the
    way a serving loop overlaps them, and the steps are captured in a graph."""
    import torch
    p, packs, scls, _x, signs, ws, ws_bytes, copies = prob
    x_host = [torch.from_numpy(p.x_bf16.view(np.int16)).view(torch.bfloat16).pin_memory() for _ in range(2)]
    y_host = [torch.empty(m, n, dtype=torch.float32).pin_memory() for _ in range(2)]
    xd = [torch.empty(m, k, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    yd = [torch.empty(m, n, dtype=torch.float32, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    sh = stream.cuda_stream

    def steps(n_steps):
        for i in range(n_steps):
            j = i % 2
            if i >= 2:
                s_in.wait_event(ev_done[j])  # compute of step i-2 no longer reads xd[j]
            with torch.cuda.stream(s_in):
                xd[j].copy_(x_host[j], non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])  # device->host copy of step i-2 no longer reads yd[j]
            tb.tb_ternary_linear(xd[j], tb.TB_BF16, packs[i % copies], scls[i % copies], fmt, m, n, k, signs, yd[j],
                                 tb.TB_FP32, ws, ws_bytes, stream=sh)
            ev_done[j].record(stream)
            s_out.wait_event(ev_done[j])
            with torch.cuda.stream(s_out):
                y_host[j].copy_(yd[j], non_blocking=True)
                ev_out[j].record(s_out)
        # join the side streams back into the main one
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    calls = 2 * copies * int(np.ceil(CALLS_PER_STEP / (2 * copies)))
    with torch.cuda.stream(stream):
        steps(2 * copies)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        with torch.cuda.graph(g, stream=stream):
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            steps(calls)
        for _ in range(args.warmup):
            g.replay()
    torch.cuda.synchronize()
    ms, per = _timed_replays(g, args.steps, stream, dev, world)
    del g
    e2e_ms = ms / (args.steps * calls)
    step_bytes = _packed_bytes(fmt, n, k)
    return {"value": round(step_bytes / (e2e_ms * 1e-3) / 1e9 * world, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(calls * m * k * 2), "d2h_bytes_per_step": int(calls * m * n * 4),
            "calls_per_step": calls, "ms_per_call": round(e2e_ms, 6), "ms_per_step": round(ms / args.steps, 4),
            "steps": args.steps, "per_call_spread": _spread(per, calls),
            "how": "CUDA graph per step; per call: pinned-host x -> device, tb_ternary_linear, device y -> pinned "
                   "host; copies and compute of consecutive calls overlap on three streams, two buffer sets"}


def _decode_entry(res, peak, peak_kind, world):
    gbs = res["step_bytes"] / (res["ms_per_call"] * 1e-3) / 1e9
    return {"value": round(gbs * world, 2), "unit": "GB/s", "ms_per_call": round(res["ms_per_call"], 6),
            "ms_per_step": round(res["ms_per_step"], 4), "calls_per_step": res["calls_per_step"],
            "per_call_spread": res["per_call_spread"], "bytes_per_call": res["step_bytes"], "steps": res["steps"],
            "kernel_path": res["path"], "weight_copies": res["copies"],
            "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4),
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                         else "fallback 6.65 TB/s"}}


def run_ours(args, rank, world):
    import torch

    from ternary_weight_signed_b200 import binding as tb
    from ternary_weight_signed_b200 import build as tbbuild
    from ternary_weight_signed_b200 import inputs

    tbbuild.build()
    tb.load()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = inputs.WORKLOADS[WORKLOAD]
    m, n, k = 1, w["n"], w["k"]
    stream = torch.cuda.Stream(device=dev)
    peak, peak_kind = _peaks()
    fmts = [args.fmt] + [f for f in ("2bit", "base3", "1bit") if f != args.fmt]
    main = None
    others = {}
    for fmt in fmts:
        p0 = 0.0 if fmt == "1bit" else w["p0"]  # 1-bit codes are -1 or +1
        res = measure_decode(args, tb, inputs, dev, stream, fmt, m, n, k, w["seed"] + rank, p0,
                             w["scale_kind"], w["outlier_rate"], world, sample=(fmt == args.fmt))
        if fmt == args.fmt:
            main = res
            e2e = measure_e2e(args, tb, dev, stream, fmt, m, n, k, res["problem"], world)
        else:
            others[fmt] = _decode_entry(res, peak, peak_kind, world)
        res.pop("problem")
        torch.cuda.empty_cache()
    prefill = run_prefill(args, dev, stream, tb, inputs, world) if args.prefill else None
    prefill_int = run_prefill(args, dev, stream, tb, inputs, world, integer=True) if args.prefill else None
    stack = (stack_cells(args, dev, stream, tb, inputs, ["2bit"], [1, 16], [0.33], ["separate", "shared_input"],
                         args.steps, inputs.STACK_LAYERS, world) if args.stack_leg else None)
    head = _decode_entry(main, peak, peak_kind, world)
    roof = head["roofline"]
    roof["traffic"] = _traffic(args.fmt)
    roof["kernel"] = {"2bit": "tb_ternary_linear decode call (gemv1_kernel, 2-bit, rotation fused)",
                      "1bit": "tb_ternary_linear decode call (gemv1_kernel, 1-bit, rotation fused)",
                      "base3": "tb_ternary_linear decode call (prep_b3_kernel + gemv_b3_kernel)"}[args.fmt]
    roof["timing"] = ("device time per call over the timed steps (back-to-back calls in a CUDA graph, CUDA events "
                      "on the launching stream)")
    return {
        "metric": METRIC,
        "value": head["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": main["steps"],
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8 codes, fp16 scales, bf16 x -> fp32 (dp2a: u8 codes x int16 fixed-point x', exact int32 per "
                 "group, fp32 scale)",
        "data": "synthetic (seeded; codes P(0)=0.33, |N(0,1)|*0.02 fp16 scales, N(0,1) bf16 x with 1% +-20 outliers)",
        "config": {"workload": f"decode GEMV gate/up M=1 K=5120 N=17408 ({args.fmt} packing)",
                   "M": m, "K": k, "N": n, "format": args.fmt, "kernel_path": main["path"],
                   "calls_per_step": main["calls_per_step"], "bytes_per_call": main["step_bytes"],
                   "weight_copies": main["copies"],
                   "l2": f"inputs larger than L2: {main['copies']} weight copies, "
                         f"{main['copies'] * main['step_bytes'] / 1e6:.0f} MB > 126 MB",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "formats": others,
        "e2e": e2e,
        "prefill": prefill,
        "prefill_integer": prefill_int,
        "stack": stack,
        "gpu_launches": main["launches"],
        "clocks": main["clocks"],
    }


def run_prefill(args, dev, stream, tb, inputs, world=1, integer=False):
    """Prefill GEMM workload (M=2048 tokens, K=5120, N=17408, 2-bit): tokens/s
    of the whole job (every rank one replica, timed as the slowest rank),
    TFLOP-equivalent/s per GPU (2*M*N*K per call) and its fraction of the
    measured dense tensor peak.  Float mode: bf16 x rotated and rounded to
    fp16, kind::f16 MMAs.  Integer mode (`integer`): int8 x, exact int32 y,
    kind::i8 MMAs.  Successive calls take successive copies of the weights (6)
    and of the activations (2), more than L2 together; the call is
    compute-bound."""
    import torch

    w = inputs.WORKLOADS["prefill_m2048_k5120_n17408"]
    m, n, k = 2048, w["n"], w["k"]
    p = inputs.make_linear_inputs(w["seed"], m, n, k, w["p0"])
    codes = torch.from_numpy(p.codes).to(dev)
    wcopies, xcopies = 6, 2
    packs = [torch.empty(tb.tb_packed_bytes("2bit", n, k), dtype=torch.uint8, device=dev)
             for _ in range(wcopies)]
    for pk in packs:
        tb.tb_pack_ternary("2bit", codes, n, k, pk)
    del codes
    scls = [torch.from_numpy(p.scales.view(np.int16)).to(dev) for _ in range(wcopies)]
    if integer:
        xi = np.random.default_rng(w["seed"]).integers(-127, 128, (m, k)).astype(np.int8)
        xs = [torch.from_numpy(xi).to(dev) for _ in range(xcopies)]
        xt, yt, ydt, signs = tb.TB_INT8, tb.TB_INT32, torch.int32, None
    else:
        xs = [torch.from_numpy(p.x_bf16.view(np.int16)).to(dev).view(torch.bfloat16) for _ in range(xcopies)]
        xt, yt, ydt, signs = tb.TB_BF16, tb.TB_BF16, torch.bfloat16, torch.from_numpy(p.signs).to(dev)
    y = torch.empty(m, n, dtype=ydt, device=dev)
    ws_bytes = tb.tb_ternary_linear_workspace("2bit", m, n, k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    sh = stream.cuda_stream

    def call(i):
        tb.tb_ternary_linear(xs[i % xcopies], xt, packs[i % wcopies], scls[i % wcopies], "2bit", m, n, k,
                             signs, y, yt, ws, ws_bytes, stream=sh)

    calls = PREFILL_CALLS_PER_STEP
    with torch.cuda.stream(stream):
        for i in range(3):
            call(i)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(calls):
                call(i)
        for _ in range(args.warmup):
            g.replay()
    stream.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    total, per = _timed_replays(g, args.steps, stream, dev, world)
    clocks = sampler.stop()
    del g
    ms = total / (args.steps * calls)
    flops = 2.0 * m * n * k
    tflops = flops / (ms * 1e-3) / 1e12
    peak, kind = _tensor_peak()
    if integer:
        peak, kind = 2.0 * peak, kind + " x 2 (nominal dense int8 : bf16 = 4.5 : 2.25 PFLOP/s)"
    return {"workload": ("prefill GEMM M=2048 K=5120 N=17408 (2bit), " +
                         ("int8 in, exact int32 out (integer mode)" if integer else "bf16 in/out")),
            "tok_s": round(m * world / (ms * 1e-3), 1), "ms_per_call": round(ms, 5),
            "calls_per_step": calls, "steps": args.steps, "ms_timed": round(total, 3),
            "l2": "6 weight copies and 2 activation copies in rotation, more than 126 MB L2",
            "per_call_spread": _spread(per, calls), "tflops_equiv": round(tflops, 2),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": round(peak, 1),
                         "unit": "TFLOP/s" if not integer else "TOP/s", "frac": round(tflops / peak, 4),
                         "peak_source": kind,
                         "frac_of_sustained": _sustained_frac(tflops, integer),
                         "dtype": "s8 x s8 -> s32 (kind::i8)" if integer else "fp16 x fp16 -> fp32 (kind::f16)",
                         "kernel": "gemm_pair_kernel (CTA pairs, cta_group::2, A = unpacked weights in TMEM)"},
            "clocks": clocks,
            "kernel_path": tb.tb_ternary_linear_path(xt, "2bit", m, n, k, not integer, True)}


def _sustained_frac(tflops, integer):
    """The same figure against the sustained (seconds-long, power-capped) bf16 measurement, for context."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            sus = float(json.load(f)["bf16_tflops_sustained"])
    except (OSError, KeyError, ValueError):
        return None
    return round(tflops / (sus * (2.0 if integer else 1.0)), 4)


def _tensor_peak():
    """Dense 16-bit tensor peak: the measured bf16 burst figure (fp16 runs at the
    same nominal rate as bf16 on B200, ratio 1)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured bf16 burst (MEASURED_PEAKS.json) x 1 for fp16"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback 1.59 PFLOP/s"


# ---------------------------------------------------------------------------- CPU oracle
def oracle_sample(fmt, seconds):
    """Times the oracle (as it stands) on a row sample of the workload."""
    from oracle import ternary_oracle as orc
    from ternary_weight_signed_b200 import inputs

    w = inputs.WORKLOADS[WORKLOAD]
    rows = 1024
    p = inputs.make_linear_inputs(w["seed"], 1, rows, w["k"], w["p0"], w["scale_kind"],
                                  w["outlier_rate"])
    t0 = time.perf_counter()
    reps = 0
    while True:
        orc.linear(p.x, p.codes, p.scales, p.signs)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    bytes_done = reps * _workload_bytes(fmt, rows, w["k"])
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        blas = 1
    return {"value": round(bytes_done / el / 1e9, 4), "unit": "GB/s", "cores": int(blas),
            "host_cpus": os.cpu_count(), "kind": "oracle",
            "sample": f"{reps} x oracle.linear on {rows} of 17408 rows (K=5120, M=1), {el:.1f} s"}


def run_sweep(args, rank, world):
    """Down-projection decode sweep (K=17408, N=5120, M in {1,2,4,8,16}, both
    packings): device time per call and packed-weight GB/s of each cell, timed
    like the headline line.  Printed as its own JSON line (not the bench line)."""
    import torch

    from ternary_weight_signed_b200 import binding as tb
    from ternary_weight_signed_b200 import build as tbbuild
    from ternary_weight_signed_b200 import inputs

    tbbuild.build()
    tb.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    peak, peak_kind = _peaks()
    w = inputs.WORKLOADS["gemv_down_k17408_n5120"]
    cells = []
    for fmt in ("2bit", "base3"):
        for m in w["ms"]:
            res = measure_decode(args, tb, inputs, dev, stream, fmt, m, w["n"], w["k"], w["seed"], w["p0"],
                                 w["scale_kind"], w["outlier_rate"], world, sample=False)
            res.pop("problem")
            e = _decode_entry(res, peak, peak_kind, world)
            e.update({"format": fmt, "M": m, "tokens_per_s": round(m / (res["ms_per_call"] * 1e-3), 1)})
            cells.append(e)
            torch.cuda.empty_cache()
    return {"sweep": "decode GEMV down K=17408 N=5120", "cells": cells}


STACK_CALLS = {
    # one call per matrix: 7 calls (7 rotations) per layer
    "separate": (("q",), ("k",), ("v",), ("o",), ("gate",), ("up",), ("down",)),
    # one call per shared input: q|k|v and gate|up stacked along N, 4 calls
    # (4 rotations) per layer
    "shared_input": (("q", "k", "v"), ("o",), ("gate", "up"), ("down",)),
}


def stack_cells(args, dev, stream, tb, inputs, fmts, ms, p0s, modes, steps, layers, world=1):
    """The synthetic 27B-class layer stack: `layers` layers x {q, k, v, o,
    gate, up, down} of distinct ternary weights (5.8 GB in 2-bit slots, 4.8 GB
    in base-3 at 64 layers).  One pass = every call of the stack in one CUDA
    graph; every call reads the synthetic input of its width (no attention or
    nonlinearity between the linears).  Calls per layer: 7 (mode "separate") or
    4 (mode "shared_input": matrices that read the same input stacked along N
    behind one rotation).  `steps` passes are timed (a pass reads the whole
    stack, far more than L2).  Per cell: device time per pass, tokens/s =
    M / time, packed-weight GB/s."""
    import torch

    seed = 4
    shapes = {name: (n, k) for name, n, k in inputs.STACK_LAYER_SHAPES}
    mat = {name: j for j, (name, _, _) in enumerate(inputs.STACK_LAYER_SHAPES)}
    peak, peak_kind = _peaks()
    kdims = sorted({k for _, k in shapes.values()})
    xin = {}
    for m in ms:
        for k in kdims:
            xb, sg = inputs.stack_activations(seed, m, k)
            xin[(m, k)] = (torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16),
                           torch.from_numpy(sg).to(dev))
    cells = []
    for p0 in p0s:
        for f in fmts:
            # every matrix generated once and packed into the buffer of its
            # call in each mode
            bufs = {mode: [] for mode in modes}
            for layer in range(layers):
                where = {}
                for mode in modes:
                    for names in STACK_CALLS[mode]:
                        k = shapes[names[0]][1]
                        ntot = sum(shapes[nm][0] for nm in names)
                        pk = torch.empty(tb.tb_packed_bytes(f, ntot, k), dtype=torch.uint8, device=dev)
                        sc = torch.empty(ntot, k // 128, dtype=torch.int16, device=dev)
                        bufs[mode].append((pk, sc, ntot, k))
                        row = 0
                        for nm in names:
                            where.setdefault(nm, []).append((pk, sc, row))
                            row += shapes[nm][0]
                for nm, (n, k) in shapes.items():
                    codes = inputs.stack_codes_torch(seed, layer, mat[nm], n, k, p0, dev)
                    scn = torch.from_numpy(inputs.stack_scales(seed, layer, mat[nm], n, k).view(np.int16)).to(dev)
                    rb = tb.tb_packed_bytes(f, 1, k)
                    for pk, sc, row in where[nm]:
                        tb.tb_pack_ternary(f, codes, n, k, pk[row * rb:(row + n) * rb])
                        sc[row:row + n].copy_(scn)
                    del codes
            torch.cuda.synchronize()
            pass_bytes = sum(_packed_bytes(f, n, k) for n, k in shapes.values()) * layers
            for mode in modes:
                for m in ms:
                    ns = {b[2] for b in bufs[mode]}
                    ys = {n: torch.empty(m, n, dtype=torch.float32, device=dev) for n in ns}
                    wsb = max(tb.tb_ternary_linear_workspace(f, m, b[2], b[3]) for b in bufs[mode])
                    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
                    sh = stream.cuda_stream
                    paths = sorted({tb.tb_ternary_linear_path(tb.TB_BF16, f, m, b[2], b[3], True, True)
                                    for b in bufs[mode]})

                    def one_pass():
                        for pk, sc, n, k in bufs[mode]:
                            x, sg = xin[(m, k)]
                            tb.tb_ternary_linear(x, tb.TB_BF16, pk, sc, f, m, n, k, sg, ys[n], tb.TB_FP32, ws, wsb,
                                                 stream=sh)

                    with torch.cuda.stream(stream):
                        one_pass()
                        g = torch.cuda.CUDAGraph()
                        with torch.cuda.graph(g, stream=stream):
                            one_pass()
                        for _ in range(max(1, args.warmup)):
                            g.replay()
                    stream.synchronize()
                    total, per = _timed_replays(g, steps, stream, dev, world)
                    ms_pass = total / steps
                    gbs = pass_bytes / (ms_pass * 1e-3) / 1e9
                    cells.append({"format": f, "p0": p0, "M": m, "mode": mode, "ms_per_pass": round(ms_pass, 4),
                                  "tokens_per_s": round(world * m / (ms_pass * 1e-3), 1),
                                  "weight_GBs": round(gbs, 1), "hbm_frac": round(gbs / peak, 4),
                                  "paths": paths, "calls_per_pass": len(bufs[mode]), "passes_timed": steps})
                    del g, ws, ys
                    torch.cuda.empty_cache()
            del bufs
            torch.cuda.empty_cache()
    return {"stack": f"synthetic 27B-class layer stack, {layers} layers x 7 linears",
            "bytes_per_pass": {f: sum(_packed_bytes(f, n, k) for n, k in shapes.values()) * layers for f in fmts},
            "peak_GBs": peak, "peak_source": peak_kind, "cells": cells}


def run_stack(args, rank, world):
    """The stack sweep (--stack): every (zero fraction, packing, call mode,
    tokens) cell asked for.  Printed as its own JSON line."""
    import torch

    from ternary_weight_signed_b200 import binding as tb
    from ternary_weight_signed_b200 import build as tbbuild
    from ternary_weight_signed_b200 import inputs

    tbbuild.build()
    tb.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    return stack_cells(args, dev, stream, tb, inputs, args.stack_fmts.split(","),
                       [int(v) for v in args.stack_ms.split(",")], [float(v) for v in args.stack_p0.split(",")],
                       args.stack_modes.split(","), args.steps, args.stack_layers, world)


def run_reference(args, rank, world):
    """The CPU oracle, as it stands, on the same workload: every step is one
    oracle.linear call on a 1024-row sample of the 17408-row matrix (about
    0.1 s on the host cores).  At most 150 s of steps are timed, so that any
    --steps K ends within a few minutes; the line reports how many ran."""
    if rank != 0:
        return None
    budget_s = 150.0
    for _ in range(min(args.warmup, 3)):
        oracle_sample(args.fmt, 0.0)
    t0 = time.perf_counter()
    vals = []
    while len(vals) < args.steps:
        vals.append(oracle_sample(args.fmt, 0.0))
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    gbs = statistics.median(v["value"] for v in vals)
    cb = dict(vals[-1])
    cb["value"] = gbs
    cb["sample"] = f"{len(vals)} steps, each one oracle.linear on 1024 of 17408 rows (K=5120, M=1)"
    return {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": len(vals), "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / len(vals) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same recipe as the GPU arm)",
        "config": {"workload": f"decode GEMV gate/up M=1 K=5120 N=17408 ({args.fmt} packing)",
                   "format": args.fmt, "parallelism": "host cores"},
        "cpu_baseline": cb,
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--fmt", default="2bit", choices=["2bit", "base3", "1bit"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-prefill", dest="prefill", action="store_false")
    ap.add_argument("--sweep", action="store_true", help="print the down-projection decode sweep instead")
    ap.add_argument("--stack", action="store_true", help="print the 64-layer stack sweep instead")
    ap.add_argument("--stack-layers", type=int, default=64)
    ap.add_argument("--stack-ms", default="1,4,16,64,512")
    ap.add_argument("--stack-p0", default="0.2,0.33,0.5")
    ap.add_argument("--stack-fmts", default="2bit,base3")
    ap.add_argument("--stack-modes", default="separate,shared_input")
    ap.add_argument("--no-stack", dest="stack_leg", action="store_false",
                    help="leave the layer-stack leg out of the bench line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    elif args.sweep:
        res = run_sweep(args, rank, world)
    elif args.stack:
        res = run_stack(args, rank, world)
    else:
        res = run_ours(args, rank, world)
        if rank == 0:
            res["cpu_baseline"] = oracle_sample(args.fmt, args.cpu_seconds) if world == 1 else None
    if world > 1 and args.impl == "ours":
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
