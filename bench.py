"""Benchmark of the ternary-g128 linear layer (signed block-Hadamard rotation
folded into the weights) on B200.

A step is one call of tb_ternary_linear on the decode GEMV workload
(M=1, K=5120, N=17408, ternary codes with P(0)=0.33, fp16 g128 scales, bf16
activations with 1% outliers): the inverse rotation of the activations and the
packed-weight GEMV.  The metric is packed-weight GB/s (codes + scales read
once per step).  Successive steps read successive copies of the weights, and
the copies together are larger than L2, so every step streams from HBM.

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
    for name in ("gemv.cuh", "hadamard.cuh", "tb_device.cuh"):
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
    fmt = args.fmt
    p = inputs.make_linear_inputs(w["seed"] + rank, m, n, k, w["p0"], w["scale_kind"],
                                  w["outlier_rate"])
    codes = torch.from_numpy(p.codes).to(dev)
    packed0 = torch.empty(tb.tb_packed_bytes(fmt, n, k), dtype=torch.uint8, device=dev)
    tb.tb_pack_ternary(fmt, codes, n, k, packed0)
    del codes
    scales0 = torch.from_numpy(p.scales.view(np.int16)).to(dev)
    step_bytes = _packed_bytes(fmt, n, k)
    copies = max(2, int(np.ceil(2.2 * L2_BYTES / step_bytes)))
    packs = [packed0] + [packed0.clone() for _ in range(copies - 1)]
    scls = [scales0] + [scales0.clone() for _ in range(copies - 1)]
    x = torch.from_numpy(p.x_bf16.view(np.int16)).to(dev).view(torch.bfloat16)
    signs = torch.from_numpy(p.signs).to(dev)
    y = torch.empty(m, n, dtype=torch.float32, device=dev)
    ws_bytes = tb.tb_ternary_linear_workspace(fmt, m, n, k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    path = tb.tb_ternary_linear_path(tb.TB_BF16, fmt, m, n, k, True, True)
    launches_per_step = 2  # activation prep (rotation + fixed point) and the streaming kernel

    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream

    def step(i):
        j = i % copies
        tb.tb_ternary_linear(x, tb.TB_BF16, packs[j], scls[j], fmt, m, n, k, signs, y, tb.TB_FP32,
                             ws, ws_bytes, stream=sh)

    def capture(nsteps, offset):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for i in range(nsteps):
                    step(offset + i)
        return g

    chunk = min(args.steps, 1200)
    chunk -= chunk % copies if chunk >= copies else 0
    chunk = max(chunk, 1)
    # warm-up: eager steps, then the captured graph
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            step(i)
    stream.synchronize()
    g_main = capture(chunk, 0)
    rem = args.steps % chunk
    g_rem = capture(rem, 0) if rem else None
    with torch.cuda.stream(stream):
        for _ in range(2):
            g_main.replay()
    stream.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps // chunk):
            g_main.replay()
        if g_rem is not None:
            g_rem.replay()
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    clocks = sampler.stop()
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_per_step = ms / args.steps

    # ---- end to end through the public call with HOST buffers: every step copies
    # x from pinned host memory, runs tb_ternary_linear and copies y back; the
    # steps are captured in a CUDA graph the way a decode loop would be.
    x_host = torch.from_numpy(p.x_bf16.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty(m, n, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(x)

    def e2e_step(i):
        x_dev.copy_(x_host, non_blocking=True)
        j = i % copies
        tb.tb_ternary_linear(x_dev, tb.TB_BF16, packs[j], scls[j], fmt, m, n, k, signs, y,
                             tb.TB_FP32, ws, ws_bytes, stream=sh)
        y_host.copy_(y, non_blocking=True)

    n_e2e = min(args.steps, 4 * chunk)
    with torch.cuda.stream(stream):
        for i in range(10):
            e2e_step(i)
    stream.synchronize()
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g_e2e, stream=stream):
            for i in range(chunk):
                e2e_step(i)
        g_e2e.replay()
    stream.synchronize()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    reps = max(1, n_e2e // chunk)
    with torch.cuda.stream(stream):
        a0.record(stream)
        for _ in range(reps):
            g_e2e.replay()
        a1.record(stream)
    a1.synchronize()
    e2e_ms = a0.elapsed_time(a1) / (reps * chunk)
    # the same without a graph: one Python call per step
    with torch.cuda.stream(stream):
        a0.record(stream)
        for i in range(200):
            e2e_step(i)
        a1.record(stream)
    a1.synchronize()
    eager_ms = a0.elapsed_time(a1) / 200
    e2e = {"value": round(step_bytes / (e2e_ms * 1e-3) / 1e9 * world, 2), "unit": "GB/s",
           "h2d_bytes_per_step": int(x.numel() * 2), "d2h_bytes_per_step": int(y.numel() * 4),
           "ms_per_step": round(e2e_ms, 5), "steps": reps * chunk,
           "how": "CUDA graph of [H2D x, tb_ternary_linear, D2H y] per step",
           "eager_ms_per_step": round(eager_ms, 5)}
    del g_e2e

    prefill = run_prefill(args, dev, stream, tb, inputs) if args.prefill else None

    gbs = step_bytes / (ms_per_step * 1e-3) / 1e9
    peak, peak_kind = _peaks()
    result = {
        "metric": METRIC,
        "value": round(gbs * world, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8 codes, fp16 scales, bf16 x -> fp32 (int8x2 dp4a, fp32 scale)",
        "data": "synthetic (seeded; codes P(0)=0.33, |N(0,1)|*0.02 fp16 scales, N(0,1) bf16 x with 1% +-20 outliers)",
        "config": {"workload": f"decode GEMV gate/up M=1 K=5120 N=17408 ({fmt} packing)",
                   "M": m, "K": k, "N": n, "format": fmt, "kernel_path": path,
                   "bytes_per_step": step_bytes, "weight_copies": copies,
                   "l2": f"inputs larger than L2: {copies} weight copies, {copies * step_bytes / 1e6:.0f} MB > 126 MB",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": _traffic(fmt),
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": "one tb_ternary_linear call (prep + streaming GEMV, PDL-overlapped)"},
        "e2e": e2e,
        "prefill": prefill,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    return result


def run_prefill(args, dev, stream, tb, inputs):
    """Prefill GEMM workload (M=2048 tokens, K=5120, N=17408, 2-bit): tokens/s,
    TFLOP-equivalent/s (2*M*N*K per call) and its fraction of the measured dense
    16-bit tensor peak.  Two weight copies alternate; the call is compute-bound."""
    import torch

    w = inputs.WORKLOADS["prefill_m2048_k5120_n17408"]
    m, n, k = 2048, w["n"], w["k"]
    p = inputs.make_linear_inputs(w["seed"], m, n, k, w["p0"])
    codes = torch.from_numpy(p.codes).to(dev)
    packs = [torch.empty(tb.tb_packed_bytes("2bit", n, k), dtype=torch.uint8, device=dev)
             for _ in range(2)]
    for pk in packs:
        tb.tb_pack_ternary("2bit", codes, n, k, pk)
    del codes
    scales = torch.from_numpy(p.scales.view(np.int16)).to(dev)
    x = torch.from_numpy(p.x_bf16.view(np.int16)).to(dev).view(torch.bfloat16)
    signs = torch.from_numpy(p.signs).to(dev)
    y = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
    ws_bytes = tb.tb_ternary_linear_workspace("2bit", m, n, k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    sh = stream.cuda_stream

    def call(i):
        tb.tb_ternary_linear(x, tb.TB_BF16, packs[i % 2], scales, "2bit", m, n, k, signs, y,
                             tb.TB_BF16, ws, ws_bytes, stream=sh)

    steps = max(10, min(200, args.steps // 100))
    with torch.cuda.stream(stream):
        for i in range(5):
            call(i)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(steps):
                call(i)
        g.replay()
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / steps
    flops = 2.0 * m * n * k
    tflops = flops / (ms * 1e-3) / 1e12
    peak, kind = _tensor_peak()
    return {"workload": "prefill GEMM M=2048 K=5120 N=17408 (2bit), bf16 in/out",
            "tok_s": round(m / (ms * 1e-3), 1), "ms_per_call": round(ms, 5), "steps": steps,
            "tflops_equiv": round(tflops, 2),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                         "peak_source": kind, "dtype": "fp16 x fp16 -> fp32 (kind::f16)"},
            "kernel_path": tb.tb_ternary_linear_path(tb.TB_BF16, "2bit", m, n, k, True, True)}


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


def run_reference(args, rank, world):
    if rank != 0:
        return None
    k_steps = args.steps
    per = max(0.2, min(2.0, 60.0 / max(k_steps + args.warmup, 1)))
    for _ in range(args.warmup):
        oracle_sample(args.fmt, per)
    t0 = time.perf_counter()
    vals = [oracle_sample(args.fmt, per) for _ in range(k_steps)]
    el = time.perf_counter() - t0
    gbs = statistics.median(v["value"] for v in vals)
    cb = dict(vals[-1])
    cb["value"] = gbs
    return {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": k_steps, "warmup": args.warmup, "ms_per_step": round(el / max(k_steps, 1) * 1e3, 3),
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
    ap.add_argument("--steps", type=int, default=200000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--fmt", default="2bit", choices=["2bit", "base3"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-prefill", dest="prefill", action="store_false")
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
