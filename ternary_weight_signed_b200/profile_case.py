"""Runs one named workload through tb_ternary_linear a few times, for profilers.

    python -m ternary_weight_signed_b200.profile_case --workload gemv_gateup_k5120_n17408 \
        [--m 1] [--fmt 2bit|base3|1bit] [--path auto|gemv|gemv_tc|gemm|simple] [--int8] [--reps 4]

Inputs are the seeded synthetic ones of the workload; nothing is checked here
(the tests do that).  Exits non-zero if a call fails or the device records a
fault.
"""
from __future__ import annotations

import argparse
import sys

import numpy as np


def main(argv=None) -> int:
    import torch

    from . import binding as tb
    from . import build as tbbuild
    from . import inputs

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gemv_gateup_k5120_n17408", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--m", type=int, default=None)
    ap.add_argument("--fmt", default="2bit", choices=["2bit", "base3", "1bit"])
    ap.add_argument("--path", default="auto", choices=["auto", "gemv", "gemv_tc", "gemm", "simple"])
    ap.add_argument("--yt", default="fp32", choices=["fp32", "bf16"])
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--int8", action="store_true", help="integer mode: int8 x, exact int32 y")
    a = ap.parse_args(argv)
    tbbuild.build()
    w = inputs.WORKLOADS[a.workload]
    m = a.m or w["ms"][0]
    n, k = w["n"], w["k"]
    p0 = 0.0 if a.fmt == "1bit" else w["p0"]  # 1-bit codes are -1 or +1
    p = inputs.make_linear_inputs(w["seed"], m, n, k, p0, w["scale_kind"], w["outlier_rate"])
    dev = torch.device("cuda:0")
    codes = torch.from_numpy(p.codes).to(dev)
    packed = torch.empty(tb.tb_packed_bytes(a.fmt, n, k), dtype=torch.uint8, device=dev)
    tb.tb_pack_ternary(a.fmt, codes, n, k, packed)
    scales = torch.from_numpy(p.scales.view(np.int16)).to(dev)
    if a.int8:
        x = torch.from_numpy(np.random.default_rng(w["seed"]).integers(-127, 128, (m, k)).astype(np.int8)).to(dev)
        xt, signs, yt = tb.TB_INT8, None, tb.TB_INT32
        y = torch.empty(m, n, dtype=torch.int32, device=dev)
    else:
        x = torch.from_numpy(p.x_bf16.view(np.int16)).to(dev).view(torch.bfloat16)
        xt, signs = tb.TB_BF16, torch.from_numpy(p.signs).to(dev)
        yt = tb.TB_FP32 if a.yt == "fp32" else tb.TB_BF16
        y = torch.empty(m, n, dtype=torch.float32 if a.yt == "fp32" else torch.bfloat16, device=dev)
    ws_bytes = tb.tb_ternary_linear_workspace(a.fmt, m, n, k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    path = {"auto": tb.TB_PATH_AUTO, "gemv": tb.TB_PATH_GEMV, "gemv_tc": tb.TB_PATH_GEMV_TC, "gemm": tb.TB_PATH_GEMM,
            "simple": tb.TB_PATH_SIMPLE}[a.path]
    for _ in range(a.reps):
        tb.tb_ternary_linear_ex(x, xt, packed, scales, a.fmt, m, n, k, signs, y, yt, ws,
                                ws_bytes, path)
    torch.cuda.synchronize()
    fault = tb.tb_get_device_fault()
    print(f"profile_case {a.workload} m={m} fmt={a.fmt} path={a.path}: done, fault={fault}")
    return 1 if fault else 0


if __name__ == "__main__":
    sys.exit(main())
