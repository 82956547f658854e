"""Helpers for the GPU tests: move seeded inputs to the device and call the
library through its C ABI."""
import numpy as np
import torch

from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import build as tbbuild

DEV = torch.device("cuda:0")


def ensure_lib():
    tbbuild.build()
    return tb.load()


def to_dev_codes(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).to(DEV)


def to_dev_scales(scales):
    return torch.from_numpy(np.ascontiguousarray(scales).view(np.int16)).to(DEV)


def to_dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def pack_dev(fmt, codes_dev, n, k):
    packed = torch.empty(tb.tb_packed_bytes(fmt, n, k), dtype=torch.uint8, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    tb.tb_pack_ternary(fmt, codes_dev, n, k, packed, cnt)
    return packed, cnt


class Problem:
    """Device copies of one seeded problem, packed in `fmt`."""

    def __init__(self, p, fmt):
        self.p = p
        self.fmt = fmt
        self.n, self.k = p.codes.shape
        self.m = p.x_bf16.shape[0]
        self.codes = to_dev_codes(p.codes)
        self.packed, cnt = pack_dev(fmt, self.codes, self.n, self.k)
        assert int(cnt.item()) == 0
        self.scales = to_dev_scales(p.scales)
        self.x = to_dev_bf16(p.x_bf16)
        self.signs = to_dev_codes(p.signs)

    def linear(self, path=tb.TB_PATH_AUTO, yt=tb.TB_FP32, x=None, xt=tb.TB_BF16, signs="default",
               packed=None, scales=None, y=None, m=None):
        m = self.m if m is None else m
        x = self.x if x is None else x
        signs = self.signs if signs == "default" else signs
        packed = self.packed if packed is None else packed
        scales = self.scales if scales is None else scales
        ydt = torch.float32 if yt == tb.TB_FP32 else torch.bfloat16
        if y is None:
            y = torch.full((m, self.n), float("nan"), dtype=ydt, device=DEV)
        ws_bytes = tb.tb_ternary_linear_workspace(self.fmt, m, self.n, self.k)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
        tb.tb_ternary_linear_ex(x, xt, packed, scales, self.fmt, m, self.n, self.k, signs, y, yt,
                                ws, ws_bytes, path)
        torch.cuda.synchronize()
        return y.float().cpu().numpy().astype(np.float64)
