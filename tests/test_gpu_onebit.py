"""GPU parity of the 1-bit g128 format (each weight -1 or +1, one FP16 scale
per 128 weights, 1.125 bits per weight: dev.to, "How Prism ML Squeezed a 27B
Model Into 3.9 GB", "Two formats ship today") against the oracle.

Packing and unpacking are bit-exact against oracle.pack / oracle.unpack
(including the count of codes that are not -1 or +1); the linear layer meets
the float tolerance of tests/tolerances.py on every path that takes 1-bit
weights (the one-token decode, fused and with the activation kernel in front,
the prefill GEMM at 2 to 2048 tokens, the plain kernel) and integer mode is
bit-exact."""
import functools

import numpy as np
import pytest
import torch

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import inputs
from tests.gpu_util import DEV, Problem, ensure_lib, to_dev_codes
from tests.tolerances import within_linear_tolerance

pytestmark = pytest.mark.gpu

GEMV, GEMM, SIMPLE, AUTO = tb.TB_PATH_GEMV, tb.TB_PATH_GEMM, tb.TB_PATH_SIMPLE, tb.TB_PATH_AUTO


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    assert tb.tb_get_device_fault() == 0


@functools.lru_cache(maxsize=None)
def _problem(seed, m, n, k, outlier=0.0):
    # p0 = 0: every code is -1 or +1 with probability 1/2
    p = inputs.make_linear_inputs(seed, m, n, k, 0.0, "abs_normal", outlier)
    ref = orc.linear(p.x, p.codes, p.scales, p.signs)
    return Problem(p, "1bit"), ref


def _check(y, ref, p):
    ok, rel, worst = within_linear_tolerance(y, ref, p.scales, p.x)
    assert ok, f"rel_l2={rel:.3e} worst_elem_ratio={worst:.3f}"


def test_pack_unpack_bitexact():
    rng = np.random.default_rng(70)
    n, k = 37, 1152
    codes = np.where(rng.random((n, k)) < 0.5, -1, 1).astype(np.int8)
    codes[3, 5] = 0
    codes[9, 100] = 2
    codes[36, k - 1] = -7
    ref, bad = orc.pack(codes, "1bit")
    assert bad == 3
    packed = torch.zeros(tb.tb_packed_bytes("1bit", n, k), dtype=torch.uint8, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    tb.tb_pack_ternary("1bit", to_dev_codes(codes), n, k, packed, cnt)
    torch.cuda.synchronize()
    assert int(cnt.item()) == 3
    assert np.array_equal(packed.cpu().numpy().reshape(ref.shape), ref)
    back = torch.zeros(n, k, dtype=torch.int8, device=DEV)
    cnt.zero_()
    tb.tb_unpack_ternary("1bit", packed, n, k, back, cnt)
    torch.cuda.synchronize()
    assert int(cnt.item()) == 0
    want, _ = orc.unpack(ref, "1bit", n, k)
    assert np.array_equal(back.cpu().numpy(), want)


def test_unpack_every_byte_value():
    vals = np.arange(256, dtype=np.uint8).reshape(16, 16)  # every byte value: 16 rows of 128 codes
    n, k = 16, 128
    dev = torch.from_numpy(vals).to(DEV)
    out = torch.zeros(n, k, dtype=torch.int8, device=DEV)
    tb.tb_unpack_ternary("1bit", dev, n, k, out)
    torch.cuda.synchronize()
    want, bad = orc.unpack(vals, "1bit", n, k)
    assert bad == 0
    assert np.array_equal(out.cpu().numpy(), want)


# (seed, m, n, k, outlier)
GEMV_CASES = [
    (80, 1, 256, 1024, 0.0),        # one block: two warps rotate it
    (81, 1, 17408, 5120, 0.01),     # gate/up shape, one warp per block
    (82, 1, 1001, 4096, 0.0),       # ragged N, two warps per block
    (83, 1, 4000, 8192, 0.0),       # eight blocks
    (84, 1, 5120, 17408, 0.0),      # down shape: activation kernel, then decode
    (85, 1, 20000, 1024, 0.0),      # rows per CTA capped
    (86, 1, 4, 2048, 0.0),          # fewer rows than one tile
]


@pytest.mark.parametrize("case", GEMV_CASES, ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_gemv_1bit(case):
    prob, ref = _problem(*case)
    _check(prob.linear(GEMV), ref, prob.p)


@pytest.mark.parametrize("case", GEMV_CASES[:3], ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_gemv_1bit_prerotated(case):
    prob, _ = _problem(*case)
    xr = orc.rotate(prob.p.x, prob.p.signs)
    ref = orc.linear(xr, prob.p.codes, prob.p.scales)
    x32 = torch.from_numpy(xr.astype(np.float32)).to(DEV)
    y = prob.linear(GEMV, x=x32, xt=tb.TB_FP32, signs=None)
    _check(y, ref, prob.p)


# (seed, m, n, k)
GEMM_CASES = [
    (90, 2, 1000, 1024),
    (91, 5, 5120, 6144),
    (92, 16, 17408, 5120),
    (93, 64, 6144, 5120),
    (94, 300, 1003, 2048),
    (95, 2048, 4096, 5120),
]


@pytest.mark.parametrize("case", GEMM_CASES, ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_gemm_1bit(case):
    prob, ref = _problem(*case)
    assert tb.tb_ternary_linear_path(tb.TB_BF16, "1bit", case[1], case[2], case[3]) == GEMM
    _check(prob.linear(AUTO), ref, prob.p)


@pytest.mark.parametrize("path", [GEMV, GEMM, SIMPLE])
def test_bf16_output_1bit(path):
    prob, ref = _problem(80, 1, 256, 1024)
    _check(prob.linear(path, yt=tb.TB_BF16), ref, prob.p)


def test_simple_1bit_ragged_k():
    p = inputs.make_linear_inputs(96, 3, 77, 640, 0.0)
    prob = Problem(p, "1bit")
    ref = orc.linear(p.x, p.codes, p.scales)
    y = prob.linear(AUTO, signs=None)
    _check(y, ref, p)


def test_integer_mode_1bit_bitexact():
    rng = np.random.default_rng(97)
    m, n, k = 5, 300, 2048
    codes = np.where(rng.random((n, k)) < 0.5, -1, 1).astype(np.int8)
    x = rng.integers(-127, 128, (m, k)).astype(np.int8)
    packed = torch.zeros(tb.tb_packed_bytes("1bit", n, k), dtype=torch.uint8, device=DEV)
    tb.tb_pack_ternary("1bit", to_dev_codes(codes), n, k, packed)
    y = torch.zeros(m, n, dtype=torch.int32, device=DEV)
    tb.tb_ternary_linear(to_dev_codes(x), tb.TB_INT8, packed, None, "1bit", m, n, k, None, y, tb.TB_INT32,
                         None, 0)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy().astype(np.int64), orc.linear_int(x, codes))


def test_gemv_1bit_repeatable():
    prob, _ = _problem(81, 1, 17408, 5120, 0.01)
    a = prob.linear(GEMV)
    b = prob.linear(GEMV)
    assert np.array_equal(a, b)
