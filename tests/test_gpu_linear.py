"""GPU parity of tb_ternary_linear against the fp64 oracle.

Float mode: relative L2 <= 2e-3 over the whole output and per element
|y - y*| <= 1e-2 * max|s| * ||x_m||_2 (tests/tolerances.py).  Integer mode:
bit-exact.  Every kernel path is exercised explicitly, at the seeded workloads'
shapes (full size where the oracle is quick), on ragged shapes and on edge
cases."""
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

GEMV, SIMPLE, AUTO = tb.TB_PATH_GEMV, tb.TB_PATH_SIMPLE, tb.TB_PATH_AUTO


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    assert tb.tb_get_device_fault() == 0


@functools.lru_cache(maxsize=None)
def _case(seed, m, n, k, p0, scale_kind="abs_normal", outlier=0.0):
    p = inputs.make_linear_inputs(seed, m, n, k, p0, scale_kind, outlier)
    ref = orc.linear(p.x, p.codes, p.scales, p.signs)
    return p, ref


@functools.lru_cache(maxsize=None)
def _problem(seed, m, n, k, p0, fmt, scale_kind="abs_normal", outlier=0.0):
    p, ref = _case(seed, m, n, k, p0, scale_kind, outlier)
    return Problem(p, fmt), ref


def _check(y, ref, p):
    ok, rel, worst = within_linear_tolerance(y, ref, p.scales, p.x)
    assert ok, f"rel_l2={rel:.3e} worst_elem_ratio={worst:.3f}"
    return rel


# (seed, m, n, k, p0, scale_kind, outlier): the named workloads plus ragged shapes
WORKLOAD_CASES = [
    (0, 1, 256, 1024, 1 / 3, "abs_normal", 0.0),       # tiny, one Hadamard block
    (1, 1, 17408, 5120, 0.33, "abs_normal", 0.01),     # gate/up decode GEMV, outliers
    (2, 1, 5120, 17408, 0.5, "lognormal", 0.0),        # down decode GEMV
    (2, 2, 5120, 17408, 0.5, "lognormal", 0.0),
    (2, 4, 5120, 17408, 0.5, "lognormal", 0.0),
    (9, 3, 1001, 2048, 0.33, "abs_normal", 0.0),       # ragged N (not a multiple of 4)
    (8, 1, 4, 1024, 0.33, "abs_normal", 0.0),          # fewer rows than one quad
    (10, 1, 20000, 1024, 0.33, "abs_normal", 0.0),     # more CTAs than SMs (rows per CTA capped)
    (11, 2, 6144, 6144, 0.2, "abs_normal", 0.0),       # q-projection shape
    (12, 1, 1024, 3072, 0.5, "abs_normal", 0.0),       # K/512 not a multiple of the stage width
    (13, 3, 5120, 6144, 0.33, "abs_normal", 0.01),     # o-projection shape
    (14, 2, 17408, 5120, 0.33, "abs_normal", 0.01),    # gate/up, two tokens (two-CTA decode kernel)
    (15, 4, 17408, 5120, 0.33, "abs_normal", 0.0),     # gate/up, four tokens
    (16, 3, 9999, 3072, 0.5, "abs_normal", 0.0),       # three tokens in a four-token kernel, ragged N
    (17, 1, 4000, 8192, 0.33, "abs_normal", 0.01),     # one token, 8 blocks: every warp rotates one
    (18, 1, 3000, 7168, 0.5, "abs_normal", 0.0),       # one token, 7 blocks, ragged rows per CTA
    (19, 1, 10000, 9216, 0.33, "abs_normal", 0.0),     # one token, 9 blocks: activation kernel, then decode
]


@pytest.mark.parametrize("case", WORKLOAD_CASES, ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_gemv_2bit(case):
    prob, ref = _problem(*case[:5], "2bit", *case[5:])
    y = prob.linear(GEMV)
    _check(y, ref, prob.p)


@pytest.mark.parametrize("case", WORKLOAD_CASES, ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_gemv_base3(case):
    prob, ref = _problem(*case[:5], "base3", *case[5:])
    y = prob.linear(GEMV)
    _check(y, ref, prob.p)


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("case", WORKLOAD_CASES[:3] + WORKLOAD_CASES[5:],
                         ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_simple_path(fmt, case):
    prob, ref = _problem(*case[:5], fmt, *case[5:])
    y = prob.linear(SIMPLE)
    _check(y, ref, prob.p)


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("m", [8, 16])
def test_down_workload_larger_m(fmt, m):
    prob, ref = _problem(2, m, 5120, 17408, 0.5, fmt, "lognormal", 0.0)
    _check(prob.linear(AUTO), ref, prob.p)


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_auto_path_matches_oracle(fmt):
    prob, ref = _problem(1, 1, 17408, 5120, 0.33, fmt, "abs_normal", 0.01)
    _check(prob.linear(AUTO), ref, prob.p)


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("path", [GEMV, SIMPLE])
def test_bf16_output(path, fmt):
    prob, ref = _problem(0, 1, 256, 1024, 1 / 3, fmt)
    y = prob.linear(path, yt=tb.TB_BF16)
    _check(y, ref, prob.p)


@pytest.mark.parametrize("path", [GEMV, SIMPLE])
@pytest.mark.parametrize("xt", [tb.TB_FP16, tb.TB_FP32])
@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_other_input_dtypes(path, xt, fmt):
    prob, ref = _problem(0, 2, 256, 1024, 1 / 3, fmt)
    xf = torch.from_numpy(prob.p.x).to(DEV)
    x = xf.to(torch.float16 if xt == tb.TB_FP16 else torch.float32)
    # bf16 values are exact in fp32; in fp16 they may round, so use fp16's own values
    xv = x.double().cpu().numpy()
    ref = orc.linear(xv, prob.p.codes, prob.p.scales, prob.p.signs)
    y = prob.linear(path, x=x, xt=xt)
    _check(y, ref, prob.p)


@pytest.mark.parametrize("xt", [tb.TB_FP16, tb.TB_FP32])
def test_one_token_input_dtypes(xt):
    """fp16 and fp32 activations through the one-token kernel's own rotation
    (strided loads of x, one warp per 1024-block)."""
    prob, _ = _problem(23, 1, 2000, 5120, 0.33, "2bit", "abs_normal", 0.01)
    x = torch.from_numpy(prob.p.x).to(DEV).to(torch.float16 if xt == tb.TB_FP16 else torch.float32)
    ref = orc.linear(x.double().cpu().numpy(), prob.p.codes, prob.p.scales, prob.p.signs)
    _check(prob.linear(GEMV, x=x, xt=xt), ref, prob.p)
    _check(prob.linear(GEMV, x=x, xt=xt, yt=tb.TB_BF16), ref, prob.p)


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("path", [GEMV, SIMPLE])
def test_prerotated_input_without_signs(path, fmt):
    prob, ref = _problem(1, 1, 17408, 5120, 0.33, fmt, "abs_normal", 0.01)
    xr = orc.rotate(prob.p.x, prob.p.signs)
    x = torch.from_numpy(xr.astype(np.float32)).to(DEV)
    y = prob.linear(path, x=x, xt=tb.TB_FP32, signs=None)
    _check(y, ref, prob.p)


def test_missing_rotation_is_wrong():
    """Without the inverse rotation the layer is silently wrong (news.ditty.ir,
    third paragraph): the GPU result must fail the tolerance."""
    prob, ref = _problem(0, 1, 256, 1024, 1 / 3, "2bit")
    y = prob.linear(GEMV, signs=None)
    ok, rel, _ = within_linear_tolerance(y, ref, prob.p.scales, prob.p.x)
    assert not ok and rel > 0.5


def test_simple_path_ragged_k_no_rotation():
    p = inputs.make_linear_inputs(12, 3, 77, 384, 0.33)
    prob = Problem(p, "2bit")
    ref = orc.linear(p.x, p.codes, p.scales, None)
    _check(prob.linear(SIMPLE, signs=None), ref, p)
    prob3 = Problem(p, "base3")
    _check(prob3.linear(AUTO, signs=None), ref, p)


def test_misaligned_pointers_take_simple_path():
    prob, ref = _problem(0, 1, 256, 1024, 1 / 3, "2bit")
    # x shifted by 2 bytes inside a larger buffer: valid for bf16, not 16-byte aligned
    big = torch.empty(1 * 1024 + 8, dtype=torch.bfloat16, device=DEV)
    big[1:1025].copy_(prob.x.reshape(-1))
    xmis = big[1:1025]
    assert xmis.data_ptr() % 16 != 0
    y = prob.linear(AUTO, x=xmis)
    _check(y, ref, prob.p)
    st = tb.tb_ternary_linear_ex(xmis, tb.TB_BF16, prob.packed, prob.scales, "2bit", 1, 256, 1024,
                                 prob.signs, torch.empty(1, 256, device=DEV), tb.TB_FP32,
                                 torch.empty(1 << 16, dtype=torch.uint8, device=DEV), 1 << 16,
                                 GEMV, check=False)
    assert st == tb.TB_ERR_SHAPE


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("m,n,k", [(1, 256, 1024), (4, 5120, 17408), (16, 300, 1152), (2, 17408, 5120)])
def test_integer_mode_bitexact(fmt, m, n, k):
    rng = np.random.default_rng(m + n + k)
    codes = inputs.draw_codes(rng, n, k, 0.4)
    x = rng.integers(-128, 128, size=(m, k)).astype(np.int8)
    dev_codes = to_dev_codes(codes)
    packed = torch.empty(tb.tb_packed_bytes(fmt, n, k), dtype=torch.uint8, device=DEV)
    tb.tb_pack_ternary(fmt, dev_codes, n, k, packed)
    y = torch.empty(m, n, dtype=torch.int32, device=DEV)
    tb.tb_ternary_linear(to_dev_codes(x), tb.TB_INT8, packed, None, fmt, m, n, k, None, y,
                         tb.TB_INT32, None, 0)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy().astype(np.int64), orc.linear_int(x, codes))


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_invalid_packed_bytes_do_not_fault(fmt):
    prob, _ = _problem(0, 1, 256, 1024, 1 / 3, fmt)
    bad = torch.full_like(prob.packed, 0xFF)
    for path in (GEMV, SIMPLE):
        y = prob.linear(path, packed=bad)
        assert y.shape == (1, 256)
    assert tb.tb_get_device_fault() == 0


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_repeated_calls_are_deterministic_gemv(fmt):
    prob, ref = _problem(2, 4, 5120, 17408, 0.5, fmt, "lognormal", 0.0)
    a = prob.linear(GEMV)
    b = prob.linear(GEMV)
    assert np.array_equal(a, b)


# ------------------------------------------------------------------ tensor-core path
GEMM = tb.TB_PATH_GEMM

GEMM_CASES = [
    (20, 5, 256, 1024, 1 / 3, "abs_normal", 0.0),      # one tile, M and N tails
    (21, 300, 1001, 2048, 0.33, "abs_normal", 0.0),    # ragged M (3 tiles) and N (4 tiles)
    (22, 129, 512, 3072, 0.2, "abs_normal", 0.0),      # M one past a tile
    (2, 16, 5120, 17408, 0.5, "lognormal", 0.0),       # down workload, M = 16
    (23, 256, 256, 5120, 0.33, "abs_normal", 0.01),    # outliers
]


@pytest.mark.parametrize("case", GEMM_CASES, ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_gemm_2bit(case):
    prob, ref = _problem(*case[:5], "2bit", *case[5:])
    _check(prob.linear(GEMM), ref, prob.p)


@pytest.mark.parametrize("m", [8, 12, 17, 300])
def test_gemm_base3_via_reencoding(m):
    """Base-3 prefill: the weights are re-encoded to 2-bit slots in the
    workspace, then the tensor-core GEMM runs on them."""
    prob, ref = _problem(27, m, 1001, 2048, 0.33, "base3", "abs_normal", 0.01)
    _check(prob.linear(GEMM), ref, prob.p)
    _check(prob.linear(AUTO), ref, prob.p)


def test_base3_tokens_beyond_one_row_tile_per_sm():
    """12 base-3 tokens and more rows than 148 x 128: re-encoded to 2-bit slots,
    then the tensor-core decode with two row tiles per CTA (automatic path) or
    the GEMM (asked for)."""
    assert tb.tb_ternary_linear_path(tb.TB_BF16, "base3", 12, 19000, 1024, True, True) == tb.TB_PATH_GEMV_TC
    prob, ref = _problem(28, 12, 19000, 1024, 0.33, "base3", "abs_normal", 0.01)
    _check(prob.linear(AUTO), ref, prob.p)
    _check(prob.linear(GEMM), ref, prob.p)


@pytest.mark.parametrize("yt", [tb.TB_FP32, tb.TB_BF16])
@pytest.mark.parametrize("xt", [tb.TB_FP16, tb.TB_FP32])
def test_gemm_dtypes(yt, xt):
    prob, _ = _problem(21, 300, 1001, 2048, 0.33, "2bit")
    x = torch.from_numpy(prob.p.x).to(DEV).to(torch.float16 if xt == tb.TB_FP16 else torch.float32)
    ref = orc.linear(x.double().cpu().numpy(), prob.p.codes, prob.p.scales, prob.p.signs)
    _check(prob.linear(GEMM, x=x, xt=xt, yt=yt), ref, prob.p)


def test_gemm_prerotated_without_signs():
    prob, ref = _problem(22, 129, 512, 3072, 0.2, "2bit")
    xr = orc.rotate(prob.p.x, prob.p.signs)
    x = torch.from_numpy(xr.astype(np.float32)).to(DEV)
    _check(prob.linear(GEMM, x=x, xt=tb.TB_FP32, signs=None), ref, prob.p)


def test_gemm_agrees_with_gemv_and_simple():
    prob, ref = _problem(2, 4, 5120, 17408, 0.5, "2bit", "lognormal", 0.0)
    yg = prob.linear(GEMM)
    _check(yg, ref, prob.p)
    ys = prob.linear(SIMPLE)
    assert np.linalg.norm(yg - ys) / np.linalg.norm(ys) < 2e-3


def test_gemm_prefill_full_size_sampled_rows():
    """The prefill workload (M=2048, K=5120, N=17408) in the launch configuration
    the bench uses, checked on 48 sampled token rows against the oracle."""
    w = inputs.WORKLOADS["prefill_m2048_k5120_n17408"]
    p = inputs.make_linear_inputs(w["seed"], 2048, w["n"], w["k"], w["p0"])
    prob = Problem(p, "2bit")
    y = prob.linear(AUTO)
    rows = np.sort(np.random.default_rng(0).choice(2048, 48, replace=False))
    ref = orc.linear(p.x[rows], p.codes, p.scales, p.signs)
    ok, rel, worst = within_linear_tolerance(y[rows], ref, p.scales, p.x[rows])
    assert ok, (rel, worst)
    assert np.isfinite(y).all()


@pytest.mark.parametrize("fmt", ["2bit", "1bit"])
@pytest.mark.parametrize("m,n,k", [(777, 9000, 1024),     # 4 x 36 tiles, ragged M and N (last CTA pair half empty)
                                   (100, 40000, 1024)])   # 128-token tiles, 157 of them
def test_gemm_several_tiles_per_cluster(fmt, m, n, k):
    """More pair tiles than clusters: each cluster walks two or three tiles
    (the read-out of one tile overlapping the next tile's first stages), with
    ragged token and row tiles; the whole output against the oracle, in fp32
    and bf16, and two calls give identical bits."""
    p0 = 0.33 if fmt == "2bit" else 0.0
    prob, ref = _problem(29, m, n, k, p0, fmt)
    y = prob.linear(GEMM)
    _check(y, ref, prob.p)
    assert np.array_equal(y, prob.linear(GEMM))
    _check(prob.linear(GEMM, yt=tb.TB_BF16), ref, prob.p)


def test_gemm_few_tiles_long_k_deterministic():
    """Few tiles (4 pair tiles) and long K (17408, 136 stages a tile): repeated
    calls give identical bits, in fp32 and bf16."""
    prob, ref = _problem(31, 64, 1000, 17408, 0.5, "2bit", "lognormal", 0.0)
    y = prob.linear(GEMM)
    _check(y, ref, prob.p)
    for _ in range(3):
        assert np.array_equal(y, prob.linear(GEMM))
    _check(prob.linear(GEMM, yt=tb.TB_BF16), ref, prob.p)


def test_gemm_invalid_bytes_no_fault():
    prob, _ = _problem(20, 5, 256, 1024, 1 / 3, "2bit")
    y = prob.linear(GEMM, packed=torch.full_like(prob.packed, 0xFF))
    assert y.shape == (5, 256)
    assert tb.tb_get_device_fault() == 0


GEMV_TC = tb.TB_PATH_GEMV_TC


# every workload shape: the tensor-core decode takes any N (two or more row
# tiles per CTA beyond 148 x 128 rows) and splits K over CTAs when rows are few
GEMV_TC_CASES = WORKLOAD_CASES


@pytest.mark.parametrize("case", GEMV_TC_CASES, ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_gemv_tensor_core_2bit(case):
    prob, ref = _problem(case[0], case[1], case[2], case[3], case[4], "2bit", case[5], case[6])
    _check(prob.linear(GEMV_TC), ref, prob.p)


@pytest.mark.parametrize("m", [5, 8, 9, 16])
def test_gemv_tensor_core_more_tokens(m):
    """5..16 tokens: 16- and 32-row activation tiles (two planes per token)."""
    prob, ref = _problem(25, m, 3001, 3072, 0.33, "2bit", "abs_normal", 0.01)
    _check(prob.linear(GEMV_TC), ref, prob.p)


@pytest.mark.parametrize("m", [5, 7])
def test_gemv_base3_token_chunks(m):
    """Five to seven tokens on base-3: one pass over the weights per chunk of four."""
    prob, ref = _problem(26, m, 1001, 2048, 0.33, "base3")
    _check(prob.linear(GEMV), ref, prob.p)


@pytest.mark.parametrize("m", [8, 16])
def test_base3_reencoded_tensor_core_decode(m):
    """Eight to sixteen tokens on base-3: the weights are re-encoded to 2-bit
    slots in the workspace, then the tensor-core decode runs on them."""
    prob, ref = _problem(26, m, 1001, 2048, 0.33, "base3")
    _check(prob.linear(tb.TB_PATH_GEMV_TC), ref, prob.p)
    _check(prob.linear(AUTO), ref, prob.p)


@pytest.mark.parametrize("m", [2, 16])
@pytest.mark.parametrize("n", [20480, 34816])
def test_gemv_tensor_core_rows_beyond_one_tile_per_sm(n, m):
    """More rows than 148 CTAs x 128 TMEM lanes: each CTA runs two row tiles in
    turn (34816 = the gate|up pair stacked along N)."""
    prob, ref = _problem(24, m, n, 1024 if n == 20480 else 5120, 0.33, "2bit")
    _check(prob.linear(GEMV_TC), ref, prob.p)


@pytest.mark.parametrize("m", [1, 3, 4, 8, 16])
@pytest.mark.parametrize("n,k", [(5120, 17408), (1024, 5120), (256, 1024), (6144, 5120), (5120, 6144)])
def test_gemv_tensor_core_k_split(n, k, m):
    """Few rows: K is split over several CTAs per row tile and the last CTA of
    a tile adds the partial sums (down, k/v, tiny, q and o shapes)."""
    prob, ref = _problem(27, m, n, k, 0.5, "2bit", "lognormal", 0.0)
    _check(prob.linear(GEMV_TC), ref, prob.p)


@pytest.mark.parametrize("n,k,m", [(5120, 17408, 16), (17408, 5120, 4), (34816, 5120, 8)])
def test_gemv_tensor_core_repeatable(n, k, m):
    """The split-K reduction adds the partial sums in a fixed order: repeated
    calls agree bit for bit."""
    prob, ref = _problem(28, m, n, k, 0.33, "2bit")
    a = prob.linear(GEMV_TC)
    b = prob.linear(GEMV_TC)
    assert np.array_equal(a, b)
    _check(a, ref, prob.p)
