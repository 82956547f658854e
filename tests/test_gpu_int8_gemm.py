"""Integer mode on the tensor cores (tcgen05 kind::i8): y[m, n] = sum_k t[n, k]
x[m, k] for int8 x, no rotation, no scales (a ternary product is an add, a
subtract or nothing: ai4coding.ru, "What is a ternary model", last
paragraph).  Bit-exact against oracle.linear_int on every packed format, at
ragged shapes, at K that is a multiple of 128 but not of 1024, and at the
prefill shape (2048 x 17408 x 5120) on sampled rows."""
import numpy as np
import pytest
import torch

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import inputs
from tests.gpu_util import DEV, ensure_lib, to_dev_codes

pytestmark = pytest.mark.gpu

GEMM, SIMPLE = tb.TB_PATH_GEMM, tb.TB_PATH_SIMPLE


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    assert tb.tb_get_device_fault() == 0


def _codes(rng, n, k, fmt, p0=0.33):
    if fmt == "1bit":
        return np.where(rng.random((n, k)) < 0.5, -1, 1).astype(np.int8)
    return inputs.draw_codes(rng, n, k, p0)


def _run(fmt, codes, x, with_ws=True, path=tb.TB_PATH_AUTO):
    n, k = codes.shape
    m = x.shape[0]
    packed = torch.zeros(tb.tb_packed_bytes(fmt, n, k), dtype=torch.uint8, device=DEV)
    tb.tb_pack_ternary(fmt, to_dev_codes(codes), n, k, packed)
    y = torch.full((m, n), -7, dtype=torch.int32, device=DEV)
    wsb = tb.tb_ternary_linear_workspace(fmt, m, n, k) if with_ws else 0
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV) if with_ws else None
    tb.tb_ternary_linear_ex(to_dev_codes(x), tb.TB_INT8, packed, None, fmt, m, n, k, None, y, tb.TB_INT32,
                            ws, wsb, path)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.int64)


# (seed, m, n, k)
CASES = [
    (60, 16, 256, 1024),
    (61, 17, 1001, 2048),
    (62, 64, 6144, 5120),
    (63, 300, 1003, 640),     # K a multiple of 128, not of 1024
    (64, 129, 4096, 17408),
    (65, 512, 5120, 6144),
]


@pytest.mark.parametrize("fmt", ["2bit", "1bit", "base3"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"m{c[1]}n{c[2]}k{c[3]}")
def test_int8_gemm_bitexact(case, fmt):
    seed, m, n, k = case
    rng = np.random.default_rng(seed)
    codes = _codes(rng, n, k, fmt)
    x = rng.integers(-128, 128, (m, k)).astype(np.int8)  # the full int8 range
    assert tb.tb_ternary_linear_path(tb.TB_INT8, fmt, m, n, k, False, True) == GEMM
    got = _run(fmt, codes, x, path=GEMM)
    assert np.array_equal(got, orc.linear_int(x, codes))


@pytest.mark.parametrize("fmt", ["2bit", "1bit"])
def test_int8_gemm_several_tiles_per_cluster(fmt):
    """94 pair tiles (more than the clusters), ragged M and N, and K = 640: the
    last stage holds 128 of its 256 codes (the copies read zeros past K)."""
    rng = np.random.default_rng(70)
    m, n, k = 300, 12000, 640
    codes = _codes(rng, n, k, fmt)
    x = rng.integers(-128, 128, (m, k)).astype(np.int8)
    got = _run(fmt, codes, x, path=GEMM)
    assert np.array_equal(got, orc.linear_int(x, codes))


@pytest.mark.parametrize("fmt", ["2bit", "1bit"])
def test_int8_long_k_with_and_without_workspace(fmt):
    """Few tiles and long K (17408: 68 stages of 256 codes), with and without a
    workspace (integer mode needs none for 2-bit and 1-bit): both exact."""
    rng = np.random.default_rng(71)
    m, n, k = 40, 700, 17408
    codes = _codes(rng, n, k, fmt)
    x = rng.integers(-128, 128, (m, k)).astype(np.int8)
    ref = orc.linear_int(x, codes)
    assert np.array_equal(_run(fmt, codes, x, with_ws=True, path=GEMM), ref)
    assert np.array_equal(_run(fmt, codes, x, with_ws=False, path=GEMM), ref)


def test_int8_extreme_values():
    """Every activation -128 or 127 and every code +-1: the largest sums."""
    rng = np.random.default_rng(66)
    m, n, k = 32, 300, 17408
    codes = np.where(rng.random((n, k)) < 0.5, -1, 1).astype(np.int8)
    codes[0] = 1
    codes[1] = -1
    x = np.where(rng.random((m, k)) < 0.5, -128, 127).astype(np.int8)
    x[0] = -128
    for fmt in ("2bit", "1bit"):
        got = _run(fmt, codes, x, path=GEMM)
        assert np.array_equal(got, orc.linear_int(x, codes)), fmt


@pytest.mark.parametrize("fmt", ["2bit", "1bit"])
def test_int8_gemm_prefill_shape_sampled_rows(fmt):
    rng = np.random.default_rng(67)
    m, n, k = 2048, 17408, 5120
    codes = _codes(rng, n, k, fmt)
    x = rng.integers(-127, 128, (m, k)).astype(np.int8)
    got = _run(fmt, codes, x)
    rows = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 48)]))
    assert np.array_equal(got[:, rows], orc.linear_int(x, codes[rows]))


def test_base3_without_workspace_takes_the_plain_kernel():
    rng = np.random.default_rng(68)
    m, n, k = 32, 500, 1024
    codes = _codes(rng, n, k, "base3")
    x = rng.integers(-127, 128, (m, k)).astype(np.int8)
    got = _run("base3", codes, x, with_ws=False)
    assert np.array_equal(got, orc.linear_int(x, codes))
    got = _run("base3", codes, x, with_ws=True)
    assert np.array_equal(got, orc.linear_int(x, codes))


def test_int8_gemm_matches_plain_kernel():
    rng = np.random.default_rng(69)
    m, n, k = 40, 777, 2048
    codes = _codes(rng, n, k, "2bit")
    x = rng.integers(-128, 128, (m, k)).astype(np.int8)
    assert np.array_equal(_run("2bit", codes, x, path=GEMM), _run("2bit", codes, x, path=SIMPLE))
