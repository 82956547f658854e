"""The C ABI without a GPU: the library builds, loads, exports every symbol the
header declares, answers its pure host queries, and rejects bad arguments
with the documented status before touching the device."""
import ctypes

import pytest

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import build as tbbuild


@pytest.fixture(scope="module")
def lib():
    tbbuild.build()
    return tb.load()


def test_exports_every_header_symbol(lib):
    names = tb.header_functions()
    assert len(names) >= 11
    for name in names:
        assert hasattr(lib, name), name
    assert set(tb._SIGNATURES) == set(names)


def test_version_and_status_strings(lib):
    assert tb.tb_version() == 10000
    for st in range(9):
        assert tb.status_string(st)
    assert tb.status_string(99) == "unknown status"


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("n,k", [(1, 128), (3, 384), (256, 1024), (17408, 5120), (5120, 17408)])
def test_packed_bytes_matches_oracle(lib, fmt, n, k):
    assert tb.tb_packed_bytes(fmt, n, k) == orc.packed_bytes(fmt, n, k)


def test_packed_bytes_rejects(lib):
    assert tb.tb_packed_bytes("2bit", 4, 100) == 0
    assert tb.tb_packed_bytes("2bit", 0, 128) == 0
    assert tb.tb_packed_bytes(7, 4, 128) == 0


def test_workspace_query(lib):
    assert tb.tb_ternary_linear_workspace("2bit", 1, 17408, 5120) >= 4 * 5120
    assert tb.tb_ternary_linear_workspace("2bit", 2048, 17408, 5120) >= 4 * 2048 * 5120
    assert tb.tb_ternary_linear_workspace("2bit", 1, 17408, 5000) == 0
    assert tb.tb_ternary_linear_workspace(5, 1, 17408, 5120) == 0


FAKE = 0x10000  # a 16-byte aligned non-null value; never dereferenced (validation fails first)


def test_pack_validation(lib):
    f = tb.tb_pack_ternary
    assert f(9, FAKE, 4, 128, FAKE, check=False, stream=0) == tb.TB_ERR_FORMAT
    assert f("2bit", None, 4, 128, FAKE, check=False, stream=0) == tb.TB_ERR_NULL
    assert f("2bit", FAKE, 4, 128, None, check=False, stream=0) == tb.TB_ERR_NULL
    assert f("2bit", FAKE, 4, 100, FAKE, check=False, stream=0) == tb.TB_ERR_SHAPE
    assert f("2bit", FAKE, 0, 128, FAKE, check=False, stream=0) == tb.TB_ERR_SHAPE
    assert f("base3", FAKE + 1, 4, 128, FAKE, check=False, stream=0) == tb.TB_ERR_ALIGN
    g = tb.tb_unpack_ternary
    assert g("2bit", FAKE, 4, 128, FAKE + 8, check=False, stream=0) == tb.TB_ERR_ALIGN
    assert g(-1, FAKE, 4, 128, FAKE, check=False, stream=0) == tb.TB_ERR_FORMAT


def test_rotate_validation(lib):
    f = tb.tb_hadamard_rotate
    bf, h, f32 = tb.TB_BF16, tb.TB_FP16, tb.TB_FP32
    assert f(None, bf, FAKE, f32, FAKE, 1, 1024, check=False, stream=0) == tb.TB_ERR_NULL
    assert f(FAKE, bf, FAKE, f32, None, 1, 1024, check=False, stream=0) == tb.TB_ERR_NULL
    assert f(FAKE, tb.TB_INT8, FAKE, f32, FAKE, 1, 1024, check=False, stream=0) == tb.TB_ERR_DTYPE
    assert f(FAKE, bf, FAKE, tb.TB_INT32, FAKE, 1, 1024, check=False, stream=0) == tb.TB_ERR_DTYPE
    assert f(FAKE, bf, FAKE, f32, FAKE, 1, 1536, check=False, stream=0) == tb.TB_ERR_SHAPE
    assert f(FAKE, bf, FAKE, f32, FAKE, 0, 1024, check=False, stream=0) == tb.TB_ERR_SHAPE
    # in place needs the same dtype
    assert f(FAKE, bf, FAKE, h, FAKE, 1, 1024, check=False, stream=0) == tb.TB_ERR_DTYPE
    assert f(FAKE + 4, f32, FAKE + 4096, f32, FAKE, 1, 1024, check=False, stream=0) == tb.TB_ERR_ALIGN
    assert f(FAKE, f32, FAKE + 4096, f32, FAKE + 2, 1, 1024, check=False, stream=0) == tb.TB_ERR_ALIGN


def _lin(**kw):
    a = dict(x=FAKE, xt=tb.TB_BF16, packed=FAKE, scales=FAKE, fmt="2bit", m=1, n=256, k=1024,
             signs=FAKE, y=FAKE, yt=tb.TB_FP32, workspace=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return tb.tb_ternary_linear(a["x"], a["xt"], a["packed"], a["scales"], a["fmt"], a["m"], a["n"],
                                a["k"], a["signs"], a["y"], a["yt"], a["workspace"], a["ws_bytes"],
                                stream=0, check=False)


def test_linear_validation(lib):
    assert _lin(fmt=3) == tb.TB_ERR_FORMAT
    assert _lin(fmt=-1) == tb.TB_ERR_FORMAT
    assert _lin(x=None) == tb.TB_ERR_NULL
    assert _lin(packed=None) == tb.TB_ERR_NULL
    assert _lin(scales=None) == tb.TB_ERR_NULL
    assert _lin(y=None) == tb.TB_ERR_NULL
    assert _lin(k=1000) == tb.TB_ERR_SHAPE
    assert _lin(k=1152) == tb.TB_ERR_SHAPE          # rotation needs K % 1024
    assert _lin(m=0) == tb.TB_ERR_SHAPE
    assert _lin(n=0) == tb.TB_ERR_SHAPE
    assert _lin(xt=tb.TB_INT32) == tb.TB_ERR_DTYPE
    assert _lin(yt=tb.TB_FP16) == tb.TB_ERR_DTYPE
    assert _lin(xt=tb.TB_INT8, yt=tb.TB_FP32, signs=None) == tb.TB_ERR_DTYPE
    assert _lin(xt=tb.TB_INT8, yt=tb.TB_INT32) == tb.TB_ERR_DTYPE  # no rotation of integers
    assert _lin(workspace=None) == tb.TB_ERR_WORKSPACE
    assert _lin(ws_bytes=16) == tb.TB_ERR_WORKSPACE
    assert _lin(x=FAKE + 1) == tb.TB_ERR_ALIGN
    assert _lin(signs=FAKE + 4) == tb.TB_ERR_ALIGN
    assert _lin(fmt="base3", packed=FAKE + 1) == tb.TB_ERR_ALIGN


def test_path_selection(lib):
    p = tb.tb_ternary_linear_path
    assert p(tb.TB_BF16, "2bit", 1, 17408, 5120) == tb.TB_PATH_GEMV
    # one token with long K and few rows (down shape), and 2-16 tokens: the
    # tensor-core decode
    assert p(tb.TB_BF16, "2bit", 1, 5120, 17408) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "2bit", 2, 17408, 5120) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "2bit", 3, 5120, 17408) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "2bit", 4, 5120, 17408) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "2bit", 1, 256, 1152, has_signs=False) == tb.TB_PATH_SIMPLE
    assert p(tb.TB_BF16, "2bit", 1, 17408, 5120, aligned16=False) == tb.TB_PATH_SIMPLE
    assert p(tb.TB_INT8, "2bit", 4, 256, 1024, has_signs=False) == tb.TB_PATH_SIMPLE
    assert p(tb.TB_BF16, "2bit", 2048, 17408, 5120) == tb.TB_PATH_GEMM
    assert p(tb.TB_BF16, "2bit", 5, 256, 1024) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "2bit", 16, 5120, 17408) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "2bit", 17, 5120, 17408) == tb.TB_PATH_GEMM
    assert p(tb.TB_BF16, "base3", 1, 17408, 5120) == tb.TB_PATH_GEMV
    assert p(tb.TB_BF16, "base3", 7, 5120, 17408) == tb.TB_PATH_GEMV
    # 8-16 tokens: re-encoded to 2-bit slots, then the tensor-core decode
    assert p(tb.TB_BF16, "base3", 8, 5120, 17408) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "base3", 16, 5120, 17408) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "base3", 17, 5120, 17408) == tb.TB_PATH_GEMM
    assert p(tb.TB_BF16, "base3", 2048, 17408, 5120) == tb.TB_PATH_GEMM
    # more weight rows than 148 x 128: the tensor-core decode runs two row
    # tiles per CTA
    assert p(tb.TB_BF16, "base3", 16, 34816, 5120) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "base3", 8, 19000, 1024) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "2bit", 4, 34816, 5120) == tb.TB_PATH_GEMV_TC
    assert p(tb.TB_BF16, "2bit", 1, 34816, 5120) == tb.TB_PATH_GEMV
    assert p(tb.TB_BF16, "2bit", 1, 256, 1000) == -1


def test_fault_query_needs_pointer(lib):
    assert lib.tb_get_device_fault(None, 0) == tb.TB_ERR_NULL


def test_ctypes_signatures_are_set(lib):
    assert lib.tb_ternary_linear.restype is ctypes.c_int
    assert len(lib.tb_ternary_linear_ex.argtypes) == 15


def _noalloc_need(m, k):
    """Scratch the decode path may write for m tokens of width k: the CUDA-core
    decode's activation stages, and for one token the one-token kernel's
    activation words (280 bytes per 128-group)."""
    need = m * (2 * k + k // 16 + 8448)
    if m == 1:
        need = max(need, (k // 128) * 280)
    return need


@pytest.mark.parametrize("m", [1, 2, 3, 4])
def test_noalloc_size_check_covers_every_decode_path(lib, m):
    # An accepted size passes the scratch check and then stops at the
    # alignment check (y is 4- but not 16-byte aligned), so nothing reaches the
    # device; a rejected one returns TB_ERR_WORKSPACE.  The boundary must be
    # where the scratch of every kernel the decode path can pick still fits.
    limit = tb.TB_NOALLOC_SCRATCH_BYTES
    largest = 0
    for blocks in range(1, 300):
        k = 1024 * blocks
        st = tb.tb_ternary_linear_noalloc(FAKE, tb.TB_BF16, FAKE, FAKE, m, 256, k, FAKE, FAKE + 4,
                                          tb.TB_FP32, stream=0, check=False)
        fits = _noalloc_need(m, k) <= limit
        assert st == (tb.TB_ERR_ALIGN if fits else tb.TB_ERR_WORKSPACE), (m, k, st)
        if fits:
            largest = k
            assert (k // 128) * 280 <= limit or m > 1
    assert largest == {1: 269312, 2: 138240, 3: 91136, 4: 66560}[m]


def test_prepare_validation(lib):
    f = tb.tb_prepare_weights
    bf = tb.TB_BF16
    assert f(FAKE, bf, FAKE, 4, 1024, 9, FAKE, FAKE, stream=0, check=False) == tb.TB_ERR_FORMAT
    assert f(None, bf, FAKE, 4, 1024, "2bit", FAKE, FAKE, stream=0, check=False) == tb.TB_ERR_NULL
    assert f(FAKE, bf, FAKE, 4, 1024, "2bit", None, FAKE, stream=0, check=False) == tb.TB_ERR_NULL
    assert f(FAKE, bf, FAKE, 4, 1024, "2bit", FAKE, None, stream=0, check=False) == tb.TB_ERR_NULL
    assert f(FAKE, tb.TB_INT8, FAKE, 4, 1024, "2bit", FAKE, FAKE, stream=0, check=False) == tb.TB_ERR_DTYPE
    assert f(FAKE, bf, FAKE, 4, 1536, "2bit", FAKE, FAKE, stream=0, check=False) == tb.TB_ERR_SHAPE
    assert f(FAKE, bf, FAKE, 0, 1024, "base3", FAKE, FAKE, stream=0, check=False) == tb.TB_ERR_SHAPE
    assert f(FAKE + 2, bf, FAKE, 4, 1024, "2bit", FAKE, FAKE, stream=0, check=False) == tb.TB_ERR_ALIGN
    assert f(FAKE, bf, FAKE, 4, 1024, "2bit", FAKE + 8, FAKE, stream=0, check=False) == tb.TB_ERR_ALIGN
    assert f(FAKE, bf, FAKE + 4, 4, 1024, "2bit", FAKE, FAKE, stream=0, check=False) == tb.TB_ERR_ALIGN


@pytest.mark.parametrize("n,k", [(1, 128), (3, 384), (17408, 5120), (5120, 17408)])
def test_packed_bytes_1bit(lib, n, k):
    assert tb.tb_packed_bytes("1bit", n, k) == orc.packed_bytes("1bit", n, k) == n * k // 8


def test_path_selection_1bit(lib):
    p = tb.tb_ternary_linear_path
    assert p(tb.TB_BF16, "1bit", 1, 17408, 5120) == tb.TB_PATH_GEMV
    assert p(tb.TB_BF16, "1bit", 1, 5120, 17408) == tb.TB_PATH_GEMV
    assert p(tb.TB_BF16, "1bit", 2, 17408, 5120) == tb.TB_PATH_GEMM
    assert p(tb.TB_BF16, "1bit", 2048, 17408, 5120) == tb.TB_PATH_GEMM
    assert p(tb.TB_BF16, "1bit", 1, 256, 640, has_signs=False) == tb.TB_PATH_SIMPLE
    assert p(tb.TB_INT8, "1bit", 4, 256, 1024, has_signs=False) == tb.TB_PATH_SIMPLE
    assert p(tb.TB_BF16, "1bit", 1, 17408, 5120, aligned16=False) == tb.TB_PATH_SIMPLE


def test_path_selection_integer_mode(lib):
    p = tb.tb_ternary_linear_path
    # kind::i8 tensor-core GEMM from 16 tokens (any K % 128), else the plain kernel
    assert p(tb.TB_INT8, "2bit", 16, 256, 1024, has_signs=False) == tb.TB_PATH_GEMM
    assert p(tb.TB_INT8, "2bit", 15, 256, 1024, has_signs=False) == tb.TB_PATH_SIMPLE
    assert p(tb.TB_INT8, "2bit", 2048, 17408, 5120, has_signs=False) == tb.TB_PATH_GEMM
    assert p(tb.TB_INT8, "1bit", 2048, 17408, 640, has_signs=False) == tb.TB_PATH_GEMM
    assert p(tb.TB_INT8, "base3", 64, 17408, 5120, has_signs=False) == tb.TB_PATH_GEMM
    assert p(tb.TB_INT8, "2bit", 2048, 17408, 5120, has_signs=False, aligned16=False) == tb.TB_PATH_SIMPLE
