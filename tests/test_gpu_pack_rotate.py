"""GPU parity: packing, unpacking and the block rotation against the oracle.

Packing and unpacking are bit-exact (codes, bytes and invalid counts).  The
rotation in fp32 is within 1e-5 relative L2 per row of the fp64 oracle; fp16 /
bf16 outputs are within the output type's rounding."""
import numpy as np
import pytest
import torch

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import inputs
from tests.gpu_util import DEV, ensure_lib, pack_dev, to_dev_codes
from tests.tolerances import ROTATE_REL_L2, rotate_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    assert tb.tb_get_device_fault() == 0


# ------------------------------------------------------------------ packing

@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("n,k,p0,seed", [(256, 1024, 1 / 3, 0), (3, 384, 0.2, 5), (1, 128, 0.5, 6),
                                         (1001, 2048, 0.33, 7)])
def test_pack_unpack_bitexact(fmt, n, k, p0, seed):
    codes = inputs.draw_codes(np.random.default_rng(seed), n, k, p0)
    packed, cnt = pack_dev(fmt, to_dev_codes(codes), n, k)
    ref, bad = orc.pack(codes, fmt)
    assert int(cnt.item()) == bad == 0
    assert np.array_equal(packed.cpu().numpy().reshape(ref.shape), ref)
    back = torch.empty(n, k, dtype=torch.int8, device=DEV)
    cnt2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    tb.tb_unpack_ternary(fmt, packed, n, k, back, cnt2)
    assert int(cnt2.item()) == 0
    assert np.array_equal(back.cpu().numpy(), codes)


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_pack_full_size_sampled_rows(fmt):
    n, k = 17408, 5120
    codes = inputs.draw_codes(np.random.default_rng(1), n, k, 0.33)
    packed, cnt = pack_dev(fmt, to_dev_codes(codes), n, k)
    assert int(cnt.item()) == 0
    host = packed.cpu().numpy().reshape(n, -1)
    rows = np.r_[0:64, 8000:8064, n - 64:n]
    ref, _ = orc.pack(codes[rows], fmt)
    assert np.array_equal(host[rows], ref)


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_pack_counts_invalid_codes(fmt):
    n, k = 4, 256
    codes = inputs.draw_codes(np.random.default_rng(3), n, k, 0.3)
    codes[0, 5] = 2
    codes[1, 77] = -2
    codes[2, 255] = 127
    codes[3, 0] = -128
    packed, cnt = pack_dev(fmt, to_dev_codes(codes), n, k)
    ref, bad = orc.pack(codes, fmt)
    assert bad == 4 and int(cnt.item()) == 4
    assert np.array_equal(packed.cpu().numpy().reshape(ref.shape), ref)


def test_unpack_2bit_every_byte():
    n, k = 4, 1024  # 1024 bytes: every byte value four times
    raw = np.tile(np.arange(256, dtype=np.uint8), 4).reshape(n, k // 4)
    packed = torch.from_numpy(raw).to(DEV)
    out = torch.empty(n, k, dtype=torch.int8, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    tb.tb_unpack_ternary("2bit", packed, n, k, out, cnt)
    ref, bad = orc.unpack(raw, "2bit", n, k)
    assert int(cnt.item()) == bad
    assert np.array_equal(out.cpu().numpy(), ref)


def test_unpack_base3_every_byte_body_and_tail():
    rng = np.random.default_rng(4)
    n, k = 40, 1024
    g = k // 128
    raw = rng.integers(0, 243, size=(n, g * 26)).astype(np.uint8)
    # every byte value once in a body position and once in a tail position
    vals = np.arange(256, dtype=np.uint8)
    body_pos = [(i // 8, (i % 8) * 26 + (i % 25)) for i in range(256)]
    for v, (r, c) in zip(vals, body_pos):
        raw[r % n, c] = v
    for i, v in enumerate(vals):
        r, grp = divmod(i, g)
        raw[(r + 7) % n, grp * 26 + 25] = v
    packed = torch.from_numpy(raw).to(DEV)
    out = torch.empty(n, k, dtype=torch.int8, device=DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    tb.tb_unpack_ternary("base3", packed, n, k, out, cnt)
    ref, bad = orc.unpack(raw, "base3", n, k)
    assert bad > 0 and int(cnt.item()) == bad
    assert np.array_equal(out.cpu().numpy(), ref)


# ------------------------------------------------------------------ rotation

_TORCH = {tb.TB_BF16: torch.bfloat16, tb.TB_FP16: torch.float16, tb.TB_FP32: torch.float32}
_OUT_TOL = {tb.TB_FP32: ROTATE_REL_L2, tb.TB_FP16: 2.0 ** -10, tb.TB_BF16: 2.0 ** -7}


@pytest.mark.parametrize("xt", [tb.TB_BF16, tb.TB_FP16, tb.TB_FP32])
@pytest.mark.parametrize("yt", [tb.TB_FP32, tb.TB_FP16, tb.TB_BF16])
@pytest.mark.parametrize("inverse", [0, 1])
@pytest.mark.parametrize("m,k", [(1, 1024), (3, 5120), (2, 17408)])
def test_rotate_matches_oracle(xt, yt, inverse, m, k):
    rng = np.random.default_rng(10 + m + k)
    signs = inputs.draw_signs(rng, k)
    x = torch.randn(m, k, generator=torch.Generator().manual_seed(k + m)).to(_TORCH[xt])
    x_ref = x.double().numpy()
    xd = x.to(DEV)
    y = torch.empty(m, k, dtype=_TORCH[yt], device=DEV)
    tb.tb_hadamard_rotate(xd, xt, y, yt, to_dev_codes(signs), m, k, inverse)
    torch.cuda.synchronize()
    ref = orc.rotate(x_ref, signs, inverse=bool(inverse))
    err = rotate_rel_err(y.double().cpu().numpy(), ref)
    assert err <= _OUT_TOL[yt], err


@pytest.mark.parametrize("dt", [tb.TB_FP32, tb.TB_BF16])
def test_rotate_in_place_and_roundtrip(dt):
    m, k = 4, 3072
    signs = inputs.draw_signs(np.random.default_rng(2), k)
    s_dev = to_dev_codes(signs)
    x = torch.randn(m, k, generator=torch.Generator().manual_seed(1)).to(_TORCH[dt])
    buf = x.to(DEV).clone()
    tb.tb_hadamard_rotate(buf, dt, buf, dt, s_dev, m, k, 0)
    ref = orc.rotate(x.double().numpy(), signs)
    torch.cuda.synchronize()
    assert rotate_rel_err(buf.double().cpu().numpy(), ref) <= _OUT_TOL[dt]
    tb.tb_hadamard_rotate(buf, dt, buf, dt, s_dev, m, k, 1)
    torch.cuda.synchronize()
    tol = 1e-6 if dt == tb.TB_FP32 else 2.0 ** -6
    assert rotate_rel_err(buf.double().cpu().numpy(), x.double().numpy()) <= tol


def test_rotate_closed_form_unit_vector():
    k = 2048
    signs = np.ones(k, dtype=np.int8)
    x = torch.zeros(1, k, dtype=torch.float32, device=DEV)
    x[0, 0] = 1.0
    x[0, 1024] = 1.0
    y = torch.empty_like(x)
    tb.tb_hadamard_rotate(x, tb.TB_FP32, y, tb.TB_FP32, to_dev_codes(signs), 1, k, 0)
    torch.cuda.synchronize()
    assert torch.all(y.cpu() == 1.0 / 32)
