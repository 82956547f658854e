"""GPU parity of tb_prepare_weights, the producer side (fold the rotation into
a dense W, round each 128-group to ternary with an fp16 mean-|w'| scale, pack;
openbonsai.org, "How it works", steps 1 "Rotate" and 2 "Round"), against the
oracle's prepare_weights / ternarize on the same input values.

The kernel folds, sums and divides in fp64 and rounds the scale once to fp16.
On these inputs every fp64 sum is exact (bf16 and fp16 values; fp32 values on
a 2^-20 grid), so codes, scales and packed bytes must equal the oracle's bit
for bit, including the hand-worked groups of tests/golden/ternarize_groups.txt
(an fp16 scale that turns 0.5 ties into 0.50012, a tie that rounds to even,
clipping, an all-zero group)."""
import numpy as np
import pytest
import torch

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import inputs
from tests.conftest import golden_rows
from tests.gpu_util import DEV, ensure_lib
from tests.tolerances import within_linear_tolerance

pytestmark = pytest.mark.gpu

WT = {"bf16": (tb.TB_BF16, torch.bfloat16), "fp16": (tb.TB_FP16, torch.float16), "fp32": (tb.TB_FP32, torch.float32)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    assert tb.tb_get_device_fault() == 0


def _prepare(w, code, signs, n, k, fmt):
    packed = torch.zeros(tb.tb_packed_bytes(fmt, n, k), dtype=torch.uint8, device=DEV)
    scales = torch.zeros(n, k // 128, dtype=torch.int16, device=DEV)
    sd = torch.from_numpy(signs).to(DEV) if signs is not None else None
    tb.tb_prepare_weights(w.to(DEV), code, sd, n, k, fmt, packed, scales)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), scales.cpu().numpy().view(np.float16)


def _dense(rng, n, k, wt):
    v = rng.standard_normal((n, k)) * 0.02
    if wt == "fp32":
        v = np.round(v * 2.0 ** 20) / 2.0 ** 20  # exact fp32 values on a 2^-20 grid
    w = torch.from_numpy(v).to(WT[wt][1])
    w[7, :128] = 0  # an all-zero group
    w[11, 1024:1152] = 0
    return w


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("wt", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("folded", [False, True])
def test_prepare_bitexact_against_oracle(fmt, wt, folded):
    rng = np.random.default_rng(40)
    n, k = 301, 3072
    w = _dense(rng, n, k, wt)
    wv = w.double().numpy()  # the exact input values
    signs = None if folded else inputs.draw_signs(rng, k)
    packed, got_s = _prepare(w, WT[wt][0], signs, n, k, fmt)
    ref_codes, ref_s = orc.ternarize(wv) if folded else orc.prepare_weights(wv, signs)
    assert np.array_equal(got_s.view(np.uint16), ref_s.view(np.uint16)), "scales differ"
    ref_packed, bad = orc.pack(ref_codes, fmt)
    assert bad == 0
    assert np.array_equal(packed.reshape(ref_packed.shape), ref_packed), "packed codes differ"
    got_codes, bad = orc.unpack(packed, fmt, n, k)
    assert bad == 0 and np.array_equal(got_codes, ref_codes)
    assert got_s[7, 0] == 0 or not folded


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_prepare_golden_groups(fmt):
    rows = golden_rows("ternarize_groups.txt")
    groups = []
    for r in rows:
        bar = r.index("|")
        w4 = [float(v) for v in r[:bar]]
        s = float(r[bar + 1])
        t4 = [int(v) for v in r[bar + 3:]]
        groups.append((w4, s, t4))
    assert len(groups) == 7
    k = 1024
    w = np.zeros((1, k))
    for g, (w4, _, _) in enumerate(groups):
        w[0, 128 * g:128 * (g + 1)] = np.tile(w4, 32)
    wt = torch.from_numpy(w).to(torch.float32)
    packed, got_s = _prepare(wt, tb.TB_FP32, None, 1, k, fmt)
    codes, bad = orc.unpack(packed, fmt, 1, k)
    assert bad == 0
    ref_codes, ref_s = orc.ternarize(wt.double().numpy())
    assert np.array_equal(got_s.view(np.uint16), ref_s.view(np.uint16))
    assert np.array_equal(codes, ref_codes)
    for g, (_, s, t4) in enumerate(groups):
        assert float(got_s[0, g]) == s, (g, float(got_s[0, g]), s)
        assert list(codes[0, 128 * g:128 * g + 4]) == t4, g
        assert np.array_equal(codes[0, 128 * g:128 * (g + 1)], np.tile(t4, 32))
    assert got_s[0, 7] == 0 and not codes[0, 896:].any()


def test_prepare_then_linear_uses_the_same_layer():
    """Prepared on the GPU, the layer computes what the oracle computes with
    the GPU's codes and scales (the linear paths are covered elsewhere)."""
    rng = np.random.default_rng(41)
    n, k, m = 512, 2048, 1
    w = torch.from_numpy(rng.standard_normal((n, k)) * 0.02).to(torch.bfloat16)
    signs = inputs.draw_signs(rng, k)
    packed = torch.zeros(tb.tb_packed_bytes("2bit", n, k), dtype=torch.uint8, device=DEV)
    scales = torch.zeros(n, k // 128, dtype=torch.int16, device=DEV)
    sd = torch.from_numpy(signs).to(DEV)
    tb.tb_prepare_weights(w.to(DEV), tb.TB_BF16, sd, n, k, "2bit", packed, scales)
    x = torch.from_numpy(rng.standard_normal((m, k))).to(torch.bfloat16)
    y = torch.empty(m, n, dtype=torch.float32, device=DEV)
    wsb = tb.tb_ternary_linear_workspace("2bit", m, n, k)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    tb.tb_ternary_linear(x.to(DEV), tb.TB_BF16, packed, scales, "2bit", m, n, k, sd, y, tb.TB_FP32, ws, wsb)
    torch.cuda.synchronize()
    codes, _ = orc.unpack(packed.cpu().numpy(), "2bit", n, k)
    s = scales.cpu().numpy().view(np.float16)
    ref = orc.linear(x.double().numpy(), codes, s, signs)
    ok, rel, worst = within_linear_tolerance(y.cpu().numpy().astype(np.float64), ref, s, x.double().numpy())
    assert ok, (rel, worst)
    # and it approximates the dense layer it came from (ternary rounding error, loose)
    dense = x.double().numpy() @ w.double().numpy().T
    assert np.linalg.norm(y.cpu().numpy() - dense) / np.linalg.norm(dense) < 0.7
