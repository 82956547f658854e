"""GPU parity on the synthetic 27B-class layer stack.

The stack's codes are generated on the device (counter-based SplitMix64, see
inputs.py); the oracle regenerates sampled rows on the host and computes those
rows of y in fp64.  First and last layer, the narrowest (k projection) and
widest-K (down) shapes, decode and prefill token counts, both packings."""
import numpy as np
import pytest
import torch

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import inputs
from tests.gpu_util import DEV, ensure_lib
from tests.tolerances import within_linear_tolerance

pytestmark = pytest.mark.gpu

SEED = 4
SHAPES = dict((name, (n, k)) for name, n, k in inputs.STACK_LAYER_SHAPES)
MAT = dict((name, j) for j, (name, _, _) in enumerate(inputs.STACK_LAYER_SHAPES))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    assert tb.tb_get_device_fault() == 0


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
@pytest.mark.parametrize("m", [1, 16, 64])
@pytest.mark.parametrize("layer,name", [(0, "k"), (63, "down")])
def test_stack_layer_sampled_rows(layer, name, m, fmt):
    n, k = SHAPES[name]
    j = MAT[name]
    p0 = 0.33
    codes = inputs.stack_codes_torch(SEED, layer, j, n, k, p0, DEV)
    packed = torch.empty(tb.tb_packed_bytes(fmt, n, k), dtype=torch.uint8, device=DEV)
    tb.tb_pack_ternary(fmt, codes, n, k, packed)
    del codes
    sc = inputs.stack_scales(SEED, layer, j, n, k)
    xb, sg = inputs.stack_activations(SEED, m, k)
    x = torch.from_numpy(xb.view(np.int16)).to(DEV).view(torch.bfloat16)
    signs = torch.from_numpy(sg).to(DEV)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    wsb = tb.tb_ternary_linear_workspace(fmt, m, n, k)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    tb.tb_ternary_linear(x, tb.TB_BF16, packed, torch.from_numpy(sc.view(np.int16)).to(DEV), fmt, m, n, k, signs,
                         y, tb.TB_FP32, ws, wsb)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, n - 1], np.random.default_rng(layer * 7 + m).integers(0, n, 40)]))
    sub = inputs.stack_codes_rows_np(SEED, layer, j, rows, k, p0)
    xf = inputs.float_from_bf16_bits(xb).astype(np.float64)
    ref = orc.linear(xf, sub, sc[rows], sg)
    got = y.cpu().numpy().astype(np.float64)[:, rows]
    ok, rel, worst = within_linear_tolerance(got, ref, sc, xf)
    assert ok, f"rel_l2={rel:.3e} worst={worst:.3f}"
