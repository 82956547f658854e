"""GPU parity on the synthetic 27B-class layer stack.

The stack's codes are generated on the device (counter-based SplitMix64, see
inputs.py); the oracle regenerates sampled rows on the host and computes those
rows of y in fp64.

Every cell of the stack workload is covered: the seven matrices of a layer
(q, k, v, o, gate, up, down), zero fractions 0.2, 0.33 and 0.5, token counts
1, 4, 16, 64 and 512, both packings.  Each zero fraction takes a different
layer (first, last, middle).  One test per (matrix, zero fraction) runs all
ten (tokens, packing) cells on one set of codes and reports every failing
cell.

The shared-input calls (q|k|v and gate|up stacked along N, one call and one
rotation per input: the inverse rotation belongs to the layer's input,
news.ditty.ir, third paragraph) are checked sub-matrix by sub-matrix."""
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
P0_LAYER = {0.2: 0, 0.33: 63, 0.5: 31}
MS = (1, 4, 16, 64, 512)
FMTS = ("2bit", "base3")
N_SAMPLE = 40

_XCACHE = {}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    assert tb.tb_get_device_fault() == 0


def _inputs(m, k):
    """The stack's activations of width k at m tokens: device bf16, device
    signs, exact float64 values and the oracle's rotation x' = R^T x."""
    if (m, k) not in _XCACHE:
        xb, sg = inputs.stack_activations(SEED, m, k)
        xf = inputs.float_from_bf16_bits(xb).astype(np.float64)
        _XCACHE[(m, k)] = (torch.from_numpy(xb.view(np.int16)).to(DEV).view(torch.bfloat16),
                           torch.from_numpy(sg).to(DEV), xf, orc.rotate(xf, sg))
    return _XCACHE[(m, k)]


def _sample_rows(n, salt):
    return np.unique(np.concatenate([[0, n - 1], np.random.default_rng(salt).integers(0, n, N_SAMPLE)]))


def _run(fmt, packed, scales_dev, m, n, k):
    x, signs, _, _ = _inputs(m, k)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    wsb = tb.tb_ternary_linear_workspace(fmt, m, n, k)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    tb.tb_ternary_linear(x, tb.TB_BF16, packed, scales_dev, fmt, m, n, k, signs, y, tb.TB_FP32, ws, wsb)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("p0", sorted(P0_LAYER))
@pytest.mark.parametrize("name", [s[0] for s in inputs.STACK_LAYER_SHAPES])
def test_stack_matrix_every_cell(name, p0):
    n, k = SHAPES[name]
    j = MAT[name]
    layer = P0_LAYER[p0]
    codes = inputs.stack_codes_torch(SEED, layer, j, n, k, p0, DEV)
    packed = {}
    for f in FMTS:
        packed[f] = torch.empty(tb.tb_packed_bytes(f, n, k), dtype=torch.uint8, device=DEV)
        tb.tb_pack_ternary(f, codes, n, k, packed[f])
    del codes
    sc = inputs.stack_scales(SEED, layer, j, n, k)
    sc_dev = torch.from_numpy(sc.view(np.int16)).to(DEV)
    rows = _sample_rows(n, layer * 7 + j)
    sub = inputs.stack_codes_rows_np(SEED, layer, j, rows, k, p0)
    failures = []
    for m in MS:
        _, _, xf, xr = _inputs(m, k)
        ref = orc.linear(xr, sub, sc[rows])  # x already rotated by the oracle
        for f in FMTS:
            got = _run(f, packed[f], sc_dev, m, n, k)[:, rows]
            ok, rel, worst = within_linear_tolerance(got, ref, sc, xf)
            path = tb.tb_ternary_linear_path(tb.TB_BF16, f, m, n, k, True, True)
            if not ok:
                failures.append(f"{f} M={m} path={path}: rel_l2={rel:.3e} worst={worst:.3f}")
    assert not failures, "; ".join(failures)


FUSED = {"qkv": ("q", "k", "v"), "gateup": ("gate", "up")}


def fused_weights(fmt, layer, names, p0):
    """Packed codes and scales of the named matrices of one layer stacked
    along N in one buffer each (rows are independent in every format, so
    stacking the packed rows is stacking the matrices)."""
    k = SHAPES[names[0]][1]
    ntot = sum(SHAPES[nm][0] for nm in names)
    packed = torch.empty(tb.tb_packed_bytes(fmt, ntot, k), dtype=torch.uint8, device=DEV)
    scs = []
    off_b = 0
    for nm in names:
        n = SHAPES[nm][0]
        codes = inputs.stack_codes_torch(SEED, layer, MAT[nm], n, k, p0, DEV)
        nb = tb.tb_packed_bytes(fmt, n, k)
        tb.tb_pack_ternary(fmt, codes, n, k, packed[off_b:off_b + nb])
        off_b += nb
        scs.append(inputs.stack_scales(SEED, layer, MAT[nm], n, k))
    return packed, np.concatenate(scs, axis=0), ntot, k


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("group", sorted(FUSED))
def test_stack_shared_input_call(group, fmt):
    names = FUSED[group]
    layer, p0 = 17, 0.33
    packed, sc, ntot, k = fused_weights(fmt, layer, names, p0)
    sc_dev = torch.from_numpy(sc.view(np.int16)).to(DEV)
    failures = []
    for m in MS:
        _, _, xf, xr = _inputs(m, k)
        got = _run(fmt, packed, sc_dev, m, ntot, k)
        off = 0
        for nm in names:
            n = SHAPES[nm][0]
            rows = _sample_rows(n, 100 + MAT[nm])
            sub = inputs.stack_codes_rows_np(SEED, layer, MAT[nm], rows, k, p0)
            s_nm = inputs.stack_scales(SEED, layer, MAT[nm], n, k)
            ref = orc.linear(xr, sub, s_nm[rows])
            ok, rel, worst = within_linear_tolerance(got[:, off + rows], ref, s_nm, xf)
            if not ok:
                failures.append(f"{nm} M={m}: rel_l2={rel:.3e} worst={worst:.3f}")
            off += n
    assert not failures, "; ".join(failures)
