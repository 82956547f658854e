"""tb_ternary_linear_noalloc: the decode path for callers that cannot allocate
device memory (plugins inside a host runtime that owns every allocation,
decode loops that must not call cudaMalloc/cudaFree because those can
synchronise the device).  It keeps its activation scratch in a fixed array
inside the library instead of taking a workspace.

The test calls it through the C ABI twice in a row and compares each result
with the oracle's (sampled rows, fp64) and with tb_ternary_linear's on the same
inputs, within the float tolerance the other tests use.  It runs alone in a
fresh process as well as after the other tests (the entry point sets itself up
on its first call)."""
import numpy as np
import pytest
import torch

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import inputs
from tests.gpu_util import DEV, Problem, ensure_lib
from tests.tolerances import within_linear_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    yield


def _noalloc(prob, yt=tb.TB_FP32):
    y = torch.full((prob.m, prob.n), float("nan"), device=DEV,
                   dtype=torch.float32 if yt == tb.TB_FP32 else torch.bfloat16)
    tb.tb_ternary_linear_noalloc(prob.x, tb.TB_BF16, prob.packed, prob.scales, prob.m, prob.n,
                                 prob.k, prob.signs, y, yt)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [inputs.make_linear_inputs(1, 1, 17408, 5120, 0.33, outlier_rate=0.01),
             inputs.make_linear_inputs(2, 4, 5120, 17408, 0.5, "lognormal")]
    for p in cases:
        prob = Problem(p, "2bit")
        rows = np.unique(np.concatenate([[0, prob.n - 1], np.random.default_rng(5).integers(0, prob.n, 300)]))
        ref = orc.linear(p.x, p.codes[rows], p.scales[rows], p.signs)
        other = prob.linear(tb.TB_PATH_AUTO)
        for _ in range(2):  # two calls in a row share the same fixed scratch
            got = _noalloc(prob)
            assert np.isfinite(got).all()
            ok, rel, worst = within_linear_tolerance(got[:, rows], ref, p.scales, p.x)
            assert ok, (rel, worst)
            ok, rel, worst = within_linear_tolerance(got, other, p.scales, p.x)
            assert ok, (rel, worst)
    assert tb.tb_get_device_fault() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    m, n, k = 4, 8, 67584  # the first K past the limit at 4 tokens
    assert m * (2 * k + k // 16 + 8448) > tb.TB_NOALLOC_SCRATCH_BYTES
    x = torch.zeros(m, k, dtype=torch.bfloat16, device=DEV)
    packed = torch.zeros(n * k // 4, dtype=torch.uint8, device=DEV)
    scales = torch.zeros(n, k // 128, dtype=torch.int16, device=DEV)
    signs = torch.ones(k, dtype=torch.int8, device=DEV)
    y = torch.empty(m, n, device=DEV)
    st = tb.tb_ternary_linear_noalloc(x, tb.TB_BF16, packed, scales, m, n, k, signs, y,
                                      tb.TB_FP32, check=False)
    assert st == tb.TB_ERR_WORKSPACE
    st = tb.tb_ternary_linear_noalloc(x[:1, :5120], tb.TB_INT8, packed, scales, 1, n, 5120, None,
                                      y, tb.TB_INT32, check=False)
    assert st == tb.TB_ERR_DTYPE
