"""Failure detection on the GPU without a fault: a bounded wait that runs out.

With the library's test hook set, the weight-copy producers of the one-token
decode kernel and of the fp16 GEMM issue nothing (a flag that nothing sets),
so every consumer's wait runs out after a short limit.  The call must return,
the device fault word must say that a consumer gave up waiting for a stage
(code 1), and once the hook is cleared the next call on the same context must
match the oracle again (the GEMM freed its tensor memory on the way out)."""
import numpy as np
import pytest

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import inputs
from tests.gpu_util import Problem, ensure_lib
from tests.tolerances import within_linear_tolerance

pytestmark = pytest.mark.gpu

FAULT_WAIT_FULL = 1
LIMIT_NS = 20_000_000  # 20 ms


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    tb.tb_test_stall_copies(0, 0)
    tb.tb_get_device_fault(clear=True)


@pytest.mark.parametrize("path,m,n,k", [(tb.TB_PATH_GEMV, 1, 17408, 5120),    # one-token decode, rotation fused
                                        (tb.TB_PATH_GEMV, 1, 10000, 9216),    # activation kernel, then decode
                                        (tb.TB_PATH_GEMM, 64, 6144, 5120)])   # fp16 GEMM (TMEM)
def test_wait_runs_out_and_next_call_is_correct(path, m, n, k):
    p = inputs.make_linear_inputs(120 + m, m, n, k, 0.33)
    prob = Problem(p, "2bit")
    ref = orc.linear(p.x, p.codes, p.scales, p.signs)
    tb.tb_get_device_fault(clear=True)
    tb.tb_test_stall_copies(1, LIMIT_NS)
    try:
        prob.linear(path)  # returns: every wait is bounded
        code = tb.tb_get_device_fault(clear=True)
    finally:
        tb.tb_test_stall_copies(0, 0)
    assert code == FAULT_WAIT_FULL, code
    for _ in range(2):
        y = prob.linear(path)
        ok, rel, worst = within_linear_tolerance(y, ref, p.scales, p.x)
        assert ok, (rel, worst)
    assert tb.tb_get_device_fault() == 0
