"""Chained calls on one stream, each call's input the previous call's output.

The decode kernels let the next kernel on the stream start early (programmatic
dependent launch) and read only the layer's packed weights, scales and signs
before they wait for the kernel ahead of them; activations, outputs and the
shared workspace are touched after that wait.  A chain x -> y -> x -> ...
issued back to back (ping-pong buffers, one workspace) must therefore give,
bit for bit, what the same chain gives with the host synchronising after every
call.  Every kernel path is covered, with the shapes that select it."""
import numpy as np
import pytest
import torch

from ternary_weight_signed_b200 import binding as tb
from ternary_weight_signed_b200 import inputs
from tests.gpu_util import DEV, ensure_lib, pack_dev, to_dev_codes, to_dev_scales

pytestmark = pytest.mark.gpu

STEPS = 6

# format, tokens M, K (= N, so that y can be the next x), x/y dtype, path
# asked for, and whether it is also the automatic choice
CASES = [
    ("2bit", 1, 5120, "bf16", tb.TB_PATH_GEMV, True),     # one launch, rotation inside
    ("2bit", 1, 5120, "fp32", tb.TB_PATH_GEMV, True),
    ("2bit", 1, 10240, "bf16", tb.TB_PATH_GEMV, True),    # activation kernel, then decode
    ("2bit", 2, 5120, "bf16", tb.TB_PATH_GEMV, False),    # CUDA-core decode for two tokens
    ("2bit", 2, 5120, "bf16", tb.TB_PATH_GEMV_TC, True),
    ("2bit", 4, 5120, "bf16", tb.TB_PATH_GEMV_TC, True),
    ("2bit", 16, 5120, "bf16", tb.TB_PATH_GEMV_TC, True),
    ("2bit", 64, 5120, "bf16", tb.TB_PATH_GEMM, True),
    ("base3", 1, 5120, "bf16", tb.TB_PATH_GEMV, True),
    ("base3", 8, 5120, "bf16", tb.TB_PATH_GEMV_TC, True),
    ("1bit", 1, 5120, "bf16", tb.TB_PATH_GEMV, True),
    ("1bit", 4, 5120, "bf16", tb.TB_PATH_GEMM, True),
]

DT = {"bf16": (tb.TB_BF16, torch.bfloat16), "fp32": (tb.TB_FP32, torch.float32)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()
    tb.tb_get_device_fault(clear=True)
    yield
    assert tb.tb_get_device_fault() == 0


def _chain(x0, layers, fmt, m, k, code, nbuf, sync, path):
    """STEPS calls, call i on layer i % 2 from buffer i % nbuf into buffer
    (i + 1) % nbuf: nbuf = 2 is a ping-pong (each call also overwrites what the
    call before it read), nbuf = STEPS + 1 keeps every output.  Nothing but the
    library's kernels runs on the stream in between.  Returns all buffers."""
    bufs = [x0.clone()] + [torch.zeros_like(x0) for _ in range(nbuf - 1)]
    ws_bytes = tb.tb_ternary_linear_workspace(fmt, m, k, k)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=DEV)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    for i in range(STEPS):
        packed, scales, signs = layers[i % 2]
        x, y = bufs[i % nbuf], bufs[(i + 1) % nbuf]
        tb.tb_ternary_linear_ex(x, code, packed, scales, fmt, m, k, k, signs, y, code, ws, ws_bytes, path,
                                stream=stream.cuda_stream)
        if sync:
            stream.synchronize()
    stream.synchronize()
    return [b.float().cpu().numpy() for b in bufs]


@pytest.mark.parametrize("fmt,m,k,dtype,path,auto", CASES)
def test_chain_matches_synchronised_chain(fmt, m, k, dtype, path, auto):
    code, tdt = DT[dtype]
    assert (tb.tb_ternary_linear_path(code, fmt, m, k, k) == path) == auto
    layers = []
    for seed in (71, 72):
        p = inputs.make_linear_inputs(seed, m, k, k, 0.0 if fmt == "1bit" else 0.33, "abs_normal", 0.01)
        packed, cnt = pack_dev(fmt, to_dev_codes(p.codes), k, k)
        assert int(cnt.item()) == 0
        layers.append((packed, to_dev_scales(p.scales), to_dev_codes(p.signs)))
        if seed == 71:
            x0 = torch.from_numpy(p.x).to(DEV).to(tdt)  # x drawn in float64, rounded like the bf16 inputs
    for nbuf in (STEPS + 1, 2):
        free = _chain(x0, layers, fmt, m, k, code, nbuf, False, path)
        ref = _chain(x0, layers, fmt, m, k, code, nbuf, True, path)
        for i, (a, b) in enumerate(zip(free, ref)):
            assert np.all(np.isfinite(b)) and np.any(b != 0), f"buffer {i}: degenerate output"
            np.testing.assert_array_equal(a, b, err_msg=f"{nbuf} buffers: buffer {i} differs from the "
                                          "synchronised chain")
