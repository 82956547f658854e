"""The synthetic layer stack's counter-based code generator (CPU).

The stack's 21.8 G codes are generated where they are used (on the GPU, with
torch) and regenerated on the host for sampled rows (numpy) when the oracle
checks a layer, so the two evaluations must agree bit for bit.  The generator
itself is pinned to the published SplitMix64 test vector."""
import numpy as np
import torch

from ternary_weight_signed_b200 import inputs


def test_splitmix64_published_vector():
    # SplitMix64 with state 1234567: the first five outputs of the reference
    # implementation (Steele, Lea, Flood 2014; the vector used by its ports)
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    assert [inputs._splitmix64_py(1234567, i) for i in range(5)] == want


def test_numpy_torch_and_scalar_agree():
    rows = [0, 3, 17, 64]
    k = 256
    a = inputs.stack_codes_rows_np(4, 63, 6, rows, k, 0.33)
    b = inputs.stack_codes_torch(4, 63, 6, 65, k, 0.33, "cpu", rows_per_chunk=7).numpy()[rows]
    assert np.array_equal(a, b)
    s = inputs.stack_state(4, 63, 6)
    lo, mid = (1 - 0.33) / 2, (1 - 0.33) / 2 + 0.33
    for r in rows:
        for kk in (0, 1, 255):
            u = (inputs._splitmix64_py(s, r * k + kk) >> 11) / 2.0**53
            t = -1 if u < lo else (0 if u < mid else 1)
            assert a[rows.index(r), kk] == t


def test_matrices_differ_and_distribution_matches():
    a = inputs.stack_codes_rows_np(4, 0, 0, range(64), 1024, 0.5)
    b = inputs.stack_codes_rows_np(4, 1, 0, range(64), 1024, 0.5)
    c = inputs.stack_codes_rows_np(4, 0, 1, range(64), 1024, 0.5)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    frac = np.bincount((a.ravel() + 1).astype(int), minlength=3) / a.size
    assert abs(frac[1] - 0.5) < 0.01 and abs(frac[0] - 0.25) < 0.01 and abs(frac[2] - 0.25) < 0.01


def test_torch_wraparound_matches_uint64():
    # int64 products wrap modulo 2^64 in torch, which is what SplitMix64 needs
    x = torch.tensor([inputs._i64(0xFFFFFFFFFFFFFFFF), 3], dtype=torch.int64)
    y = x * inputs._i64(inputs._SM_M1)
    want = [(0xFFFFFFFFFFFFFFFF * inputs._SM_M1) & inputs._U64, (3 * inputs._SM_M1) & inputs._U64]
    assert [v & inputs._U64 for v in y.tolist()] == want
