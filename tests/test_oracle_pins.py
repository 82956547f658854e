"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources of truth used here: hand-derived byte tables from the format
definitions (tests/golden), the textbook Sylvester construction and its closed
form H[i, j] = (-1)^popcount(i & j), scipy's Hadamard routine, an in-test
fast Walsh-Hadamard transform written as plain loops, brute-force integer sums,
and the add/subtract formulation of the ternary product (ai4coding.ru, "What is
a ternary model").
"""
import math

import numpy as np
import pytest
import scipy.linalg

from oracle import ternary_oracle as orc
from ternary_weight_signed_b200 import inputs
from tests.tolerances import within_linear_tolerance

H1024 = orc.sylvester_hadamard(1024)


# ----------------------------------------------------------------- Hadamard

def test_small_hadamard_matches_textbook(golden):
    rows = golden("hadamard_small.txt")
    mats, cur = {}, None
    for r in rows:
        if r[0].startswith("H"):
            cur = r[0]
            mats[cur] = []
        else:
            mats[cur].append([int(v) for v in r])
    assert np.array_equal(orc.sylvester_hadamard(2), np.array(mats["H2"]))
    assert np.array_equal(orc.sylvester_hadamard(4), np.array(mats["H4"]))


def test_hadamard_closed_form():
    i = np.arange(1024)[:, None]
    j = np.arange(1024)[None, :]
    pop = np.vectorize(lambda v: bin(v).count("1"))(i & j)
    assert np.array_equal(H1024, np.where(pop % 2 == 0, 1, -1))


def test_hadamard_orthogonal_integer():
    assert np.array_equal(H1024 @ H1024.T, 1024 * np.eye(1024, dtype=np.int64))


def test_hadamard_equals_scipy():
    assert np.array_equal(H1024, scipy.linalg.hadamard(1024))


def test_rotation_block_orthonormal():
    d = inputs.draw_signs(np.random.default_rng(5), 1024)
    r = orc.rotation_matrix(d)
    assert np.abs(r @ r.T - np.eye(1024)).max() < 1e-12


# ----------------------------------------------------------------- rotation

def _fwht_loops(v):
    """Unnormalised natural-order fast Walsh-Hadamard transform, plain loops."""
    a = list(v)
    h = 1
    n = len(a)
    while h < n:
        for start in range(0, n, 2 * h):
            for i in range(start, start + h):
                u, w = a[i], a[i + h]
                a[i], a[i + h] = u + w, u - w
        h *= 2
    return np.array(a)


def test_rotate_special_cases():
    ones = np.ones(1024, dtype=np.int8)
    e0 = np.zeros((1, 1024))
    e0[0, 0] = 1.0
    assert np.array_equal(orc.rotate(e0, ones), np.full((1, 1024), 1.0 / 32))
    d = inputs.draw_signs(np.random.default_rng(1), 1024)
    x = d[None, :].astype(np.float64)
    expect = np.zeros((1, 1024))
    expect[0, 0] = 32.0
    assert np.abs(orc.rotate(x, d) - expect).max() < 1e-12


def test_rotate_unit_vectors_closed_form():
    d = inputs.draw_signs(np.random.default_rng(2), 1024)
    for j in (0, 1, 77, 512, 1023):
        x = np.zeros((1, 1024))
        x[0, j] = 1.0
        got = orc.rotate(x, d)[0]
        i = np.arange(1024)
        pop = np.array([bin(v).count("1") for v in (i & j)])
        expect = d[j] * np.where(pop % 2 == 0, 1.0, -1.0) / 32.0
        assert np.abs(got - expect).max() < 1e-15


def test_rotate_matches_loop_fwht_with_signs():
    rng = np.random.default_rng(3)
    k = 2048
    d = inputs.draw_signs(rng, k)
    x = rng.standard_normal((2, k))
    got = orc.rotate(x, d)
    for m in range(2):
        for b in range(k // 1024):
            sl = slice(1024 * b, 1024 * (b + 1))
            ref = _fwht_loops(d[sl] * x[m, sl]) / 32.0
            assert np.abs(got[m, sl] - ref).max() < 1e-12
    back = orc.rotate(got, d, inverse=True)
    assert np.abs(back - x).max() < 1e-12
    # inverse = signs after the transform
    for b in range(k // 1024):
        sl = slice(1024 * b, 1024 * (b + 1))
        ref_inv = d[sl] * _fwht_loops(x[0, sl]) / 32.0
        assert np.abs(orc.rotate(x[:1], d, inverse=True)[0, sl] - ref_inv).max() < 1e-12


def test_rotate_preserves_norm_and_blocks_independent():
    rng = np.random.default_rng(4)
    d = inputs.draw_signs(rng, 3072)
    x = rng.standard_normal((3, 3072))
    y = orc.rotate(x, d)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    x2 = x.copy()
    x2[:, 1024:2048] += 1.0
    y2 = orc.rotate(x2, d)
    assert np.array_equal(y2[:, :1024], y[:, :1024])
    assert np.array_equal(y2[:, 2048:], y[:, 2048:])


def test_fold_invariant():
    """(R^T x) . (W R)^T = x . W^T for a dense W (R orthogonal)."""
    rng = np.random.default_rng(6)
    k, n = 2048, 64
    d = inputs.draw_signs(rng, k)
    w = rng.standard_normal((n, k))
    x = rng.standard_normal((3, k))
    # row n of W R is (R^T w_n)^T, i.e. the forward transform of w_n
    w_folded = orc.rotate(w, d)
    lhs = orc.rotate(x, d) @ w_folded.T
    rhs = x @ w.T
    assert np.abs(lhs - rhs).max() < 1e-11 * np.abs(rhs).max()


def test_fold_weights_definition_matches_row_transform():
    """W R block by block equals applying R^T to every row (the fold invariant's
    form), and (R^T x) . (W R)^T = x . W^T."""
    rng = np.random.default_rng(16)
    k, n = 2048, 16
    d = inputs.draw_signs(rng, k)
    w = rng.standard_normal((n, k))
    x = rng.standard_normal((2, k))
    wf = orc.fold_weights(w, d)
    assert np.abs(wf - orc.rotate(w, d)).max() < 1e-12
    assert np.abs(orc.rotate(x, d) @ wf.T - x @ w.T).max() < 1e-11 * np.abs(x @ w.T).max()


# ----------------------------------------------------------------- producer side

def test_ternarize_worked_groups(golden):
    rows = golden("ternarize_groups.txt")
    for r in rows:
        bar1, bar2 = r.index("|"), r.index("|", r.index("|") + 1)
        pat = np.array([float(v) for v in r[:bar1]])
        want_s = float(r[bar1 + 1])
        want_t = np.array([int(v) for v in r[bar2 + 1:]], dtype=np.int8)
        codes, scales = orc.ternarize(np.tile(pat, 32)[None, :])
        assert scales.dtype == np.float16 and float(scales[0, 0]) == want_s, (pat, scales[0, 0])
        assert np.array_equal(codes[0], np.tile(want_t, 32)), (pat, codes[0, :4])


def test_ternarize_recovers_scaled_ternary_groups():
    """w = c * t per group (t ternary with a fraction f of nonzeros, c > 0):
    mean |w| = c f, every |w / s| is 0 or 1 / f >= 1, so the codes come back
    exactly and the scale is fp16(c f)."""
    rng = np.random.default_rng(17)
    n, k = 6, 1024
    t = inputs.draw_codes(rng, n, k, 0.4)
    t[0, :128] = 0  # an all-zero group
    c = np.exp2(rng.integers(-6, 3, size=(n, k // 128))).astype(np.float64)
    w = t * np.repeat(c, 128, axis=1)
    codes, scales = orc.ternarize(w)
    assert np.array_equal(codes, t)
    f = np.abs(t).reshape(n, k // 128, 128).mean(axis=2)
    assert np.array_equal(scales, (c * f).astype(np.float16))
    assert scales[0, 0] == 0


def test_ternarize_symmetries():
    rng = np.random.default_rng(18)
    w = rng.standard_normal((4, 512))
    codes, scales = orc.ternarize(w)
    c2, s2 = orc.ternarize(-w)
    assert np.array_equal(c2, -codes) and np.array_equal(s2, scales)
    c3, s3 = orc.ternarize(8.0 * w)  # a power of two: every fp16 scale scales exactly
    assert np.array_equal(c3, codes) and np.array_equal(s3, (8 * scales.astype(np.float64)).astype(np.float16))


def test_prepare_weights_inverts_an_unfolded_ternary_layer():
    """Start from ternary codes and power-of-two scales as the folded layer
    W', unfold it (W = W' R^T), and prepare W: the fold must give W' back and
    the rounding its codes and scales (all groups dense, so s = c exactly).  A
    fold with R^T instead of R, or a missing sign, gives other codes."""
    rng = np.random.default_rng(19)
    n, k = 5, 2048
    d = inputs.draw_signs(rng, k)
    t = rng.choice(np.array([-1, 1], dtype=np.int8), size=(n, k))
    s = np.exp2(rng.integers(-8, 0, size=(n, k // 128))).astype(np.float16)
    w_folded = orc.dequantize(t, s)
    w = orc.rotate(w_folded, d, inverse=True)  # rows times R^T: W = W' R^T
    codes, scales = orc.prepare_weights(w, d)
    assert np.array_equal(codes, t) and np.array_equal(scales, s)
    x = rng.standard_normal((2, k))
    y = orc.linear(x, codes, scales, d)
    assert np.abs(y - x @ w.T).max() < 1e-10 * np.abs(x @ w.T).max()
    wrong, _ = orc.ternarize(orc.rotate(w, d, inverse=True))  # folded with R^T
    assert not np.array_equal(wrong, t)


# ----------------------------------------------------------------- linear

def test_linear_hand_computed(golden):
    codes = np.ones((2, 128), dtype=np.int8)
    codes[1, 1::2] = -1
    scales = np.array([[0.5], [2.0]], dtype=np.float16)
    xs = {"ramp": np.arange(1, 129, dtype=np.float64), "ones": np.ones(128)}
    for kind, y0, y1 in golden("linear_small.txt"):
        y = orc.linear(xs[kind][None, :], codes, scales)
        assert y[0, 0] == float(y0) and y[0, 1] == float(y1)


def test_dequantize_brute_force():
    rng = np.random.default_rng(7)
    codes = inputs.draw_codes(rng, 3, 256, 0.3)
    scales = inputs.draw_scales(rng, 3, 256)
    w = orc.dequantize(codes, scales)
    for n in range(3):
        for k in range(256):
            assert w[n, k] == float(scales[n, k // 128]) * int(codes[n, k])


def test_linear_add_sub_formulation():
    """y = sum_g s_g (sum of x' where t=+1 minus sum of x' where t=-1)."""
    p = inputs.make_linear_inputs(11, 2, 5, 1024, 0.33)
    y = orc.linear(p.x, p.codes, p.scales, p.signs)
    xr = np.stack([_fwht_loops(p.signs * p.x[m]) / 32.0 for m in range(2)])
    for m in range(2):
        for n in range(5):
            acc = 0.0
            for g in range(1024 // 128):
                plus = minus = 0.0
                for k in range(128 * g, 128 * (g + 1)):
                    if p.codes[n, k] == 1:
                        plus += xr[m, k]
                    elif p.codes[n, k] == -1:
                        minus += xr[m, k]
                acc += float(p.scales[n, g]) * (plus - minus)
            assert abs(acc - y[m, n]) < 1e-12 * max(1.0, abs(y[m, n]))


def test_linear_int_brute_force():
    rng = np.random.default_rng(8)
    codes = inputs.draw_codes(rng, 4, 256, 0.2)
    x = rng.integers(-127, 128, size=(3, 256)).astype(np.int8)
    y = orc.linear_int(x, codes)
    for m in range(3):
        for n in range(4):
            assert y[m, n] == sum(int(codes[n, k]) * int(x[m, k]) for k in range(256))


def test_missing_rotation_fails_tolerance():
    """Skipping the inverse rotation gives a silently wrong answer (news.ditty.ir,
    third paragraph): it must fail the float tolerance by a wide margin."""
    p = inputs.make_linear_inputs(0, 1, 256, 1024, 1.0 / 3.0)
    ref = orc.linear(p.x, p.codes, p.scales, p.signs)
    wrong = orc.linear(p.x, p.codes, p.scales, None)
    ok, rel, _ = within_linear_tolerance(wrong, ref, p.scales, p.x)
    assert not ok and rel > 0.5
    ok, _, _ = within_linear_tolerance(ref.astype(np.float32), ref, p.scales, p.x)
    assert ok


# ----------------------------------------------------------------- packings

def _pack_scalar(codes, fmt):
    """Byte-by-byte packer written as plain loops, for tiny matrices."""
    n, k = codes.shape
    rows = []
    for r in range(n):
        out = []
        c = [int(t) + 1 if int(t) in (-1, 0, 1) else 1 for t in codes[r]]
        if fmt == "2bit":
            for i in range(k // 4):
                out.append(sum(c[4 * i + j] << (2 * j) for j in range(4)))
        else:
            for g in range(k // 128):
                cg = c[128 * g:128 * g + 128] + [1, 1]
                for i in range(26):
                    out.append(sum(cg[5 * i + j] * 3 ** j for j in range(5)))
        rows.append(out)
    return np.array(rows, dtype=np.uint8)


def test_pack_2bit_golden(golden):
    for r in golden("pack_2bit.txt"):
        t = np.array([[int(v) for v in r[:4]] * 32], dtype=np.int8)  # one 128-group
        packed, bad = orc.pack(t, "2bit")
        assert bad == 0 and np.all(packed == int(r[4]))
        back, bad = orc.unpack(packed, "2bit", 1, 128)
        assert bad == 0 and np.array_equal(back, t)


def test_unpack_2bit_invalid_golden(golden):
    for r in golden("unpack_2bit_invalid.txt"):
        byte = int(r[0])
        packed = np.full((1, 32), 85, dtype=np.uint8)
        packed[0, 5] = byte
        codes, bad = orc.unpack(packed, "2bit", 1, 128)
        assert bad == int(r[5])
        assert list(codes[0, 20:24]) == [int(v) for v in r[1:5]]
        assert np.all(codes[0, :20] == 0) and np.all(codes[0, 24:] == 0)


def test_pack_base3_golden(golden):
    for r in golden("pack_base3.txt"):
        t = np.zeros((1, 128), dtype=np.int8)
        if r[0] == "B":
            t[0, 10:15] = [int(v) for v in r[1:6]]
            packed, bad = orc.pack(t, "base3")
            assert bad == 0 and packed[0, 2] == int(r[6])
        else:
            t[0, 125:128] = [int(v) for v in r[1:4]]
            packed, bad = orc.pack(t, "base3")
            assert bad == 0 and packed[0, 25] == int(r[4])
        back, bad = orc.unpack(packed, "base3", 1, 128)
        assert bad == 0 and np.array_equal(back, t)


def test_unpack_base3_invalid_golden(golden):
    for pos, byte, count in golden("unpack_base3_invalid.txt"):
        packed, _ = orc.pack(np.ones((1, 128), dtype=np.int8), "base3")
        idx = 3 if pos == "B" else 25
        packed[0, idx] = int(byte)
        codes, bad = orc.unpack(packed, "base3", 1, 128)
        assert bad == int(count)
        sl = slice(15, 20) if pos == "B" else slice(125, 128)
        if bad:
            assert np.all(codes[0, sl] == 0)
        mask = np.ones(128, dtype=bool)
        mask[sl] = False
        assert np.all(codes[0, mask] == 1)


def test_exhaustive_2bit_bytes():
    """Every one of the 256 byte values: valid ones (81) round-trip exactly."""
    valid = 0
    for b in range(256):
        packed = np.full((1, 32), b, dtype=np.uint8)
        codes, bad = orc.unpack(packed, "2bit", 1, 128)
        slots = [(b >> (2 * j)) & 3 for j in range(4)]
        assert bad == 32 * sum(s == 3 for s in slots)
        if bad == 0:
            valid += 1
            again, bad2 = orc.pack(codes, "2bit")
            assert bad2 == 0 and np.array_equal(again, packed)
    assert valid == 81


def test_exhaustive_base3_bytes():
    valid_body = valid_tail = 0
    base, _ = orc.pack(np.zeros((1, 128), dtype=np.int8), "base3")
    for b in range(256):
        for idx in (0, 25):
            packed = base.copy()
            packed[0, idx] = b
            codes, bad = orc.unpack(packed, "base3", 1, 128)
            if bad == 0:
                again, _ = orc.pack(codes, "base3")
                assert np.array_equal(again, packed)
                if idx == 0:
                    valid_body += 1
                else:
                    valid_tail += 1
    assert valid_body == 243 and valid_tail == 27


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_pack_matches_scalar_loops_and_roundtrips(fmt):
    rng = np.random.default_rng(9)
    codes = inputs.draw_codes(rng, 5, 512, 0.33)
    packed, bad = orc.pack(codes, fmt)
    assert bad == 0
    assert np.array_equal(packed, _pack_scalar(codes, fmt))
    back, bad = orc.unpack(packed, fmt, 5, 512)
    assert bad == 0 and np.array_equal(back, codes)


@pytest.mark.parametrize("fmt", ["2bit", "base3"])
def test_pack_counts_invalid_codes(fmt):
    codes = np.zeros((2, 128), dtype=np.int8)
    codes[0, 3] = 2
    codes[1, 100] = -5
    codes[1, 127] = 127
    packed, bad = orc.pack(codes, fmt)
    assert bad == 3
    back, bad2 = orc.unpack(packed, fmt, 2, 128)
    assert bad2 == 0 and np.all(back == 0)


def test_pack_1bit_worked_bytes(golden):
    for r in golden("pack_1bit.txt"):
        byte = int(r[0], 16)
        want = np.array([int(v) for v in r[1:]], dtype=np.int8)
        codes, bad = orc.unpack(np.array([[byte]] * 16, dtype=np.uint8).reshape(1, 16), "1bit", 1, 128)
        assert bad == 0 and np.array_equal(codes[0, :8], want), (hex(byte), codes[0, :8])
        packed, bad = orc.pack(np.tile(want, 16)[None, :], "1bit")
        assert bad == 0 and np.all(packed == byte)


def test_pack_1bit_round_trip_and_invalid_codes():
    rng = np.random.default_rng(50)
    t = rng.choice(np.array([-1, 1], dtype=np.int8), size=(7, 1024))
    packed, bad = orc.pack(t, "1bit")
    assert bad == 0 and packed.shape == (7, 128) and orc.packed_bytes("1bit", 7, 1024) == 7 * 128
    back, bad = orc.unpack(packed, "1bit", 7, 1024)
    assert bad == 0 and np.array_equal(back, t)
    # every one of the 256 byte values is a valid code byte and comes back
    allb = np.arange(256, dtype=np.uint8)[None, :].repeat(1, 0).reshape(1, 256)
    codes, bad = orc.unpack(np.tile(allb, (1, 4)), "1bit", 1, 8192)
    assert bad == 0 and set(np.unique(codes)) == {-1, 1}
    again, _ = orc.pack(codes, "1bit")
    assert np.array_equal(again, np.tile(allb, (1, 4)))
    # zeros and out-of-range codes are counted and packed as -1
    t2 = t.copy()
    t2[0, :3] = [0, 2, -5]
    p2, bad2 = orc.pack(t2, "1bit")
    assert bad2 == 3
    back2, _ = orc.unpack(p2, "1bit", 7, 1024)
    assert np.all(back2[0, :3] == -1)
    # the pages' ~1.125 bits per weight for 1-bit g128, as this layout's arithmetic
    assert orc.bits_per_weight("1bit") == 1.125


def test_bits_per_weight_arithmetic():
    n, k = 17408, 5120
    assert orc.packed_bytes("2bit", n, k) * 8 / (n * k) + 16 / 128 == 2.125
    assert orc.packed_bytes("base3", n, k) * 8 / (n * k) + 16 / 128 == 1.75
    assert orc.bits_per_weight("2bit") == 2.125 and orc.bits_per_weight("base3") == 1.75
    # The pages' figures as arithmetic: 1-bit g128 is 1 + 16/128 = 1.125 bits
    # (dev.to, two formats list); a trit carries log2(3) = 1.585 bits and with the
    # shared scale costs about 1.71 (news.ditty.ir, second paragraph).
    assert 1 + 16 / 128 == 1.125
    assert round(math.log2(3), 3) == 1.585
    assert round(math.log2(3) + 16 / 128, 2) == 1.71
    # The sizes of the two GGUF packings, 5.95 GB vs 7.21 GB, stand in about the
    # ratio of our two layouts (inference, not a statement of the pages).
    assert abs(5.95 / 7.21 - 1.75 / 2.125) < 0.005


# ----------------------------------------------------------------- inputs

def test_input_recipe_properties():
    p = inputs.make_linear_inputs(1, 1, 64, 5120, 0.33, outlier_rate=0.01)
    frac0 = float((p.codes == 0).mean())
    assert abs(frac0 - 0.33) < 0.01
    assert abs(float((p.codes == 1).mean()) - float((p.codes == -1).mean())) < 0.01
    xv = p.x
    assert np.array_equal(inputs.bf16_bits_from_float(xv), p.x_bf16)
    assert 20 <= int((np.abs(xv) == 20.0).sum()) <= 90
    assert set(np.unique(p.signs)) == {-1, 1}
    q = inputs.make_linear_inputs(1, 1, 64, 5120, 0.33, outlier_rate=0.01)
    assert np.array_equal(p.codes, q.codes) and np.array_equal(p.x_bf16, q.x_bf16)


def test_bf16_rounding_ties_to_even():
    f = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38], dtype=np.float32)
    b = inputs.bf16_bits_from_float(f)
    back = inputs.float_from_bf16_bits(b)
    assert back[0] == 1.0 and back[1] == 1.0 + 2 ** -6 and back[2] == -2.5
