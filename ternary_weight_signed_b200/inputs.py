"""Seeded synthetic inputs for the ternary-g128 linear layer.

This module only draws random numbers and rounds them to the storage types the
layer consumes (int8 codes, fp16 scales, bf16 activations, int8 signs).  It holds
none of the layer's arithmetic (no packing, no rotation, no products), so both
the CPU oracle tests and the CUDA path can take their inputs from here without
sharing any of the method.

Recipe (the pages print no workload, so these follow the layer's definition on
the Bonsai 2 27B page of news.ditty.ir, "ternary g128" paragraph, and the shapes
of a 27B-class model):

* ``numpy.random.default_rng(seed)``; draw order codes -> scales -> activations
  -> signs, each drawn once for the whole array.
* codes t in {-1, 0, +1}: one uniform u in [0, 1) per weight, row-major;
  t = -1 if u < (1-p0)/2, 0 if u < (1-p0)/2 + p0, else +1.
* scales: fp16 round-to-nearest-even of |N(0,1)| * 0.02 ("abs_normal") or of
  exp(N(mu, sigma)) ("lognormal"), one per 128 consecutive weights of a row.
* activations: bf16 round-to-nearest-even of N(0,1); with an outlier rate p,
  each element independently becomes 20 * sign(another normal draw) (exact in
  bf16).  The rounded values are the ground truth for both sides.
* signs: one +-1 per input coordinate (length K), uniform.
"""
from __future__ import annotations

import dataclasses

import numpy as np

GROUP = 128  # weights per fp16 scale along K
BLOCK = 1024  # Hadamard block length along K

_CHUNK = 1 << 22  # uniforms drawn per slice when generating codes


def bf16_bits_from_float(a: np.ndarray) -> np.ndarray:
    """Round float32/float64 values to bf16 (round to nearest, ties to even).

    Returns the bf16 bit patterns as uint16.  NaN is not produced by the
    generators, so it is not handled.
    """
    f = np.asarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    return u.astype(np.uint16)


def float_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Exact float32 values of bf16 bit patterns."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def draw_codes(rng: np.random.Generator, n: int, k: int, p0: float) -> np.ndarray:
    """Ternary codes [n, k] int8 with P(0) = p0 and P(+1) = P(-1)."""
    total = n * k
    out = np.empty(total, dtype=np.int8)
    lo = (1.0 - p0) / 2.0
    mid = lo + p0
    pos = 0
    while pos < total:
        m = min(_CHUNK, total - pos)
        u = rng.random(m)
        seg = np.ones(m, dtype=np.int8)
        seg[u < mid] = 0
        seg[u < lo] = -1
        out[pos:pos + m] = seg
        pos += m
    return out.reshape(n, k)


def draw_scales(rng: np.random.Generator, n: int, k: int, kind: str = "abs_normal",
                mu: float = -4.0, sigma: float = 0.5) -> np.ndarray:
    """fp16 group scales [n, k/128]."""
    g = k // GROUP
    if kind == "abs_normal":
        v = np.abs(rng.standard_normal((n, g))) * 0.02
    elif kind == "lognormal":
        v = np.exp(rng.normal(mu, sigma, (n, g)))
    else:
        raise ValueError(f"unknown scale distribution {kind!r}")
    return v.astype(np.float16)


def draw_activations(rng: np.random.Generator, m: int, k: int,
                     outlier_rate: float = 0.0) -> np.ndarray:
    """bf16 activations [m, k] as uint16 bit patterns."""
    v = rng.standard_normal((m, k))
    if outlier_rate > 0.0:
        hit = rng.random((m, k)) < outlier_rate
        sgn = np.where(rng.standard_normal((m, k)) < 0.0, -20.0, 20.0)
        v = np.where(hit, sgn, v)
    return bf16_bits_from_float(v)


def draw_signs(rng: np.random.Generator, k: int) -> np.ndarray:
    """+-1 rotation signs [k] int8."""
    return np.where(rng.random(k) < 0.5, -1, 1).astype(np.int8)


@dataclasses.dataclass
class LinearInputs:
    """One seeded problem: codes [N,K] int8, scales [N,K/128] fp16,
    activations [M,K] bf16 bits (uint16), signs [K] int8."""

    codes: np.ndarray
    scales: np.ndarray
    x_bf16: np.ndarray
    signs: np.ndarray

    @property
    def x(self) -> np.ndarray:
        """Activations as exact float64 values."""
        return float_from_bf16_bits(self.x_bf16).astype(np.float64)


def make_linear_inputs(seed: int, m: int, n: int, k: int, p0: float,
                       scale_kind: str = "abs_normal", outlier_rate: float = 0.0,
                       mu: float = -4.0, sigma: float = 0.5) -> LinearInputs:
    """Draw one problem in the documented order (codes, scales, activations, signs)."""
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    rng = np.random.default_rng(seed)
    codes = draw_codes(rng, n, k, p0)
    scales = draw_scales(rng, n, k, scale_kind, mu, sigma)
    x = draw_activations(rng, m, k, outlier_rate)
    signs = draw_signs(rng, k)
    return LinearInputs(codes, scales, x, signs)


# The five workloads, named by what they are.  ``fmts`` lists the packings the
# workload is run in; "2bit" = 2-bit slots, "base3" = 5 trits per byte.
WORKLOADS = {
    "tiny_k1024_n256": dict(seed=0, ms=(1,), n=256, k=1024, p0=1.0 / 3.0,
                            scale_kind="abs_normal", outlier_rate=0.0, fmts=("2bit",)),
    "gemv_gateup_k5120_n17408": dict(seed=1, ms=(1,), n=17408, k=5120, p0=0.33,
                                     scale_kind="abs_normal", outlier_rate=0.01,
                                     fmts=("2bit", "base3")),
    "gemv_down_k17408_n5120": dict(seed=2, ms=(1, 2, 4, 8, 16), n=5120, k=17408, p0=0.5,
                                   scale_kind="lognormal", outlier_rate=0.0,
                                   fmts=("2bit", "base3")),
    "prefill_m2048_k5120_n17408": dict(seed=3, ms=(2048,), n=17408, k=5120, p0=0.33,
                                       scale_kind="abs_normal", outlier_rate=0.0,
                                       fmts=("2bit",)),
}

# Linear shapes (N outputs, K inputs) of one layer of the synthetic 27B-class stack.
STACK_LAYER_SHAPES = (
    ("q", 6144, 5120), ("k", 1024, 5120), ("v", 1024, 5120), ("o", 5120, 6144),
    ("gate", 17408, 5120), ("up", 17408, 5120), ("down", 5120, 17408),
)
STACK_LAYERS = 64


def workload_inputs(name: str, m: int | None = None) -> LinearInputs:
    """Inputs of a named workload at token count ``m`` (default: its first)."""
    w = WORKLOADS[name]
    mm = w["ms"][0] if m is None else m
    return make_linear_inputs(w["seed"], mm, w["n"], w["k"], w["p0"], w["scale_kind"],
                              w["outlier_rate"])


# ---------------------------------------------------------------------------
# The synthetic layer stack: 64 layers x 7 matrices, 21.8 G ternary codes, too
# many to draw on the host, so its codes come from a counter-based generator
# that the device (torch) and the host (numpy) evaluate identically: code
# (n, k) of matrix `mat` of layer `layer` is a function of its index alone.
#
# Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
# number generators", OOPSLA 2014): with a 64-bit state s and the counter i,
#   z = s + (i + 1) * 0x9E3779B97F4A7C15
#   z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
#   z = (z ^ (z >> 27)) * 0x94D049BB133111EB
#   out = z ^ (z >> 31)                         (all mod 2^64, logical shifts)
# u = (out >> 11) * 2^-53 is uniform in [0, 1) and becomes a code with the
# same thresholds as draw_codes.  The state of a matrix is the SplitMix64
# output for counter 0 of the state seed * 2^20 + layer * 16 + mat.  Scales,
# activations and signs of the stack are small and come from numpy's default
# generator seeded with (seed, layer, mat) (stack_scales, stack_activations).

_SM_GOLDEN = 0x9E3779B97F4A7C15
_SM_M1 = 0xBF58476D1CE4E5B9
_SM_M2 = 0x94D049BB133111EB
_U64 = (1 << 64) - 1


def _splitmix64_py(state: int, i: int) -> int:
    z = (state + (i + 1) * _SM_GOLDEN) & _U64
    z = ((z ^ (z >> 30)) * _SM_M1) & _U64
    z = ((z ^ (z >> 27)) * _SM_M2) & _U64
    return z ^ (z >> 31)


def stack_state(seed: int, layer: int, mat: int) -> int:
    """64-bit generator state of one matrix of the stack."""
    return _splitmix64_py((seed << 20) + layer * 16 + mat, 0)


def _codes_from_uniform_bits(top53, p0: float, xp):
    lo = (1.0 - p0) / 2.0
    mid = lo + p0
    u = top53.astype(xp.float64) * (1.0 / 9007199254740992.0)
    out = xp.ones(u.shape, dtype=xp.int8)
    out[u < mid] = 0
    out[u < lo] = -1
    return out


def stack_codes_rows_np(seed: int, layer: int, mat: int, rows, k: int, p0: float) -> np.ndarray:
    """Codes of the given rows (any order) of one stack matrix, [len(rows), k] int8 (host)."""
    rows = np.asarray(rows, dtype=np.uint64)
    s = np.uint64(stack_state(seed, layer, mat))
    i = rows[:, None] * np.uint64(k) + np.arange(k, dtype=np.uint64)[None, :]
    with np.errstate(over="ignore"):
        z = s + (i + np.uint64(1)) * np.uint64(_SM_GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_SM_M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_SM_M2)
        z = z ^ (z >> np.uint64(31))
    return _codes_from_uniform_bits(z >> np.uint64(11), p0, np)


def _i64(c: int) -> int:
    """A 64-bit constant as the signed value with the same bits."""
    return c - (1 << 64) if c >= (1 << 63) else c


def stack_codes_torch(seed: int, layer: int, mat: int, n: int, k: int, p0: float, device,
                      rows_per_chunk: int = 1024):
    """All codes of one stack matrix, [n, k] int8, computed on `device` with torch
    int64 arithmetic (wrap-around products, logical shifts by masking)."""
    import torch

    s = _i64(stack_state(seed, layer, mat))
    out = torch.empty((n, k), dtype=torch.int8, device=device)
    col = torch.arange(k, dtype=torch.int64, device=device)

    def lsr(z, sh):
        return (z >> sh) & ((1 << (64 - sh)) - 1)

    lo = (1.0 - p0) / 2.0
    mid = lo + p0
    for r0 in range(0, n, rows_per_chunk):
        r1 = min(n, r0 + rows_per_chunk)
        i = torch.arange(r0, r1, dtype=torch.int64, device=device)[:, None] * k + col[None, :]
        z = s + (i + 1) * _i64(_SM_GOLDEN)
        z = (z ^ lsr(z, 30)) * _i64(_SM_M1)
        z = (z ^ lsr(z, 27)) * _i64(_SM_M2)
        z = z ^ lsr(z, 31)
        u = lsr(z, 11).to(torch.float64) * (1.0 / 9007199254740992.0)
        seg = torch.ones_like(u, dtype=torch.int8)
        seg[u < mid] = 0
        seg[u < lo] = -1
        out[r0:r1] = seg
    return out


def stack_scales(seed: int, layer: int, mat: int, n: int, k: int) -> np.ndarray:
    """fp16 g128 scales of one stack matrix, |N(0,1)| * 0.02."""
    rng = np.random.default_rng([seed, layer, mat, 1])
    return draw_scales(rng, n, k, "abs_normal")


def stack_activations(seed: int, m: int, k: int) -> tuple[np.ndarray, np.ndarray]:
    """bf16 activations [m, k] (bits) and +-1 signs [k] for the stack's inputs
    of width k (one per input width; the linears' inputs are independent)."""
    rng = np.random.default_rng([seed, k, m, 2])
    return draw_activations(rng, m, k), draw_signs(rng, k)
