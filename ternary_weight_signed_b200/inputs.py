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
