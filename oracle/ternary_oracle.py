"""CPU oracle for the ternary-g128 linear layer with a signed block-Hadamard rotation.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module.  It shares no code with the
CUDA path and imports nothing from it.  Everything is plain NumPy in float64 (or
exact integers), written for a reader to check against the definitions by eye,
not for speed.

What the layer computes (sources are the pages' sections):

* "Ternary g128" (news.ditty.ir, Bonsai 2 27B, second paragraph; ai4coding.ru,
  "What is a ternary model"): every weight is -1, 0 or +1 and every run of 128
  consecutive weights along the input dimension shares one FP16 scale, so the
  dequantised weight is w[n, k] = s[n, k // 128] * t[n, k].
* Block Hadamard rotation (news.ditty.ir, second and third paragraphs;
  openbonsai.org, "How it works", step 1 "Rotate"): an orthogonal, signed
  Hadamard rotation on blocks of 1024 inputs is folded into every weight matrix
  (W' = W R), and its inverse is applied to the activations at run time
  (x' = R^T x), so that W' x' = W R R^T x = W x.
* Add/sub MAC (ai4coding.ru, "What is a ternary model", last paragraph):
  multiplying by a ternary weight is an addition, a subtraction or nothing.
* The two packings (news.ditty.ir, paragraph on the CUDA GGUF files) are named
  there only as "dense trit" and "2-bit slot" packings; the byte layouts below
  are this library's own definitions of those two ideas.

Readings taken where the pages are silent:

* R_b = diag(d_b) H / 32 with H the Sylvester Hadamard matrix of order 1024 in
  natural order and d_b the +-1 signs of block b; the run-time transform is
  x'_b = R_b^T x_b = (H / 32)(d_b * x_b).  ``inverse`` applies x_b = R_b x'_b.
* 2-bit slots: code c = t + 1 in {0, 1, 2}; byte i of a row holds k = 4i..4i+3,
  weight 4i+j in bits 2j..2j+1.  c = 3 is invalid (decodes to t = 0, counted).
* base-3: every 128-group is its own 26-byte run.  Bytes 0..24 hold
  k = 5i..5i+4 as sum_j c_{5i+j} 3^j (lowest k = least significant digit);
  byte 25 holds k = 125..127 in digits 0..2 and c = 1 (t = 0) in digits 3 and 4.
  A byte >= 243, or a last byte whose digits 3 and 4 are not both 1, is invalid:
  all codes it carries decode to t = 0 and it is counted once.
* Codes outside {-1, 0, 1} given to the packer are packed as t = 0 and counted.
* 1-bit g128 (dev.to, "How Prism ML Squeezed a 27B Model Into 3.9 GB", the
  list of the two formats that ship: each weight -1 or +1 with one scale per
  128 weights, about 1.125 bits): byte i of a row holds k = 8i..8i+7, weight
  8i+j in bit j, bit 1 = +1 and bit 0 = -1.  Any other code given to the
  packer (0 included) is packed as -1 and counted; every byte is valid.
* Integer mode: y[m, n] = sum_k t[n, k] x[m, k] for int8 x, no scales, no rotation.
* Producer side (openbonsai.org, "How it works", steps 1 "Rotate" and 2
  "Round"): the pages round with sequential GPTQ on calibration data, which
  needs a model and data; the stand-in here is plain rounding to the nearest
  level with one scale per group.  The scale is the group's mean |w'| (after
  the fold), rounded to fp16; t = clip(rint(w' / s), -1, 1) with that fp16 s
  (rint: halves to even); a group of zeros gets s = 0 and t = 0.

Parity: every function here is pinned by the CPU tests (closed forms,
exhaustive byte tables, brute force, library routines); none is "parity
unpinned".
"""
from __future__ import annotations

import numpy as np

GROUP = 128
BLOCK = 1024
FMT_2BIT = "2bit"
FMT_BASE3 = "base3"
FMT_1BIT = "1bit"
BASE3_GROUP_BYTES = 26


# --------------------------------------------------------------------------
# Rotation
# --------------------------------------------------------------------------

def sylvester_hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (a power of two), natural order.

    H_1 = [1];  H_2m = [[H_m, H_m], [H_m, -H_m]].  Integer entries (int64).
    """
    if n < 1 or n & (n - 1):
        raise ValueError("order must be a power of two")
    h = np.ones((1, 1), dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def rotation_matrix(signs_block: np.ndarray) -> np.ndarray:
    """R_b = diag(d_b) H / 32 for one 1024-block of signs (float64)."""
    d = np.asarray(signs_block, dtype=np.float64)
    if d.shape != (BLOCK,):
        raise ValueError("one block of 1024 signs expected")
    h = sylvester_hadamard(BLOCK).astype(np.float64)
    return np.diag(d) @ h / np.sqrt(BLOCK)


def rotate(x: np.ndarray, signs: np.ndarray, inverse: bool = False) -> np.ndarray:
    """Apply the block rotation to the rows of x [M, K] (K a multiple of 1024).

    inverse=False: x'_b = R_b^T x_b (what the run time applies to activations).
    inverse=True:  x_b  = R_b x'_b.
    Explicit fp64 matrix products, one 1024 x 1024 matrix per block.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    m, k = x.shape
    if k % BLOCK:
        raise ValueError("K must be a multiple of 1024")
    signs = np.asarray(signs)
    if signs.shape != (k,):
        raise ValueError("one sign per input coordinate expected")
    out = np.empty_like(x)
    for b in range(k // BLOCK):
        sl = slice(b * BLOCK, (b + 1) * BLOCK)
        r = rotation_matrix(signs[sl])
        mat = r if inverse else r.T
        out[:, sl] = x[:, sl] @ mat.T
    return out


def fold_weights(w: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """W' = W R for a dense W [N, K]: block b of every row times R_b
    (explicit fp64 products; the run time then applies R^T to x)."""
    w = np.atleast_2d(np.asarray(w, dtype=np.float64))
    n, k = w.shape
    if k % BLOCK:
        raise ValueError("K must be a multiple of 1024")
    signs = np.asarray(signs)
    if signs.shape != (k,):
        raise ValueError("one sign per input coordinate expected")
    out = np.empty_like(w)
    for b in range(k // BLOCK):
        sl = slice(b * BLOCK, (b + 1) * BLOCK)
        out[:, sl] = w[:, sl] @ rotation_matrix(signs[sl])
    return out


# --------------------------------------------------------------------------
# Ternary g128 weights
# --------------------------------------------------------------------------

def ternarize(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round a dense [N, K] matrix to ternary g128: per 128-group the scale
    s = fp16(mean |w|) and the codes t = clip(rint(w / s), -1, 1) (s = 0:
    t = 0).  Returns (codes int8 [N, K], scales fp16 [N, K/128])."""
    w = np.atleast_2d(np.asarray(w, dtype=np.float64))
    n, k = w.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    codes = np.zeros((n, k), dtype=np.int8)
    scales = np.zeros((n, k // GROUP), dtype=np.float16)
    for r in range(n):
        for g in range(k // GROUP):
            grp = w[r, g * GROUP:(g + 1) * GROUP]
            s = np.float16(np.mean(np.abs(grp)))
            scales[r, g] = s
            if s == 0:
                continue
            q = np.rint(grp / np.float64(s))
            codes[r, g * GROUP:(g + 1) * GROUP] = np.clip(q, -1, 1).astype(np.int8)
    return codes, scales


def prepare_weights(w: np.ndarray, signs: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """The producer side of the layer: fold the rotation into a dense W, then
    round to ternary g128 (codes, scales) for ``linear`` with these signs."""
    return ternarize(fold_weights(w, signs))


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """w[n, k] = float64(s[n, k // 128]) * t[n, k]."""
    t = np.asarray(codes, dtype=np.int64)
    n, k = t.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    s = np.asarray(scales).astype(np.float64)
    if s.shape != (n, k // GROUP):
        raise ValueError("scales must be [N, K/128]")
    return np.repeat(s, GROUP, axis=1) * t


def linear(x: np.ndarray, codes: np.ndarray, scales: np.ndarray,
           signs: np.ndarray | None = None) -> np.ndarray:
    """y = x' W^T in float64, x [M, K], codes [N, K], scales [N, K/128].

    With ``signs`` the activations are first rotated, x' = R^T x (the weights
    are taken to be stored with R already folded in); without, x is taken as
    already rotated.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    xr = rotate(x, signs) if signs is not None else x
    w = dequantize(codes, scales)
    return xr @ w.T


def linear_int(x_int8: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """Integer mode: y[m, n] = sum_k t[n, k] x[m, k], exact int64."""
    x = np.atleast_2d(np.asarray(x_int8, dtype=np.int64))
    t = np.asarray(codes, dtype=np.int64)
    return x @ t.T


# --------------------------------------------------------------------------
# Packings
# --------------------------------------------------------------------------

def packed_bytes(fmt: str, n: int, k: int) -> int:
    """Bytes of packed codes (scales are separate: N * K/128 * 2 bytes)."""
    if k % GROUP:
        raise ValueError("K must be a multiple of 128")
    if fmt == FMT_2BIT:
        return n * (k // 4)
    if fmt == FMT_BASE3:
        return n * (k // GROUP) * BASE3_GROUP_BYTES
    if fmt == FMT_1BIT:
        return n * (k // 8)
    raise ValueError(f"unknown format {fmt!r}")


def _valid_code_mask(codes: np.ndarray) -> np.ndarray:
    return (codes == -1) | (codes == 0) | (codes == 1)


def pack(codes: np.ndarray, fmt: str) -> tuple[np.ndarray, int]:
    """Pack int8 codes [N, K] -> (uint8 [N, row_bytes], invalid code count)."""
    t = np.asarray(codes).astype(np.int64)
    n, k = t.shape
    if fmt == FMT_1BIT:
        ok1 = (t == -1) | (t == 1)
        bit = (t == 1).astype(np.int64).reshape(n, k // 8, 8)
        byte = sum(bit[..., j] << j for j in range(8))
        return byte.astype(np.uint8), int((~ok1).sum())
    ok = _valid_code_mask(t)
    invalid = int((~ok).sum())
    c = np.where(ok, t + 1, 1)  # biased code, invalid -> t = 0
    if fmt == FMT_2BIT:
        c4 = c.reshape(n, k // 4, 4)
        byte = c4[..., 0] + 4 * c4[..., 1] + 16 * c4[..., 2] + 64 * c4[..., 3]
        return byte.astype(np.uint8), invalid
    if fmt == FMT_BASE3:
        g = k // GROUP
        cg = c.reshape(n, g, GROUP)
        full = cg[:, :, :125].reshape(n, g, 25, 5)
        body = (full[..., 0] + 3 * full[..., 1] + 9 * full[..., 2]
                + 27 * full[..., 3] + 81 * full[..., 4])
        tail = cg[:, :, 125] + 3 * cg[:, :, 126] + 9 * cg[:, :, 127] + 27 * 1 + 81 * 1
        out = np.concatenate([body, tail[:, :, None]], axis=2)
        return out.reshape(n, g * BASE3_GROUP_BYTES).astype(np.uint8), invalid
    raise ValueError(f"unknown format {fmt!r}")


def unpack(packed: np.ndarray, fmt: str, n: int, k: int) -> tuple[np.ndarray, int]:
    """Unpack uint8 [N, row_bytes] -> (int8 codes [N, K], invalid count)."""
    p = np.asarray(packed).astype(np.int64).reshape(n, -1)
    if fmt == FMT_1BIT:
        if p.shape[1] != k // 8:
            raise ValueError("row bytes must be K/8")
        bits = np.stack([(p >> j) & 1 for j in range(8)], axis=-1).reshape(n, k)
        return (2 * bits - 1).astype(np.int8), 0
    if fmt == FMT_2BIT:
        if p.shape[1] != k // 4:
            raise ValueError("row bytes must be K/4")
        c = np.stack([(p >> (2 * j)) & 3 for j in range(4)], axis=-1).reshape(n, k)
        bad = c == 3
        t = np.where(bad, 0, c - 1)
        return t.astype(np.int8), int(bad.sum())
    if fmt == FMT_BASE3:
        g = k // GROUP
        if p.shape[1] != g * BASE3_GROUP_BYTES:
            raise ValueError("row bytes must be 26 * K/128")
        pg = p.reshape(n, g, BASE3_GROUP_BYTES)
        digits = np.stack([(pg // 3 ** j) % 3 for j in range(5)], axis=-1)  # [n,g,26,5]
        bad = pg >= 243
        bad[:, :, 25] |= (digits[:, :, 25, 3] != 1) | (digits[:, :, 25, 4] != 1)
        t = np.where(bad[..., None], 0, digits - 1)
        body = t[:, :, :25, :].reshape(n, g, 125)
        tail = t[:, :, 25, :3]
        codes = np.concatenate([body, tail], axis=2).reshape(n, k)
        return codes.astype(np.int8), int(bad.sum())
    raise ValueError(f"unknown format {fmt!r}")


def bits_per_weight(fmt: str, k: int = BLOCK) -> float:
    """Packed code bits plus one 16-bit scale per 128 weights, per weight."""
    return 8.0 * packed_bytes(fmt, 1, k) / k + 16.0 / GROUP
