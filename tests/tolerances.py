"""Float tolerances for the linear layer and the rotation, stated once.

Linear (fp32 or bf16 output against the float64 oracle):
  * relative L2 over the whole [M, N] output <= 2e-3;
  * every element |y - y*| <= 1e-2 * max|s| * ||x_m||_2, with max|s| over the
    whole scale matrix and ||x_m||_2 the norm of activation row m (equal for x
    and x', the rotation being orthogonal).
Rotation (fp32 output): per row ||x' - x'*||_2 / ||x'*||_2 <= 1e-5.
"""
import numpy as np

LINEAR_REL_L2 = 2e-3
LINEAR_ELEM = 1e-2
ROTATE_REL_L2 = 1e-5


def within_linear_tolerance(y, ref, scales, x):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(y - ref)) / max(denom, 1e-300)
    smax = float(np.abs(np.asarray(scales, dtype=np.float64)).max())
    xn = np.linalg.norm(np.atleast_2d(np.asarray(x, dtype=np.float64)), axis=1)
    bound = LINEAR_ELEM * smax * xn[:, None]
    elem_ok = bool(np.all(np.abs(y - ref) <= bound))
    return (rel <= LINEAR_REL_L2 and elem_ok), rel, float((np.abs(y - ref) / bound).max())


def rotate_rel_err(y, ref):
    y = np.atleast_2d(np.asarray(y, dtype=np.float64))
    ref = np.atleast_2d(np.asarray(ref, dtype=np.float64))
    num = np.linalg.norm(y - ref, axis=1)
    den = np.maximum(np.linalg.norm(ref, axis=1), 1e-300)
    return float((num / den).max())
