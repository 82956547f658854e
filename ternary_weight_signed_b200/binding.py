"""ctypes binding of libternary_b200.so: the same names as the C entry points.

Argument marshalling only: tensors are passed by ``data_ptr()``, streams by
their ``cuda_stream`` handle, and every computation happens in the library's
kernels.  A missing library raises; nothing falls back to another
implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

from . import build as _build

TB_OK, TB_ERR_NULL, TB_ERR_SHAPE, TB_ERR_DTYPE, TB_ERR_FORMAT = 0, 1, 2, 3, 4
TB_ERR_ALIGN, TB_ERR_CUDA, TB_ERR_WORKSPACE, TB_ERR_DEVICE = 5, 6, 7, 8
TB_FMT_2BIT, TB_FMT_BASE3, TB_FMT_1BIT = 0, 1, 2
TB_BF16, TB_FP16, TB_FP32, TB_INT8, TB_INT32 = 0, 1, 2, 3, 4
TB_PATH_AUTO, TB_PATH_GEMV, TB_PATH_GEMM, TB_PATH_SIMPLE, TB_PATH_GEMV_TC = 0, 1, 2, 3, 4

FORMATS = {"2bit": TB_FMT_2BIT, "base3": TB_FMT_BASE3, "1bit": TB_FMT_1BIT}

HEADER = os.path.join(_build.ROOT, "include", "ternary_b200.h")

_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGNATURES = {
    "tb_status_string": (ctypes.c_char_p, [_int]),
    "tb_version": (_int, []),
    "tb_packed_bytes": (_sz, [_int, _i64, _i64]),
    "tb_pack_ternary": (_int, [_int, _vp, _i64, _i64, _vp, _vp, _vp]),
    "tb_unpack_ternary": (_int, [_int, _vp, _i64, _i64, _vp, _vp, _vp]),
    "tb_hadamard_rotate": (_int, [_vp, _int, _vp, _int, _vp, _i64, _i64, _int, _vp]),
    "tb_prepare_weights": (_int, [_vp, _int, _vp, _i64, _i64, _int, _vp, _vp, _vp]),
    "tb_ternary_linear_workspace": (_sz, [_int, _i64, _i64, _i64]),
    "tb_ternary_linear": (_int, [_vp, _int, _vp, _vp, _int, _i64, _i64, _i64, _vp, _vp, _int,
                                 _vp, _sz, _vp]),
    "tb_ternary_linear_ex": (_int, [_vp, _int, _vp, _vp, _int, _i64, _i64, _i64, _vp, _vp, _int,
                                    _vp, _sz, _int, _vp]),
    "tb_ternary_linear_path": (_int, [_int, _int, _i64, _i64, _i64, _int, _int]),
    "tb_get_device_fault": (_int, [ctypes.POINTER(ctypes.c_uint32), _int]),
    "tb_test_stall_copies": (_int, [ctypes.c_uint32, ctypes.c_uint64]),
    "tb_ternary_linear_noalloc": (_int, [_vp, _int, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _int,
                                         _vp]),
}

_LIB = None


class TBError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_string(status)})")


def header_functions() -> list[str]:
    """Names of the functions the public header declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:[\w\*]+\s+)+\**(tb_\w+)\s*\(", text, re.M)))


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    p = path or _build.LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with __graft_entry__.build() "
                           "(there is no other implementation to fall back to)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _fmt(f):
    return FORMATS[f] if isinstance(f, str) else int(f)


def dtype_code(t) -> int:
    import torch
    m = {torch.bfloat16: TB_BF16, torch.float16: TB_FP16, torch.float32: TB_FP32,
         torch.int8: TB_INT8, torch.int32: TB_INT32}
    return m[t]


def _done(st: int, where: str, check: bool) -> int:
    if check and st != TB_OK:
        raise TBError(st, where)
    return st


def status_string(st: int) -> str:
    return load().tb_status_string(st).decode()


def tb_version() -> int:
    return load().tb_version()


def tb_packed_bytes(fmt, n: int, k: int) -> int:
    return load().tb_packed_bytes(_fmt(fmt), n, k)


def tb_pack_ternary(fmt, codes, n, k, packed, invalid=None, stream=None, check=True):
    st = load().tb_pack_ternary(_fmt(fmt), _ptr(codes), n, k, _ptr(packed), _ptr(invalid),
                                _stream(stream))
    return _done(st, "tb_pack_ternary", check)


def tb_unpack_ternary(fmt, packed, n, k, codes, invalid=None, stream=None, check=True):
    st = load().tb_unpack_ternary(_fmt(fmt), _ptr(packed), n, k, _ptr(codes), _ptr(invalid),
                                  _stream(stream))
    return _done(st, "tb_unpack_ternary", check)


def tb_hadamard_rotate(x, xt, y, yt, signs, m, k, inverse=0, stream=None, check=True):
    st = load().tb_hadamard_rotate(_ptr(x), xt, _ptr(y), yt, _ptr(signs), m, k, int(inverse),
                                   _stream(stream))
    return _done(st, "tb_hadamard_rotate", check)


def tb_prepare_weights(w, wt, signs, n, k, fmt, packed, scales, stream=None, check=True):
    st = load().tb_prepare_weights(_ptr(w), wt, _ptr(signs), n, k, _fmt(fmt), _ptr(packed),
                                   _ptr(scales), _stream(stream))
    return _done(st, "tb_prepare_weights", check)


def tb_ternary_linear_workspace(fmt, m, n, k) -> int:
    return load().tb_ternary_linear_workspace(_fmt(fmt), m, n, k)


def tb_ternary_linear(x, xt, packed, scales, fmt, m, n, k, signs, y, yt, workspace, ws_bytes,
                      stream=None, check=True):
    st = load().tb_ternary_linear(_ptr(x), xt, _ptr(packed), _ptr(scales), _fmt(fmt), m, n, k,
                                  _ptr(signs), _ptr(y), yt, _ptr(workspace), ws_bytes,
                                  _stream(stream))
    return _done(st, "tb_ternary_linear", check)


def tb_ternary_linear_ex(x, xt, packed, scales, fmt, m, n, k, signs, y, yt, workspace, ws_bytes,
                         path, stream=None, check=True):
    st = load().tb_ternary_linear_ex(_ptr(x), xt, _ptr(packed), _ptr(scales), _fmt(fmt), m, n, k,
                                     _ptr(signs), _ptr(y), yt, _ptr(workspace), ws_bytes, path,
                                     _stream(stream))
    return _done(st, "tb_ternary_linear_ex", check)


def tb_ternary_linear_path(xt, fmt, m, n, k, has_signs=True, aligned16=True) -> int:
    return load().tb_ternary_linear_path(xt, _fmt(fmt), m, n, k, int(has_signs), int(aligned16))


TB_NOALLOC_SCRATCH_BYTES = 589824


def tb_ternary_linear_noalloc(x, xt, packed, scales, m, n, k, signs, y, yt, stream=None,
                              check=True):
    """The decode path with the library's fixed scratch instead of a workspace
    (for callers that cannot allocate device memory; see the C header)."""
    st = load().tb_ternary_linear_noalloc(_ptr(x), xt, _ptr(packed), _ptr(scales), m, n, k,
                                          _ptr(signs), _ptr(y), yt, _stream(stream))
    return _done(st, "tb_ternary_linear_noalloc", check)


def tb_get_device_fault(clear=False) -> int:
    v = ctypes.c_uint32(0)
    _done(load().tb_get_device_fault(ctypes.byref(v), int(clear)), "tb_get_device_fault", True)
    return v.value


def tb_test_stall_copies(stall, wait_limit_ns=0):
    """Failure-detection test hook (see the C header): with stall the weight
    copies of the one-token decode and of the fp16 GEMM are not issued and the
    waits for them run out after wait_limit_ns (0 = the default 2 s)."""
    _done(load().tb_test_stall_copies(int(bool(stall)), int(wait_limit_ns)), "tb_test_stall_copies", True)
