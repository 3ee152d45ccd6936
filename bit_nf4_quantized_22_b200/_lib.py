"""ctypes loader for libqlora.so (the C ABI declared in include/qlora.h)."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqlora.so")

QLORA_OK = 0
QLORA_EINVAL = 1
QLORA_EUNSUPPORTED = 2
QLORA_ECUDA = 3
QLORA_EWORKSPACE = 4
STATUS_NONFINITE = 1
STATUS_TIMEOUT = 2

# every symbol include/qlora.h declares
EXPORTS = (
    "qlora_strerror", "qlora_version", "qlora_check_codebook", "nf4_quantize",
    "nf4_dequantize", "qlora_workspace_size", "qlora_forward", "qlora_backward",
    "qlora_launch_count", "qlora_profile_enable", "qlora_profile_reset", "qlora_profile_read",
    "qlora_profile_kinds", "qlora_profile_read_each",
    "qlora_forward_noalloc", "qlora_merge", "qlora_selftest_wait_timeout", "nf4_dequantize_dtype",
    "nf4_codebook", "fp4_codebook",
)


class NF4WeightC(ctypes.Structure):
    """Mirror of nf4_weight_t."""
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("block", ctypes.c_int32),
        ("double_quant", ctypes.c_int32),
        ("dq_group", ctypes.c_int32),
        ("compute_dtype", ctypes.c_int32),
        ("packed", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("absmax_code", ctypes.c_void_p),
        ("dq_step", ctypes.c_void_p),
        ("dq_mean", ctypes.c_void_p),
    ]


class QLoRAError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} (code {code})")


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"libqlora.so not found at {p}; build it with "
            "`python -m bit_nf4_quantized_22_b200.build`")
    lib = ctypes.CDLL(p)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    W = ctypes.POINTER(NF4WeightC)
    lib.qlora_strerror.restype = ctypes.c_char_p
    lib.qlora_strerror.argtypes = [ctypes.c_int]
    lib.qlora_version.restype = ctypes.c_int
    lib.qlora_version.argtypes = []
    lib.qlora_check_codebook.restype = ctypes.c_int
    lib.qlora_check_codebook.argtypes = [P]
    lib.nf4_quantize.restype = ctypes.c_int
    lib.nf4_quantize.argtypes = [P, W, P, P, P]
    lib.nf4_dequantize.restype = ctypes.c_int
    lib.nf4_dequantize.argtypes = [W, P, P, P]
    lib.nf4_dequantize_dtype.restype = ctypes.c_int
    lib.nf4_dequantize_dtype.argtypes = [W, P, i32, P, P]
    lib.qlora_workspace_size.restype = sz
    lib.qlora_workspace_size.argtypes = [i64, W, i32, i32, i32]
    lib.qlora_forward.restype = ctypes.c_int
    lib.qlora_forward.argtypes = [P, i64, W, P, P, P, i32, ctypes.c_float, i32, P, P, P, sz, P, P]
    lib.qlora_backward.restype = ctypes.c_int
    lib.qlora_backward.argtypes = [P, P, i64, W, P, P, P, i32, ctypes.c_float, i32, P, P, P, P, P,
                                   sz, P, P]
    lib.qlora_launch_count.restype = ctypes.c_int64
    lib.qlora_launch_count.argtypes = []
    lib.qlora_profile_enable.restype = None
    lib.qlora_profile_enable.argtypes = [ctypes.c_int]
    lib.qlora_profile_reset.restype = None
    lib.qlora_profile_reset.argtypes = []
    lib.qlora_profile_read.restype = ctypes.c_int
    lib.qlora_profile_read.argtypes = [i32, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_double)]
    lib.qlora_profile_kinds.restype = None
    lib.qlora_profile_kinds.argtypes = [ctypes.c_uint32]
    lib.qlora_profile_read_each.restype = ctypes.c_int
    lib.qlora_profile_read_each.argtypes = [i32, i64, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]
    lib.qlora_forward_noalloc.restype = ctypes.c_int
    lib.qlora_forward_noalloc.argtypes = [P, i64, W, P, P, P, i32, ctypes.c_float, i32, P, P, P, P]
    lib.qlora_selftest_wait_timeout.restype = ctypes.c_int
    lib.qlora_selftest_wait_timeout.argtypes = [P, P]
    lib.qlora_merge.restype = ctypes.c_int
    lib.qlora_merge.argtypes = [W, P, P, P, i32, ctypes.c_float, i32, P, P]
    lib.nf4_codebook.restype = ctypes.c_int
    lib.nf4_codebook.argtypes = [ctypes.c_double, P]
    lib.fp4_codebook.restype = ctypes.c_int
    lib.fp4_codebook.argtypes = [P]
    _lib = lib
    return lib


def strerror(code: int) -> str:
    try:
        return load().qlora_strerror(code).decode()
    except Exception:
        return str(code)


def check(code: int, what: str) -> None:
    if code != QLORA_OK:
        raise QLoRAError(code, what)
