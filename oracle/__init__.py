"""CPU oracle for the QLoRA linear layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 reference of everything the CUDA library computes: the NF4
codebook, blockwise quantization with optional double quantization,
dequantization, and the layer forward/backward.  Only the test suite,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package.  It shares no code with the CUDA path; the arithmetic lives in
``nf4_oracle.c`` (each function there cites the passage it follows) and this
module only marshals numpy arrays into it.

Array conventions: bf16 tensors are passed as ``numpy.uint16`` bit patterns;
the weight is ``Wt:[Dout, Din]`` fp32; results of the layer are fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# 1 - (1/32 + 1/30)/2: the tail probability of the outermost NF4 level.
NF4_DELTA = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
DQ_GROUP = 256
BLOCK = 64
STATUS_NONFINITE = 1


def build(force: bool = False) -> str:
    """Compile nf4_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-ffp-contract=off", "-fopenmp",
               "-D_GNU_SOURCE", "-shared", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.orc_normal_cdf.restype = ctypes.c_double
        lib.orc_normal_cdf.argtypes = [ctypes.c_double]
        lib.orc_normal_ppf.restype = ctypes.c_double
        lib.orc_normal_ppf.argtypes = [ctypes.c_double]
        lib.orc_nf4_codebook.restype = None
        lib.orc_nf4_codebook.argtypes = [ctypes.c_double, P]
        lib.orc_fp4_codebook.restype = None
        lib.orc_fp4_codebook.argtypes = [P]
        lib.orc_e4m3_value.restype = ctypes.c_double
        lib.orc_e4m3_value.argtypes = [ctypes.c_int]
        lib.orc_e4m3_encode.restype = ctypes.c_int
        lib.orc_e4m3_encode.argtypes = [ctypes.c_double]
        lib.orc_quantize.restype = ctypes.c_int
        lib.orc_quantize.argtypes = [P, i64, i64, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P, P, P, P,
                                     P]
        lib.orc_dequantize.restype = None
        lib.orc_dequantize.argtypes = [i64, i64, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P, P, P, P,
                                       P, P]
        lib.orc_dequantize_dt.restype = None
        lib.orc_dequantize_dt.argtypes = [i64, i64, ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P, P, P,
                                          P, P, ctypes.c_int, P]
        lib.orc_fp16_bits.restype = None
        lib.orc_fp16_bits.argtypes = [P, i64, P]
        lib.orc_adapter_down.restype = None
        lib.orc_adapter_down.argtypes = [P, i64, i64, P, ctypes.c_int, ctypes.c_int, P, ctypes.c_int]
        lib.orc_fp16_decode.restype = None
        lib.orc_fp16_decode.argtypes = [P, i64, P]
        lib.orc_forward.restype = None
        lib.orc_forward.argtypes = [P, i64, i64, i64, P, P, P, ctypes.c_int, ctypes.c_double,
                                    ctypes.c_int, P, P, ctypes.c_int]
        lib.orc_merge.restype = None
        lib.orc_merge.argtypes = [i64, i64, P, P, P, ctypes.c_int, ctypes.c_double, ctypes.c_int, P,
                                  ctypes.c_int]
        lib.orc_grad_G.restype = None
        lib.orc_grad_G.argtypes = [P, i64, i64, P, ctypes.c_int, P, ctypes.c_int]
        lib.orc_backward_dx.restype = None
        lib.orc_backward_dx.argtypes = [P, i64, i64, i64, P, P, P, ctypes.c_int, ctypes.c_double,
                                        ctypes.c_int, P, ctypes.c_int]
        lib.orc_backward_dadb.restype = None
        lib.orc_backward_dadb.argtypes = [P, P, i64, i64, i64, P, P, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_int, P, P, ctypes.c_int]
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_num_threads.argtypes = []
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_L().orc_num_threads())


def normal_cdf(x: float) -> float:
    return float(_L().orc_normal_cdf(float(x)))


def normal_ppf(p: float) -> float:
    return float(_L().orc_normal_ppf(float(p)))


def nf4_codebook(delta: float = NF4_DELTA) -> np.ndarray:
    out = np.zeros(16, dtype=np.float32)
    _L().orc_nf4_codebook(float(delta), _p(out))
    return out


def fp4_codebook() -> np.ndarray:
    """The FP4 (E2M1 / 6) table: 16 non-decreasing fp32 levels, -0 before +0."""
    out = np.zeros(16, dtype=np.float32)
    _L().orc_fp4_codebook(_p(out))
    return out


def e4m3_value(code: int) -> float:
    """The value of an E4M3 code with the sign bit clear (0 .. 0x7E)."""
    return float(_L().orc_e4m3_value(int(code)))


def e4m3_encode(x: float) -> int:
    """The E4M3 code nearest to x >= 0 (ties to the even mantissa; >= 448 -> 448)."""
    return int(_L().orc_e4m3_encode(float(x)))


# Double-quantization codes of the first-level scales: the unsigned 8-bit
# code (step = max / 255), the signed INT8 absmax code (step = max / 127), the
# signed INT8 code of the scales minus their group mean, and the 8-bit float
# (E4M3) code (step = max / 448).
DQ_VARIANTS = {"u8": 1, "s8": 2, "mean": 3, "f8": 4}


@dataclass
class QuantizedWeight:
    rows: int
    cols: int
    double_quant: bool
    packed: np.ndarray            # uint8 [rows*cols/2]
    absmax: np.ndarray | None     # float32 [nb]
    codes: np.ndarray | None      # uint8 [nb] (int8 two's complement for "mean")
    steps: np.ndarray | None      # float32 [ceil(nb/256)]
    status: int
    block: int = BLOCK            # weights per first-level scale
    dq_variant: str = "u8"
    offsets: np.ndarray | None = None   # float32 [ceil(nb/256)] group means ("mean")

    @property
    def dq_code(self) -> int:
        return DQ_VARIANTS[self.dq_variant] if self.double_quant else 0

    @property
    def nbytes(self) -> int:
        n = self.packed.nbytes
        for a in (self.absmax, self.codes, self.steps, self.offsets):
            if a is not None:
                n += a.nbytes
        return n


def quantize(W: np.ndarray, codebook: np.ndarray, double_quant: bool,
             dq_group: int = DQ_GROUP, block: int = BLOCK, dq_variant: str = "u8") -> QuantizedWeight:
    W = _c(W, np.float32)
    rows, cols = W.shape
    assert block % 2 == 0 and cols % block == 0
    cb = _c(codebook, np.float32)
    nb = rows * cols // block
    packed = np.zeros(rows * cols // 2, dtype=np.uint8)
    absmax = None if double_quant else np.zeros(nb, dtype=np.float32)
    codes = np.zeros(nb, dtype=np.uint8) if double_quant else None
    ng = (nb + dq_group - 1) // dq_group
    steps = np.zeros(ng, dtype=np.float32) if double_quant else None
    offsets = np.zeros(ng, dtype=np.float32) if double_quant and dq_variant == "mean" else None
    dq = DQ_VARIANTS[dq_variant] if double_quant else 0
    st = _L().orc_quantize(_p(W), rows, cols, block, _p(cb), dq, dq_group,
                           _p(packed), _p(absmax), _p(codes), _p(steps), _p(offsets))
    return QuantizedWeight(rows, cols, double_quant, packed, absmax, codes, steps, int(st), block,
                           dq_variant, offsets)


def dequantize(q: QuantizedWeight, codebook: np.ndarray, dq_group: int = DQ_GROUP) -> np.ndarray:
    """bf16 bit patterns [rows, cols]."""
    cb = _c(codebook, np.float32)
    out = np.zeros((q.rows, q.cols), dtype=np.uint16)
    _L().orc_dequantize(q.rows, q.cols, q.block, _p(cb), q.dq_code, dq_group, _p(q.packed),
                        _p(q.absmax), _p(q.codes), _p(q.steps), _p(q.offsets), _p(out))
    return out


DTYPES = {"bf16": 0, "fp16": 1, "fp32": 2}


def dequantize_dt(q: QuantizedWeight, codebook: np.ndarray, dtype: str,
                  dq_group: int = DQ_GROUP) -> np.ndarray:
    """[rows, cols] in the compute dtype: uint16 bit patterns for bf16 and
    fp16, float32 values for fp32."""
    cb = _c(codebook, np.float32)
    out = np.zeros((q.rows, q.cols), dtype=np.float32 if dtype == "fp32" else np.uint16)
    _L().orc_dequantize_dt(q.rows, q.cols, q.block, _p(cb), q.dq_code, dq_group,
                           _p(q.packed), _p(q.absmax), _p(q.codes), _p(q.steps), _p(q.offsets),
                           DTYPES[dtype], _p(out))
    return out


def fp16_bits(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32).reshape(-1)
    out = np.zeros(x.size, dtype=np.uint16)
    _L().orc_fp16_bits(_p(x), x.size, _p(out))
    return out


# 16-bit element formats of the layer's arrays (the compute dtype)
FMT16 = {"bf16": 0, "fp16": 1}


def fp16_decode(h: np.ndarray) -> np.ndarray:
    h = _c(h, np.uint16).reshape(-1)
    out = np.zeros(h.size, dtype=np.float64)
    _L().orc_fp16_decode(_p(h), h.size, _p(out))
    return out


def adapter_down(X, A, r: int, pool_group: int = 1, dtype: str = "bf16") -> np.ndarray:
    X = _c(X, np.uint16)
    A = _c(A, np.uint16)
    M, Din = X.shape
    T = np.zeros((M, r), dtype=np.float64)
    _L().orc_adapter_down(_p(X), M, Din, _p(A), r, pool_group, _p(T), FMT16[dtype])
    return T


def forward(X, Wt, A, B, r: int, alpha: float, pool_group: int = 1, dtype: str = "bf16"):
    """Returns (y fp64 [M, Dout], T fp64 [M, r]).  X, Wt, A, B hold bf16 or
    fp16 bit patterns (dtype)."""
    X = _c(X, np.uint16)
    Wt = _c(Wt, np.uint16)
    A = _c(A, np.uint16)
    B = _c(B, np.uint16)
    M, Din = X.shape
    Dout = Wt.shape[0]
    Y = np.zeros((M, Dout), dtype=np.float64)
    T = np.zeros((M, r), dtype=np.float64)
    _L().orc_forward(_p(X), M, Din, Dout, _p(Wt), _p(A), _p(B), r, float(alpha), pool_group,
                     _p(Y), _p(T), FMT16[dtype])
    return Y, T


def merge(Wt, A, B, r: int, alpha: float, pool_group: int = 1, dtype: str = "bf16") -> np.ndarray:
    """W_eff fp64 [Dout, Din] = dequantized Wt + (alpha/r) (A B) in the stored
    orientation; pooled: (alpha/r)/g (A_p B) shared by each group's inputs."""
    Wt = _c(Wt, np.uint16)
    A = _c(A, np.uint16)
    B = _c(B, np.uint16)
    Dout, Din = Wt.shape
    out = np.zeros((Dout, Din), dtype=np.float64)
    _L().orc_merge(Din, Dout, _p(Wt), _p(A), _p(B), r, float(alpha), pool_group, _p(out), FMT16[dtype])
    return out


def grad_G(dY, B, r: int, dtype: str = "bf16") -> np.ndarray:
    dY = _c(dY, np.uint16)
    B = _c(B, np.uint16)
    M, Dout = dY.shape
    G = np.zeros((M, r), dtype=np.float64)
    _L().orc_grad_G(_p(dY), M, Dout, _p(B), r, _p(G), FMT16[dtype])
    return G


def backward_dx(dY, Wt, A, B, r: int, alpha: float, pool_group: int = 1,
                dtype: str = "bf16") -> np.ndarray:
    dY = _c(dY, np.uint16)
    Wt = _c(Wt, np.uint16)
    A = _c(A, np.uint16)
    B = _c(B, np.uint16)
    M, Dout = dY.shape
    Din = Wt.shape[1]
    dX = np.zeros((M, Din), dtype=np.float64)
    _L().orc_backward_dx(_p(dY), M, Din, Dout, _p(Wt), _p(A), _p(B), r, float(alpha),
                         pool_group, _p(dX), FMT16[dtype])
    return dX


def backward_dadb(X, dY, A, B, r: int, alpha: float, pool_group: int = 1,
                  want_dA: bool = True, want_dB: bool = True, dtype: str = "bf16"):
    X = _c(X, np.uint16)
    dY = _c(dY, np.uint16)
    A = _c(A, np.uint16)
    B = _c(B, np.uint16)
    M, Din = X.shape
    Dout = dY.shape[1]
    dA = np.zeros((Din // pool_group, r), dtype=np.float64) if want_dA else None
    dB = np.zeros((r, Dout), dtype=np.float64) if want_dB else None
    _L().orc_backward_dadb(_p(X), _p(dY), M, Din, Dout, _p(A), _p(B), r, float(alpha),
                           pool_group, _p(dA), _p(dB), FMT16[dtype])
    return dA, dB


def backward(X, dY, Wt, A, B, r: int, alpha: float, pool_group: int = 1, dtype: str = "bf16"):
    """Returns (dX, dA, dB), all fp64."""
    dX = backward_dx(dY, Wt, A, B, r, alpha, pool_group, dtype)
    dA, dB = backward_dadb(X, dY, A, B, r, alpha, pool_group, dtype=dtype)
    return dX, dA, dB
