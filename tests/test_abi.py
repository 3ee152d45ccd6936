"""The C-ABI library: it loads, exports every symbol include/qlora.h declares,
and rejects invalid arguments on the host (no GPU needed: validation runs
before anything is enqueued)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from conftest import ROOT

import bit_nf4_quantized_22_b200 as q
from bit_nf4_quantized_22_b200 import _lib


@pytest.fixture(scope="module")
def lib():
    from bit_nf4_quantized_22_b200 import build
    build.build()
    return q.load()


def header_functions():
    text = open(os.path.join(ROOT, "include", "qlora.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert set(names) == set(_lib.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_strerror(lib):
    assert lib.qlora_version() == 200
    assert lib.qlora_strerror(0) == b"ok"
    assert lib.qlora_strerror(4) == b"workspace too small"


def _cb(vals):
    return (ctypes.c_float * 16)(*vals)


def test_codebook_validation(lib):
    good = q.nf4_codebook().tolist()
    assert lib.qlora_check_codebook(_cb(good)) == 0
    bad_order = list(good); bad_order[3], bad_order[4] = bad_order[4], bad_order[3]
    no_zero = [v if v != 0 else 1e-3 for v in good]
    out_of_range = list(good); out_of_range[15] = 1.5
    nan = list(good); nan[2] = float("nan")
    for b in (bad_order, no_zero, out_of_range, nan):
        assert lib.qlora_check_codebook(_cb(b)) == _lib.QLORA_EINVAL
    assert lib.qlora_check_codebook(None) == _lib.QLORA_EINVAL


def _wc(rows=64, cols=128, dq=1, block=64, group=256, ptrs=True):
    fake = 1 << 20 if ptrs else 0   # never dereferenced: validation fails first or no launch
    return _lib.NF4WeightC(rows, cols, block, dq, group, 0, fake, fake, fake, fake, fake)


def test_dq_variant_validation(lib):
    """double_quant is a code kind 0..4; the mean-offset kind needs dq_mean."""
    cb = _cb(q.nf4_codebook().tolist())
    W = ctypes.c_void_p(1 << 20)
    for bad in (-1, 5):
        assert lib.nf4_quantize(W, ctypes.byref(_wc(dq=bad)), cb, None, None) == _lib.QLORA_EINVAL
    wc = _wc(dq=3)
    wc.dq_mean = None
    assert lib.nf4_quantize(W, ctypes.byref(wc), cb, None, None) == _lib.QLORA_EINVAL
    assert ctypes.sizeof(_lib.NF4WeightC) == 72 and _lib.NF4WeightC.dq_mean.offset == 64


def test_quantize_rejects_bad_arguments(lib):
    cb = _cb(q.nf4_codebook().tolist())
    W = ctypes.c_void_p(1 << 20)
    E = _lib
    assert lib.nf4_quantize(W, ctypes.byref(_wc(cols=100)), cb, None, None) == E.QLORA_EINVAL
    for blk in (16, 48, 512):
        assert lib.nf4_quantize(W, ctypes.byref(_wc(block=blk)), cb, None, None) == E.QLORA_EUNSUPPORTED
    assert lib.nf4_quantize(W, ctypes.byref(_wc(block=128, cols=192)), cb, None, None) == E.QLORA_EINVAL
    assert lib.nf4_dequantize(ctypes.byref(_wc(block=256, cols=128)), cb, W, None) == E.QLORA_EINVAL
    assert lib.nf4_dequantize(ctypes.byref(_wc(block=96)), cb, W, None) == E.QLORA_EUNSUPPORTED
    for bad_dtype in (-1, 3):
        assert lib.nf4_dequantize_dtype(ctypes.byref(_wc()), cb, bad_dtype, W, None) == E.QLORA_EINVAL
    assert lib.nf4_dequantize_dtype(ctypes.byref(_wc()), cb, 1, ctypes.c_void_p((1 << 20) + 8),
                                    None) == E.QLORA_EINVAL
    assert lib.nf4_dequantize_dtype(ctypes.byref(_wc(rows=0)), cb, 2, W, None) == E.QLORA_OK
    assert lib.nf4_quantize(W, ctypes.byref(_wc(group=128)), cb, None, None) == E.QLORA_EUNSUPPORTED
    assert lib.nf4_quantize(W, ctypes.byref(_wc(ptrs=False)), cb, None, None) == E.QLORA_EINVAL
    assert lib.nf4_quantize(None, ctypes.byref(_wc()), cb, None, None) == E.QLORA_EINVAL
    assert lib.nf4_quantize(ctypes.c_void_p((1 << 20) + 4), ctypes.byref(_wc()), cb, None, None) == E.QLORA_EINVAL
    assert lib.nf4_quantize(W, None, cb, None, None) == E.QLORA_EINVAL
    assert lib.nf4_quantize(W, ctypes.byref(_wc()), None, None, None) == E.QLORA_EINVAL
    # an empty weight is a valid no-op
    assert lib.nf4_quantize(W, ctypes.byref(_wc(rows=0)), cb, None, None) == E.QLORA_OK


def test_layer_rejects_bad_arguments(lib):
    cb = _cb(q.nf4_codebook().tolist())
    P = ctypes.c_void_p(1 << 20)
    w = _wc(rows=64, cols=128)
    E = _lib

    def fwd(M=4, wc=w, r=8, alpha=16.0, g=1, X=P, Y=P, ws=P, nbytes=1 << 30):
        return lib.qlora_forward(X, M, ctypes.byref(wc), cb, P, P, r, alpha, g, Y, None, ws, nbytes,
                                 None, None)

    assert fwd(r=0) == E.QLORA_EINVAL
    assert fwd(r=257) == E.QLORA_EINVAL
    assert fwd(alpha=float("inf")) == E.QLORA_EINVAL
    assert fwd(alpha=float("nan")) == E.QLORA_EINVAL
    assert fwd(g=2) == E.QLORA_EINVAL
    assert fwd(M=-1) == E.QLORA_EINVAL
    assert fwd(X=None) == E.QLORA_EINVAL
    assert fwd(Y=ctypes.c_void_p((1 << 20) + 2)) == E.QLORA_EINVAL
    assert fwd(wc=_wc(rows=60)) == E.QLORA_EUNSUPPORTED          # Dout % 8
    assert fwd(wc=_wc(rows=0)) == E.QLORA_EINVAL
    for blk in (32, 128, 256):                       # the layer needs blocks of 64
        assert fwd(wc=_wc(block=blk, cols=256)) == E.QLORA_EUNSUPPORTED
        assert lib.qlora_merge(ctypes.byref(_wc(block=blk, cols=256)), cb, P, P, 8, 16.0, 1, P,
                               None) == E.QLORA_EUNSUPPORTED
    assert fwd(nbytes=16) == E.QLORA_EWORKSPACE
    assert fwd(ws=None) == E.QLORA_EWORKSPACE
    assert fwd(M=0) == E.QLORA_OK                                 # empty batch: no-op
    rc = lib.qlora_backward(P, None, 4, ctypes.byref(w), cb, P, P, 8, 16.0, 1, None, P, P, P, P,
                            1 << 30, None, None)
    assert rc == E.QLORA_EINVAL
    # dA needs x
    rc = lib.qlora_backward(None, P, 4, ctypes.byref(w), cb, P, P, 8, 16.0, 1, None, None, P, None,
                            P, 1 << 30, None, None)
    assert rc == E.QLORA_EINVAL


def test_workspace_size_deterministic(lib):
    for M, rows, cols, r, g in [(1, 4096, 4096, 16, 1), (16, 256, 256, 8, 1), (4096, 11008, 4096, 64, 1),
                                (8192, 28672, 8192, 64, 64), (17, 200, 192, 3, 1)]:
        w = _wc(rows=rows, cols=cols)
        a = lib.qlora_workspace_size(M, ctypes.byref(w), r, g, 0)
        b = lib.qlora_workspace_size(M, ctypes.byref(w), r, g, 1)
        assert a > 0 and b > 0
        assert a == lib.qlora_workspace_size(M, ctypes.byref(w), r, g, 0)
    assert lib.qlora_workspace_size(4, ctypes.byref(_wc(cols=100)), 8, 1, 0) == 0
    assert lib.qlora_workspace_size(4, ctypes.byref(_wc()), 0, 1, 0) == 0


@pytest.mark.parametrize("delta", [None, 1 - 1 / 32, 0.9, 0.99, 0.75, 0.999])
def test_product_codebook_matches_oracle(orc, delta):
    """The library's nf4_codebook (its own inverse normal: AS 241 plus a
    Halley step) gives the oracle's table (bisection on erfc) bit for bit."""
    a = (q.nf4_codebook() if delta is None else q.nf4_codebook(delta)).numpy()
    b = orc.nf4_codebook() if delta is None else orc.nf4_codebook(delta)
    assert np.array_equal(a.view(np.int32), b.view(np.int32))
    assert a[0] == -1 and a[7] == 0 and a[15] == 1


def test_product_fp4_codebook_matches_oracle(orc, lib):
    """fp4_codebook (the library's E2M1 construction) gives the oracle's FP4
    table bit for bit, -0 included, and passes the codebook check."""
    a = q.fp4_codebook().numpy()
    b = orc.fp4_codebook()
    assert np.array_equal(a.view(np.int32), b.view(np.int32))
    assert lib.qlora_check_codebook(_cb(a.tolist())) == 0
    assert lib.fp4_codebook(None) == _lib.QLORA_EINVAL


def test_codebook_check_repeated_levels(lib):
    """Only the zero may repeat (twice, as -0 and +0); any other repeat, or a
    third zero, is refused."""
    base = q.nf4_codebook().tolist()
    two_zeros = base[:7] + [-0.0, 0.0] + base[9:]
    assert lib.qlora_check_codebook(_cb(two_zeros)) == 0
    three_zeros = base[:6] + [0.0, -0.0, 0.0] + base[9:]
    assert lib.qlora_check_codebook(_cb(three_zeros)) == _lib.QLORA_EINVAL
    repeat = list(base); repeat[11] = repeat[10]
    assert lib.qlora_check_codebook(_cb(repeat)) == _lib.QLORA_EINVAL


def test_codebook_call_rejects_bad_delta(lib):
    out = (ctypes.c_float * 16)()
    for bad in (0.5, 0.3, 1.0, 1.5, float("nan")):
        assert lib.nf4_codebook(bad, out) == _lib.QLORA_EINVAL
    assert lib.nf4_codebook(0.9, None) == _lib.QLORA_EINVAL
    assert lib.nf4_codebook(0.9677083333333333, out) == 0
    assert lib.qlora_check_codebook(out) == 0


def test_binding_requires_cuda_tensors(lib):
    W = torch.zeros(64, 64)
    with pytest.raises(TypeError):
        q.quantize(W)


def test_header_is_plain_c(tmp_path):
    """include/qlora.h is a C ABI: it compiles as strict C99 (and as C++),
    with no torch, CUDA or C++ types in its signatures."""
    import shutil
    import subprocess
    src = tmp_path / "use.c"
    src.write_text('#include "qlora.h"\n'
                   "int main(void) { nf4_weight_t w = {0}; (void)w;\n"
                   "  return qlora_version() > 0 ? 0 : 1; }\n")
    inc = os.path.join(ROOT, "include")
    for cc, flags in (("gcc", ["-std=c99", "-pedantic-errors", "-Wall", "-Werror"]),
                      ("g++", ["-std=c++17", "-Wall", "-Werror", "-x", "c++"])):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not installed")
        r = subprocess.run([cc, *flags, "-I", inc, "-fsyntax-only", str(src)],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
    text = open(os.path.join(inc, "qlora.h")).read()
    code = re.sub(r"//[^\n]*", "", re.sub(r"/\*.*?\*/", "", text, flags=re.S))   # comments may name them
    for word in ("torch", "at::", "cudaStream_t", "__nv_bfloat16", "std::"):
        assert word not in code, word
