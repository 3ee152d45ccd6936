"""The benchmark hooks: qlora_profile_* times only the kinds in the mask (kind
0 the tensor-core GEMM, 2 the quantize kernel), reads each launch's duration in
launch order, and refuses an unknown kind."""
import ctypes

import pytest
import torch

from helpers import dev_bf16
from bit_nf4_quantized_22_b200 import synth
from bit_nf4_quantized_22_b200.synth import LinearSpec

pytestmark = pytest.mark.gpu


def _read(lib, kind):
    n, ms = ctypes.c_int64(), ctypes.c_double()
    rc = lib.qlora_profile_read(kind, ctypes.byref(n), ctypes.byref(ms))
    return rc, n.value, ms.value


def _each(lib, kind, cap):
    arr = (ctypes.c_double * max(cap, 1))()
    n = ctypes.c_int64()
    rc = lib.qlora_profile_read_each(kind, cap, arr, ctypes.byref(n))
    return rc, n.value, list(arr[:min(cap, n.value)])


def _layer_and_quantize(qlib, a, w, spec):
    x, A, B, dy = dev_bf16(a["x"]), dev_bf16(a["A"]), dev_bf16(a["B"]), dev_bf16(a["dY"])
    y, T = qlib.forward(x, w, A, B, spec.alpha)
    qlib.backward(x, dy, w, A, B, spec.alpha, T=T)
    qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=True, out=w)
    torch.cuda.synchronize()


def test_profile_kinds_mask_and_each(qlib):
    from bit_nf4_quantized_22_b200 import _lib
    lib = _lib.load()
    spec = LinearSpec("p", 512, 768, 16, 32.0, True)
    a = synth.draw(spec, 128, 3, 0)
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=True)
    torch.cuda.synchronize()
    try:
        # every kind
        lib.qlora_profile_reset()
        lib.qlora_profile_enable(1)
        _layer_and_quantize(qlib, a, w, spec)
        lib.qlora_profile_enable(0)
        rc0, n0, ms0 = _read(lib, 0)
        rc2, n2, _ = _read(lib, 2)
        assert (rc0, rc2, n0, n2) == (0, 0, 2, 1) and ms0 > 0
        rc, n, each = _each(lib, 0, 8)
        assert rc == 0 and n == 2 and len(each) == 2
        assert all(t > 0 for t in each) and abs(sum(each) - ms0) <= 1e-6 * max(ms0, 1.0)
        rc, n, each1 = _each(lib, 0, 1)          # a short array takes the first launch only
        assert rc == 0 and n == 2 and each1 == each[:1]
        # only the GEMM
        lib.qlora_profile_reset()
        lib.qlora_profile_kinds(1 << 0)
        lib.qlora_profile_enable(1)
        _layer_and_quantize(qlib, a, w, spec)
        lib.qlora_profile_enable(0)
        assert _read(lib, 0)[:2] == (0, 2)
        assert _read(lib, 2)[:2] == (0, 0)
    finally:
        lib.qlora_profile_enable(0)
        lib.qlora_profile_kinds(0xFFFFFFFF)
    assert _read(lib, 5)[0] != 0 and _read(lib, -1)[0] != 0
    assert _each(lib, 0, -1)[0] != 0
    n = ctypes.c_int64()
    assert lib.qlora_profile_read_each(0, 4, None, ctypes.byref(n)) != 0
