"""The FP4 table on the GPU (bitsandbytes article (CSDN) 6.4-6.5: the
library's other 4-bit type, a float-style table; read as E2M1 / 6 with -0 and
+0 both present).  Quantize and dequantize are bit-exact against the oracle,
including weights in zero's basin (first nearest level: -0) and values at
and around every decision threshold; the layer is within the parity
tolerance on the small-M and the tensor-core paths."""
import numpy as np
import pytest
import torch

from helpers import assert_close, dev_bf16, host_f64, unpack
from test_gpu_quantize import _adversarial_W, _check_same
from bit_nf4_quantized_22_b200 import synth
from bit_nf4_quantized_22_b200.synth import LinearSpec

pytestmark = pytest.mark.gpu


def _fp4(orc):
    cb = orc.fp4_codebook()
    return cb


@pytest.mark.parametrize("block", [32, 64, 128, 256])
@pytest.mark.parametrize("dq", [False, True])
def test_fp4_quantize_bit_exact(orc, qlib, block, dq):
    cb = _fp4(orc)
    rng = np.random.default_rng(block + dq)
    W = (rng.standard_normal((64, 1024)) * 0.03).astype(np.float32)
    W[0, :8] = [1e-9, -1e-9, 0.0, -0.0, 1e-6, -1e-6, 3e-8, -3e-8]
    W[1, :block] = 0.0
    w = _check_same(orc, qlib, W, dq, cb, block)
    assert not np.any(unpack(w.packed.cpu().numpy()) == 8)      # the +0 code is never written


def test_fp4_adversarial_thresholds(orc, qlib):
    cb = _fp4(orc)
    W = _adversarial_W(cb)
    _check_same(orc, qlib, W, False, cb)
    _check_same(orc, qlib, W, True, cb)


def _layer_case(orc, qlib, spec, M, cfg):
    cb = _fp4(orc)
    cb_t = torch.from_numpy(cb.copy())
    a = synth.draw(spec, M, cfg, 0)
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=spec.double_quant, codebook=cb_t)
    x, A, B, dy = dev_bf16(a["x"]), dev_bf16(a["A"]), dev_bf16(a["B"]), dev_bf16(a["dY"])
    y, T = qlib.forward(x, w, A, B, spec.alpha, spec.pool_group, codebook=cb_t)
    dX, dA, dB = qlib.backward(x, dy, w, A, B, spec.alpha, spec.pool_group, T=T, codebook=cb_t)
    torch.cuda.synchronize()
    Wt = orc.dequantize(orc.quantize(a["W"], cb, spec.double_quant), cb)
    y_ref, _ = orc.forward(a["x"], Wt, a["A"], a["B"], spec.r, spec.alpha, spec.pool_group)
    dX_ref, dA_ref, dB_ref = orc.backward(a["x"], a["dY"], Wt, a["A"], a["B"], spec.r, spec.alpha,
                                          spec.pool_group)
    assert_close(host_f64(y), y_ref, "y")
    assert_close(host_f64(dX), dX_ref, "dX")
    assert_close(host_f64(dA), dA_ref, "dA")
    assert_close(host_f64(dB), dB_ref, "dB")


@pytest.mark.parametrize("M", [1, 16, 300])
def test_fp4_layer(orc, qlib, M):
    """M <= 16: the streamed GEMVs; M = 300: the tcgen05 GEMM."""
    _layer_case(orc, qlib, LinearSpec("fp4", 2048, 1032, 16, 32.0, True), M, 31)


def test_fp4_merge(orc, qlib):
    cb = _fp4(orc)
    cb_t = torch.from_numpy(cb.copy())
    spec = LinearSpec("fp4m", 512, 264, 8, 16.0, True)
    a = synth.draw(spec, 1, 32, 0, which=("W", "A", "B"))
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=True, codebook=cb_t)
    out = qlib.merge(w, dev_bf16(a["A"]), dev_bf16(a["B"]), spec.alpha, codebook=cb_t)
    torch.cuda.synchronize()
    Wt = orc.dequantize(orc.quantize(a["W"], cb, True), cb)
    ref = orc.merge(Wt, a["A"], a["B"], spec.r, spec.alpha)
    assert_close(host_f64(out), ref, "W_eff")
