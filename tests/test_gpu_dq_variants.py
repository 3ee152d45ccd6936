"""Double-quantization variants on the GPU against the oracle (bitsandbytes
article (CSDN) 7.2 gives the structure, not the 8-bit code; 4.1 gives the
symmetric INT8 absmax code): the signed INT8 code (step = group max / 127),
the code of the scales minus their group mean, and the 8-bit float (E4M3)
code (step = group max / 448).  Quantize and dequantize
are bit-exact (packed indices, codes, steps, means, bf16 weights); the layer
and the merge are within the parity tolerance."""
import numpy as np
import pytest
import torch

from helpers import assert_close, dev_bf16, host_bits, host_f64
from bit_nf4_quantized_22_b200 import synth
from bit_nf4_quantized_22_b200.synth import LinearSpec

pytestmark = pytest.mark.gpu

VARIANTS = ["s8", "mean", "f8"]


def _check(orc, qlib, W, variant, block=64, cb=None):
    cb = orc.nf4_codebook() if cb is None else cb
    cb_t = torch.from_numpy(cb.copy())
    ref = orc.quantize(W, cb, True, block=block, dq_variant=variant)
    w = qlib.quantize(torch.from_numpy(W).cuda(), double_quant=True, codebook=cb_t, block=block,
                      dq_variant=variant)
    torch.cuda.synchronize()
    assert np.array_equal(w.packed.cpu().numpy(), ref.packed)
    assert np.array_equal(w.codes.cpu().numpy(), ref.codes)
    assert np.array_equal(w.steps.cpu().numpy().view(np.uint32), ref.steps.view(np.uint32))
    if variant == "mean":
        assert np.array_equal(w.means.cpu().numpy().view(np.uint32), ref.offsets.view(np.uint32))
    deq = host_bits(qlib.dequantize(w, codebook=cb_t))
    assert np.array_equal(deq, orc.dequantize(ref, cb))
    return w


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("block", [32, 64, 128, 256])
def test_dq_variant_quantize_bit_exact(orc, qlib, variant, block):
    rng = np.random.default_rng(block + len(variant))
    W = (rng.standard_t(4, (96, 2048)) * 0.02).astype(np.float32)   # ragged last group
    W[5, :block] = 0.0                                               # an all-zero block
    W[9, :block] *= 40.0                                             # an outlier block
    _check(orc, qlib, W, variant, block)


@pytest.mark.parametrize("variant", VARIANTS)
def test_dq_variant_partial_groups(orc, qlib, variant):
    """A single partial group, and groups whose scales are all equal (the
    mean-offset step is then 0)."""
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((3, 320)) * 0.05).astype(np.float32)
    _check(orc, qlib, W, variant)
    Wc = np.tile(np.array([0.5, -0.25] * 32, np.float32), (8, 4))    # every block absmax 0.5
    _check(orc, qlib, Wc, variant)


def _layer(orc, qlib, spec, M, cfg, variant):
    cb = orc.nf4_codebook()
    a = synth.draw(spec, M, cfg, 0)
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=True, dq_variant=variant)
    x, A, B, dy = dev_bf16(a["x"]), dev_bf16(a["A"]), dev_bf16(a["B"]), dev_bf16(a["dY"])
    y, T = qlib.forward(x, w, A, B, spec.alpha, spec.pool_group)
    dX, dA, dB = qlib.backward(x, dy, w, A, B, spec.alpha, spec.pool_group, T=T)
    W_eff = qlib.merge(w, A, B, spec.alpha, spec.pool_group)
    torch.cuda.synchronize()
    Wt = orc.dequantize(orc.quantize(a["W"], cb, True, dq_variant=variant), cb)
    y_ref, _ = orc.forward(a["x"], Wt, a["A"], a["B"], spec.r, spec.alpha, spec.pool_group)
    dX_ref, dA_ref, dB_ref = orc.backward(a["x"], a["dY"], Wt, a["A"], a["B"], spec.r, spec.alpha,
                                          spec.pool_group)
    assert_close(host_f64(y), y_ref, "y")
    assert_close(host_f64(dX), dX_ref, "dX")
    assert_close(host_f64(dA), dA_ref, "dA")
    assert_close(host_f64(dB), dB_ref, "dB")
    assert_close(host_f64(W_eff), orc.merge(Wt, a["A"], a["B"], spec.r, spec.alpha, spec.pool_group),
                 "W_eff")


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M", [1, 16, 260])
def test_dq_variant_layer(orc, qlib, variant, M):
    """M <= 16: the streamed GEMVs (and, at Din/64 not a multiple of 8, the
    register GEMVs); M = 260: the tcgen05 GEMM."""
    _layer(orc, qlib, LinearSpec("dqv", 2048, 1032, 16, 32.0, True), M, 41, variant)
    _layer(orc, qlib, LinearSpec("dqr", 1088, 264, 8, 16.0, True), M, 42, variant)


def test_dq_f8_ties_and_subnormals(orc, qlib):
    """The E4M3 scale code on quotients that sit exactly on midpoints between
    neighbouring values (ties to the even code), one float either side of
    them, in the subnormal range and at the top: group max 448 makes the
    step exactly 1, so each quotient is the block absmax itself."""
    import torch
    vals = [float(v) for v in torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float()]
    a = [448.0]
    for lo, hi in zip(vals, vals[1:]):
        mid = np.float32((lo + hi) / 2)
        a += [float(mid), float(np.nextafter(mid, np.float32(0))), float(np.nextafter(mid, np.float32(1e9)))]
    rng = np.random.default_rng(3)
    a += list(rng.uniform(0, 448, 384 - len(a)))          # 384 blocks: 24 rows of 16
    a = np.array(a, np.float32)
    blocks = (rng.uniform(-1, 1, (a.size, 64)) * a[:, None] * 0.9).astype(np.float32)
    blocks[:, 11] = -a                                   # the block absmax is a
    for g in range(0, a.size, 256):                      # every group's max is 448: step 1
        blocks[g, 7] = 448.0
    _check(orc, qlib, blocks.reshape(-1, 64 * 16), "f8")
