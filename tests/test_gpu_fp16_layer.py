"""The layer in the fp16 compute dtype (bitsandbytes article (CSDN) 8.3: the
dequantized weight and the arithmetic are FP32, BF16 or FP16; 8.5: FP16's
narrower range) against the oracle's fp16 layer: x, A, B, dY, y and dX in
IEEE binary16, the weight dequantized to RN_fp16(RN32(a_hat c_q)), fp32
accumulation.  Same tolerance as the bf16 layer."""
import numpy as np
import pytest
import torch

from helpers import assert_close, host_bits, host_f64
from bit_nf4_quantized_22_b200 import synth
from bit_nf4_quantized_22_b200.synth import LinearSpec

pytestmark = pytest.mark.gpu


def dev_f16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).cuda()


def run_f16(orc, qlib, spec, M, cfg, lin=0, rows=None, check_dadb=True):
    a = synth.draw(spec, M, cfg, lin, fmt="fp16")
    cb = orc.nf4_codebook()
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=spec.double_quant,
                      compute_dtype=torch.float16)
    x, A, B, dy = dev_f16(a["x"]), dev_f16(a["A"]), dev_f16(a["B"]), dev_f16(a["dY"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, T = qlib.forward(x, w, A, B, spec.alpha, spec.pool_group, status=status)
    dX, dA, dB = qlib.backward(x, dy, w, A, B, spec.alpha, spec.pool_group, T=T, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert y.dtype == torch.float16 and dX.dtype == torch.float16
    ref_q = orc.quantize(a["W"], cb, spec.double_quant)
    Wt = orc.dequantize_dt(ref_q, cb, "fp16")
    sel = np.arange(M) if rows is None else rows
    y_ref, T_ref = orc.forward(a["x"][sel], Wt, a["A"], a["B"], spec.r, spec.alpha, spec.pool_group,
                               dtype="fp16")
    assert_close(host_f64(y)[sel], y_ref, "y")
    assert_close(host_f64(T)[sel], T_ref, "T")
    dX_ref = orc.backward_dx(a["dY"][sel], Wt, a["A"], a["B"], spec.r, spec.alpha, spec.pool_group,
                             dtype="fp16")
    assert_close(host_f64(dX)[sel], dX_ref, "dX")
    if check_dadb:
        dA_ref, dB_ref = orc.backward_dadb(a["x"], a["dY"], a["A"], a["B"], spec.r, spec.alpha,
                                           spec.pool_group, dtype="fp16")
        assert_close(host_f64(dA), dA_ref, "dA")
        assert_close(host_f64(dB), dB_ref, "dB")
    return w, a


def test_fp16_config1(orc, qlib):
    cfg = synth.CONFIGS[1]
    run_f16(orc, qlib, cfg["linears"][0], cfg["M"][0], 1)


@pytest.mark.parametrize("M", [1, 16])
def test_fp16_config2_decode(orc, qlib, M):
    run_f16(orc, qlib, synth.CONFIGS[2]["linears"][0], M, 2)


def test_fp16_config3_sampled(orc, qlib):
    cfg = synth.CONFIGS[3]
    rows = np.array([0, 1, 255, 256, 1023, 2048, 4000, 4095])
    run_f16(orc, qlib, cfg["linears"][0], cfg["M"][0], 3, rows=rows, check_dadb=False)


@pytest.mark.parametrize("M,Din,Dout,dq,g", [
    (5, 1088, 264, True, 1),      # register GEMVs (Din/64 = 17)
    (3, 1536, 296, False, 1),     # streamed GEMVs, ragged tile, half slice
    (9, 512, 136, True, 64),      # pooled adapter, GEMV
    (130, 512, 136, True, 64),    # pooled adapter, tensor-core path
    (300, 320, 264, True, 1),     # tensor-core path, ragged tiles
])
def test_fp16_paths(orc, qlib, M, Din, Dout, dq, g):
    run_f16(orc, qlib, LinearSpec("h", Din, Dout, 8, 16.0, dq, pool_group=g), M, 51, lin=Din + M)


def test_fp16_merge_and_dequantize(orc, qlib):
    """The merged weight in fp16 against the oracle's merge of the fp16
    dequantized weight; the fp16 dequantize is bit-exact."""
    spec = LinearSpec("hm", 512, 264, 8, 16.0, True)
    a = synth.draw(spec, 1, 52, 0, which=("W", "A", "B"), fmt="fp16")
    cb = orc.nf4_codebook()
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=True, compute_dtype=torch.float16)
    out = qlib.merge(w, dev_f16(a["A"]), dev_f16(a["B"]), spec.alpha)
    deq = qlib.dequantize(w, dtype=torch.float16)
    torch.cuda.synchronize()
    assert out.dtype == torch.float16
    Wt = orc.dequantize_dt(orc.quantize(a["W"], cb, True), cb, "fp16")
    assert np.array_equal(host_bits(deq), Wt)
    assert_close(host_f64(out), orc.merge(Wt, a["A"], a["B"], spec.r, spec.alpha, dtype="fp16"), "W_eff")


def test_fp16_inputs_required(qlib):
    """A weight set to fp16 takes fp16 arrays; bf16 ones are refused."""
    w = qlib.quantize(torch.randn(64, 128, device="cuda"), compute_dtype=torch.float16)
    x = torch.zeros(2, 128, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(128, 4, dtype=torch.float16, device="cuda")
    B = torch.zeros(4, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(TypeError):
        qlib.forward(x, w, A, B, 4.0)
