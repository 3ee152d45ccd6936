"""GPU parity of qlora_merge against the oracle's merge (W_eff = dequant(W4)
+ (alpha/r) A B, stored [Dout, Din]; pooled: (A_p B)/g shared per group),
within the floating-point tolerance of the layer outputs, and exactly equal
to nf4_dequantize when the adapter is zero."""
import numpy as np
import pytest
import torch

from helpers import assert_close, dev_bf16, host_bits, host_f64
from bit_nf4_quantized_22_b200 import synth
from bit_nf4_quantized_22_b200.synth import LinearSpec

pytestmark = pytest.mark.gpu


def _case(orc, qlib, spec, cfg, lin=0):
    a = synth.draw(spec, 1, cfg, lin, which=("W", "A", "B"))
    cb = orc.nf4_codebook()
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=spec.double_quant)
    A, B = dev_bf16(a["A"]), dev_bf16(a["B"])
    out = qlib.merge(w, A, B, spec.alpha, spec.pool_group)
    torch.cuda.synchronize()
    ref_q = orc.quantize(a["W"], cb, spec.double_quant)
    Wt = orc.dequantize(ref_q, cb)
    ref = orc.merge(Wt, a["A"], a["B"], spec.r, spec.alpha, spec.pool_group)
    assert_close(host_f64(out), ref, "W_eff")
    return w, A, B, out


@pytest.mark.parametrize("Din,Dout,r,dq,pool", [
    (256, 256, 8, False, 1),
    (320, 200, 3, True, 1),       # ragged: Dout % 64, Din % 256, odd rank
    (1024, 136, 100, True, 1),    # rank past 64 (two 64-wide B^T pitches)
    (512, 136, 8, True, 64),      # pooled adapter
    (4096, 4096, 16, True, 1),
    (192, 204, 24, False, 1),     # Dout % 8 != 0: B staged element by element
    (4096, 1024, 256, True, 1),   # largest rank: two adapter buffers; several units per CTA
    (4096, 2048, 64, True, 64),   # pooled, several units and row tiles per CTA
])
def test_merge_matches_oracle(orc, qlib, Din, Dout, r, dq, pool):
    spec = LinearSpec("m", Din, Dout, r, 2.0 * r, dq, pool_group=pool)
    _case(orc, qlib, spec, 15, lin=Din + r)


def test_merge_zero_adapter_is_dequantize(orc, qlib):
    spec = LinearSpec("m", 512, 264, 16, 32.0, True)
    w, A, B, _ = _case(orc, qlib, spec, 15, lin=7)
    out = qlib.merge(w, A, torch.zeros_like(B), spec.alpha)
    deq = qlib.dequantize(w)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), host_bits(deq))


def test_merge_full_size_70b_sampled_rows(orc, qlib):
    """The 8192 -> 28672 weight with r = 64: every output checked on sampled rows."""
    spec = synth.CONFIGS[5]["linears"][0]
    a = synth.draw(spec, 1, 5, 0, which=("W", "A", "B"))
    cb = orc.nf4_codebook()
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=True)
    out = qlib.merge(w, dev_bf16(a["A"]), dev_bf16(a["B"]), spec.alpha)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 63, 64, 12345, 28671])
    ref_q = orc.quantize(a["W"][rows], cb, True)
    Wt = orc.dequantize(ref_q, cb)
    ref = orc.merge(Wt, a["A"], a["B"][:, rows], spec.r, spec.alpha)
    assert_close(host_f64(out[torch.from_numpy(rows).cuda()]), ref, "W_eff rows")
