"""GPU parity of nf4_quantize / nf4_dequantize against the oracle: bit-exact
on packed indices, absmax, double-quant codes and steps, and dequantized bf16
weights."""
import numpy as np
import pytest
import torch

from helpers import dev_bf16, host_bits, unpack
from bit_nf4_quantized_22_b200 import synth

pytestmark = pytest.mark.gpu


def _gpu_quant(qlib, W, dq, cb=None, block=64):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = qlib.quantize(torch.from_numpy(W).cuda(), double_quant=dq, codebook=cb, status=status,
                      block=block)
    torch.cuda.synchronize()
    return w, int(status.item())


def _check_same(orc, qlib, W, dq, cb_np=None, block=64):
    cb_np = orc.nf4_codebook() if cb_np is None else cb_np
    cb_t = torch.from_numpy(cb_np.copy())
    ref = orc.quantize(W, cb_np, dq, block=block)
    w, st = _gpu_quant(qlib, W, dq, cb_t, block)
    assert st == ref.status
    gp = w.packed.cpu().numpy()
    if not np.array_equal(gp, ref.packed):
        a, b = unpack(gp), unpack(ref.packed)
        bad = np.flatnonzero(a != b)
        raise AssertionError(f"{bad.size} indices differ, first at {bad[:5]}: gpu {a[bad[:5]]} ref {b[bad[:5]]}")
    if dq:
        assert np.array_equal(w.steps.cpu().numpy().view(np.uint32), ref.steps.view(np.uint32))
        assert np.array_equal(w.codes.cpu().numpy(), ref.codes)
    else:
        assert np.array_equal(w.absmax.cpu().numpy().view(np.uint32), ref.absmax.view(np.uint32))
    deq = host_bits(qlib.dequantize(w, codebook=cb_t))
    assert np.array_equal(deq, orc.dequantize(ref, cb_np))
    return w


@pytest.mark.parametrize("dq", [False, True])
def test_config1_quantize(orc, qlib, dq):
    spec = synth.CONFIGS[1]["linears"][0]
    W = synth.draw(spec, 16, 1, which=("W",))["W"]
    _check_same(orc, qlib, W, dq)


@pytest.mark.parametrize("shape", [(8, 64), (3, 192), (37, 320), (256, 4160)])
@pytest.mark.parametrize("dq", [False, True])
def test_ragged_shapes(orc, qlib, shape, dq):
    """Block counts that leave a partial CTA and a partial double-quant group."""
    rng = np.random.default_rng(hash(shape) % 2**32)
    W = (rng.standard_t(4, size=shape) * 0.02).astype(np.float32)
    _check_same(orc, qlib, W, dq)


def _adversarial_W(cb, block=64):
    """Blocks holding +-a and values at and within a few ulps of every decision
    threshold, for several absmax magnitudes (incl. subnormal-range scales)."""
    from fractions import Fraction as Fr
    rows = []
    for a in (1.0, 0.0371, 3.1e-3, 2.0 ** -120, 1.7e30, 6.1e-39):
        a = np.float32(a)
        vals = []
        for j in range(15):
            t = (Fr(float(cb[j])) + Fr(float(cb[j + 1]))) / 2 * Fr(float(a))
            x = np.float32(float(t))
            for k in range(-3, 4):
                y = x
                for _ in range(abs(k)):
                    y = np.nextafter(y, np.float32(np.inf if k > 0 else -np.inf))
                vals.append(y)
        vals = np.array(vals, dtype=np.float32)
        for s in range(0, vals.size, block - 2):
            blk = np.zeros(block, np.float32)
            blk[0], blk[1] = a, -a
            chunk = vals[s:s + block - 2]
            blk[2:2 + chunk.size] = chunk
            rows.append(blk)
    return np.stack(rows).reshape(-1, block)


def test_adversarial_thresholds(orc, qlib):
    W = _adversarial_W(orc.nf4_codebook())
    _check_same(orc, qlib, W, False)
    _check_same(orc, qlib, W, True)


def test_custom_codebooks(orc, qlib):
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((64, 256)) * 0.05).astype(np.float32)
    W[3, :64] = 0
    uniform = np.array([-1, -.75, -.5, -.375, -.25, -.125, -.0625, 0, .0625, .125, .25, .375,
                        .5, .625, .75, 1], dtype=np.float32)
    tiny = np.array([-1, -.9, -.8, -.7, -.6, -.5, -2.0 ** -60, 0, .5, .6, .7, .75, .8, .85, .9, 1],
                    dtype=np.float32)
    # levels at least 0.1 apart: thresholds far enough apart for the bin-table kernel
    wide = np.array([-1, -.85, -.7, -.55, -.4, -.25, -.1, 0, .1, .25, .4, .55, .7, .8, .9, 1],
                    dtype=np.float32)
    for cb in (uniform, tiny, orc.nf4_codebook(1 - 1 / 32), wide):
        # exact ties on the uniform table's midpoints, and on this table's own
        W2 = W.copy()
        W2[0, :16] = (np.concatenate([[1.0], (uniform[:-1] + uniform[1:]) / 2])).astype(np.float32)
        W2[1, :16] = (np.concatenate([[1.0], (cb[:-1] + cb[1:]) / 2])).astype(np.float32)
        W2[1, 16:31] = np.nextafter(W2[1, 1:16], np.float32(-np.inf))
        W2[1, 31:46] = np.nextafter(W2[1, 1:16], np.float32(np.inf))
        _check_same(orc, qlib, W2, True, cb)


def test_special_blocks_and_status(orc, qlib):
    W = np.zeros((4, 128), np.float32)
    W[1, :64] = -0.0
    W[2, 0], W[2, 1] = 0.5, -0.5
    W[3, 64:] = 1e-42                       # subnormal block
    _check_same(orc, qlib, W, True)
    # scales outside [2^-100, 2^100] take the search path of the fast kernel
    rng = np.random.default_rng(5)
    W2 = (rng.standard_normal((4, 256)) * 0.05).astype(np.float32)
    W2[0, :64] *= np.float32(2.0 ** 110)
    W2[1, 64:128] *= np.float32(2.0 ** -110)
    W2[2, 128:192] *= np.float32(2.0 ** 100)
    W2[3, 192:] *= np.float32(2.0 ** -96)
    _check_same(orc, qlib, W2, False)
    _check_same(orc, qlib, W2, True)
    W[0, 5] = np.nan
    _, st = _gpu_quant(qlib, W, True)
    assert st == 1
    W[0, 5] = np.inf
    _, st = _gpu_quant(qlib, W, False)
    assert st == 1


def test_double_quant_code_ties(orc, qlib):
    """Block scales on and next to the code midpoints: group max 255/16 makes
    the step exactly 1/16, so a = (k + 1/2)/16 is a tie that rounds to even."""
    rng = np.random.default_rng(17)
    nb = 256
    a = np.empty(nb, np.float32)
    a[0] = 255 / 16
    k = np.arange(1, nb) % 255
    ties = ((k + 0.5) / 16).astype(np.float32)
    a[1:] = ties
    a[100:140] = np.nextafter(ties[99:139], np.float32(np.inf))
    a[140:180] = np.nextafter(ties[139:179], np.float32(-np.inf))
    blocks = (rng.uniform(-1, 1, (nb, 64)) * a[:, None] * 0.9).astype(np.float32)
    blocks[:, 7] = -a
    W = blocks.reshape(4, 64 * 64)
    _check_same(orc, qlib, W, True)
    ref = orc.quantize(W, orc.nf4_codebook(), True)
    assert ref.steps[0] == np.float32(1 / 16)
    assert list(ref.codes[1:4]) == [2, 2, 4] and ref.codes[255] == 0   # 1.5, 2.5, 3.5, 0.5


def test_empty_weight(qlib):
    w = qlib.NF4Weight.empty(0, 64, True)
    qlib.quantize(torch.zeros(0, 64, device="cuda"), out=w)
    torch.cuda.synchronize()


@pytest.mark.parametrize("cfg,lin", [(3, 0), (4, 6)])
def test_full_size_quantize(orc, qlib, cfg, lin):
    """Full-size matrices of the training-shaped workloads, bit-exact."""
    spec = synth.CONFIGS[cfg]["linears"][lin]
    W = synth.draw(spec, 1, cfg, lin, which=("W",))["W"]
    _check_same(orc, qlib, W, spec.double_quant)


def test_full_size_quantize_70b(orc, qlib):
    """The 8192 x 28672 matrix (235M weights), bit-exact on every output."""
    spec = synth.CONFIGS[5]["linears"][0]
    W = synth.draw(spec, 1, 5, 0, which=("W",))["W"]
    _check_same(orc, qlib, W, True)


# ------------------------------------------------------------ other block sizes

BLOCKS = [32, 128, 256]


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("shape,dq", [((3, 256), False), ((37, 512), True), ((129, 1280), True),
                                      ((129, 1280), False)])
def test_block_sizes_ragged(orc, qlib, block, shape, dq):
    """Blocks of 32, 128 and 256 weights: partial CTAs and partial double-quant
    groups, bit-exact indices, scales and dequantized weights."""
    rng = np.random.default_rng(block * 1000 + shape[0])
    W = (rng.standard_t(4, size=shape) * 0.02).astype(np.float32)
    w = _check_same(orc, qlib, W, dq, block=block)
    nb = W.size // block
    assert (w.codes if dq else w.absmax).numel() == nb


@pytest.mark.parametrize("block", BLOCKS)
def test_block_sizes_adversarial_and_special(orc, qlib, block):
    cb = orc.nf4_codebook()
    W = _adversarial_W(cb, block)
    _check_same(orc, qlib, W, False, block=block)
    _check_same(orc, qlib, W, True, block=block)
    rng = np.random.default_rng(block)
    S = (rng.standard_normal((6, 2 * 256)) * 0.05).astype(np.float32)
    S[0, :block] = 0.0                                  # all-zero block
    S[1, :block] = -0.0
    S[2, block:2 * block] = 1e-42                       # subnormal block
    S[3, :block] *= np.float32(2.0 ** 110)              # scales outside [2^-100, 2^100]: the search path
    S[4, block:2 * block] *= np.float32(2.0 ** -110)
    S[5, :block] *= np.float32(2.0 ** -96)
    _check_same(orc, qlib, S, False, block=block)
    _check_same(orc, qlib, S, True, block=block)
    S[0, 3] = np.nan
    assert _gpu_quant(qlib, S, True, block=block)[1] == 1


@pytest.mark.parametrize("block", [32, 256])
def test_block_sizes_custom_codebooks(orc, qlib, block):
    """A codebook too dense for the bin table (the search path throughout) and
    one the table serves, with exact ties on their own midpoints."""
    rng = np.random.default_rng(19 + block)
    W = (rng.standard_normal((16, 512)) * 0.05).astype(np.float32)
    tiny = np.array([-1, -.9, -.8, -.7, -.6, -.5, -2.0 ** -60, 0, .5, .6, .7, .75, .8, .85, .9, 1],
                    dtype=np.float32)
    wide = np.array([-1, -.85, -.7, -.55, -.4, -.25, -.1, 0, .1, .25, .4, .55, .7, .8, .9, 1],
                    dtype=np.float32)
    for cb in (tiny, wide):
        W2 = W.copy()
        W2[1, :16] = (np.concatenate([[1.0], (cb[:-1] + cb[1:]) / 2])).astype(np.float32)
        W2[1, 16:31] = np.nextafter(W2[1, 1:16], np.float32(-np.inf))
        _check_same(orc, qlib, W2, True, cb, block=block)


def test_block_size_full_size_up_proj(orc, qlib):
    """The 4096 x 11008 weight in blocks of 128 with double quantization."""
    spec = synth.CONFIGS[3]["linears"][0]
    W = synth.draw(spec, 1, 3, 0, which=("W",))["W"]
    _check_same(orc, qlib, W, True, block=128)


def test_block_size_layer_calls_refused(qlib):
    """The layer kernels read one scale per 64 inputs: other sizes are refused
    loudly rather than misread."""
    W = torch.zeros(64, 256, device="cuda")
    w = qlib.quantize(W, block=32)
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(256, 8, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        qlib.forward(x, w, A, B, 16.0)
    with pytest.raises(RuntimeError):
        qlib.merge(w, A, B, 16.0)


# ------------------------------------------------------------ compute dtypes

@pytest.mark.parametrize("block", [32, 64, 256])
@pytest.mark.parametrize("dq", [False, True])
def test_dequantize_compute_dtypes(orc, qlib, block, dq):
    """fp16 and fp32 outputs bit-exact against the oracle, including scales
    whose products overflow fp16 and ones in its subnormal range."""
    rng = np.random.default_rng(41 + block)
    cb = orc.nf4_codebook()
    W = (rng.standard_t(4, (37, 1024)) * 0.5).astype(np.float32)
    W[3] *= np.float32(1e5)
    W[5] *= np.float32(1e-6)
    W[7, :block] = 0.0
    ref = orc.quantize(W, cb, dq, block=block)
    w, _ = _gpu_quant(qlib, W, dq, block=block)
    for name, dt in (("fp16", torch.float16), ("fp32", torch.float32), ("bf16", torch.bfloat16)):
        got = qlib.dequantize(w, dtype=dt)
        torch.cuda.synchronize()
        want = orc.dequantize_dt(ref, cb, name)
        g = got.cpu().view(torch.int32 if dt == torch.float32 else torch.int16).numpy()
        assert np.array_equal(g.view(want.dtype), want), name
