"""Pins for the oracle's QLoRA layer forward and backward.

Forward: y = x dequant(W4) + (alpha/r) x A B ("从 LoRA 到 QLoRA、QA-LoRA" section 2,
W_eff = dequant(W4) + (alpha/r) A B; bitsandbytes article (CSDN) 12.2/12.4,
s = lora_alpha / r).  Backward: the gradient runs through the frozen base for
dX, and A, B get gradients; W gets none (CSDN 12.4).  Pooled adapter:
y = x dequant(W4) + pool(x) A B (QA-LoRA sections 3-5).
"""
from fractions import Fraction as Fr

import numpy as np
import pytest

from conftest import floats, read_golden


def bf16(x):
    """fp64/fp32 -> bf16 bits with round-to-nearest-even (input encoding)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def f64(b):
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- worked examples

def test_worked_lora_example(orc):
    """Din=4, Dout=2, r=1: with a zero base, x = e_i gives row i of dW = A x B.
    alpha = r so that alpha/r = 1 (the example carries no scale)."""
    g = read_golden("lora_worked_example.txt")
    Din, Dout, r = int(g["Din"]), int(g["Dout"]), int(g["r"])
    A = bf16(np.array(floats(g["A"])).reshape(Din, r))
    B = bf16(np.array(floats(g["B"])).reshape(r, Dout))
    dW = np.array(floats(g["dW"])).reshape(Din, Dout)
    Wt = np.zeros((Dout, Din), dtype=np.uint16)       # dequant of an all-zero block is 0
    X = bf16(np.eye(Din))
    Y, T = orc.forward(X, Wt, A, B, r, alpha=r)
    # exactly A_i * B with the bf16 inputs ...
    np.testing.assert_array_equal(Y, f64(A) @ f64(B))
    # ... which is the printed dW up to the bf16 rounding of B (0.1, -0.2)
    np.testing.assert_allclose(Y, dW, rtol=2 ** -8, atol=0)
    np.testing.assert_array_equal(T, f64(A))


def test_rank2_is_sum_of_outer_products(orc):
    """r = 2: dW = a1 b1 + a2 b2 (same section, "如果 r=2")."""
    A = bf16(np.array([[2.0, 1.0], [0.5, -1.0], [-1.0, 0.25], [1.5, 2.0]]))
    B = bf16(np.array([[0.1, -0.2], [0.5, 0.75]]))
    Y, _ = orc.forward(bf16(np.eye(4)), np.zeros((2, 4), np.uint16), A, B, 2, alpha=2)
    a, b = f64(A), f64(B)
    np.testing.assert_array_equal(Y, np.outer(a[:, 0], b[0]) + np.outer(a[:, 1], b[1]))


def test_pooled_example(orc):
    g = read_golden("pooled_adapter_example.txt")
    gs = int(g["group_size"])
    X = bf16(np.array([floats(g["x"])]))
    A = bf16(np.array(floats(g["A"])).reshape(-1, 1))
    B = bf16(np.array(floats(g["B"])).reshape(1, -1))
    Y, T = orc.forward(X, np.zeros((2, 4), np.uint16), A, B, 1, alpha=1, pool_group=gs)
    assert T[0, 0] == float(g["pool_x_A"])                      # 4.75
    np.testing.assert_allclose(Y[0], floats(g["y"]), rtol=2 ** -8)
    np.testing.assert_array_equal(Y[0], 4.75 * f64(B)[0])
    # pool(x) itself: with A = e_k the adapter output T is pool(x)[k]
    for k, pk in enumerate(floats(g["pool_x"])):
        Ak = np.zeros((2, 1)); Ak[k, 0] = 1
        _, Tk = orc.forward(X, np.zeros((2, 4), np.uint16), bf16(Ak), B, 1, 1, pool_group=gs)
        assert Tk[0, 0] == pk


def test_pooled_group_shared_update(orc):
    """Every input column of a group receives the same update A_g B / g:
    [0.1, -0.2] for group 1 and [0.025, -0.05] for group 2."""
    g = read_golden("pooled_adapter_example.txt")
    gs = int(g["group_size"])
    A = bf16(np.array(floats(g["A"])).reshape(-1, 1))
    B = bf16(np.array(floats(g["B"])).reshape(1, -1))
    Y, _ = orc.forward(bf16(np.eye(4)), np.zeros((2, 4), np.uint16), A, B, 1, 1, pool_group=gs)
    g1, g2 = floats(g["group1_update"]), floats(g["group2_update"])
    for col, ref in ((0, g1), (1, g1), (2, g2), (3, g2)):
        np.testing.assert_allclose(Y[col], ref, rtol=2 ** -8)
    assert np.array_equal(Y[0], Y[1]) and np.array_equal(Y[2], Y[3])
    # dense-equivalence: pooled == dense LoRA with A_dense[k'g+i] = A_p[k'] / g
    A_dense = bf16(np.repeat(f64(A) / gs, gs, axis=0))
    Yd, _ = orc.forward(bf16(np.eye(4)), np.zeros((2, 4), np.uint16), A_dense, B, 1, 1)
    np.testing.assert_array_equal(Y, Yd)


# ---------------------------------------------------------------- base path

def _problem(rng, M, Din, Dout, r, wscale=0.02):
    W = (rng.standard_normal((Dout, Din)) * wscale).astype(np.float32)
    X = bf16(rng.standard_normal((M, Din)))
    A = bf16(rng.standard_normal((Din, r)) / np.sqrt(r))
    B = bf16(rng.standard_normal((r, Dout)) * 0.01)
    dY = bf16(rng.standard_normal((M, Dout)))
    return W, X, A, B, dY


def test_B_zero_is_plain_matmul(orc):
    """B = 0 (LoRA's initialisation, airsota card section 3) leaves
    y = x dequant(W4), here checked against numpy's matmul; dA = 0."""
    rng = np.random.default_rng(11)
    W, X, A, B, dY = _problem(rng, 5, 128, 24, 4)
    B[:] = 0
    cb = orc.nf4_codebook()
    Wt = orc.dequantize(orc.quantize(W, cb, True), cb)
    Y, _ = orc.forward(X, Wt, A, B, 4, alpha=8)
    np.testing.assert_allclose(Y, f64(X) @ f64(Wt).T, rtol=1e-13, atol=1e-13)
    dX, dA, dB = orc.backward(X, dY, Wt, A, B, 4, 8)
    assert np.all(dA == 0)
    np.testing.assert_allclose(dX, f64(dY) @ f64(Wt), rtol=1e-13, atol=1e-13)


def test_scale_alpha_over_r(orc):
    """alpha = r gives the unscaled LoRA update of the worked example; the
    adapter term is proportional to alpha and inversely to r."""
    rng = np.random.default_rng(12)
    W, X, A, B, _ = _problem(rng, 3, 64, 8, 2)
    Wt = np.zeros((8, 64), np.uint16)
    y1, _ = orc.forward(X, Wt, A, B, 2, alpha=2)
    y3, _ = orc.forward(X, Wt, A, B, 2, alpha=6)
    np.testing.assert_allclose(y1, f64(X) @ f64(A) @ f64(B), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(y3, 3 * y1, rtol=1e-13, atol=1e-15)


def test_dequantized_weight_dq_rounding(orc):
    """Dequant with double quant: w = RN_bf16(RN32(RN32(code * f) * c_q)),
    recomputed here exactly from the stored codes."""
    rng = np.random.default_rng(13)
    cb = orc.nf4_codebook()
    W = (rng.standard_normal((4, 640)) * 0.02).astype(np.float32)
    q = orc.quantize(W, cb, True)
    out = orc.dequantize(q, cb).reshape(-1)
    idx = np.empty(W.size, np.int64)
    idx[0::2] = q.packed >> 4
    idx[1::2] = q.packed & 15
    for e in range(0, W.size, 7):
        b = e // 64
        ah = np.float32(Fr(int(q.codes[b])) * Fr(float(q.steps[b // 256])))
        w32 = np.float32(Fr(float(ah)) * Fr(float(cb[idx[e]])))
        assert out[e] == bf16(w32)


# ---------------------------------------------------------------- backward by finite differences

@pytest.mark.parametrize("pool_group", [1, 64])
def test_backward_finite_differences(orc, pool_group):
    """L = sum(dY * y) is linear in x, in A (B fixed) and in B (A fixed), so a
    forward difference with any representable step equals the derivative."""
    rng = np.random.default_rng(21 + pool_group)
    M, Din, Dout, r, alpha = 3, 128, 8, 2, 5.0
    W, X, A, B, dY = _problem(rng, M, Din, Dout, r)
    if pool_group > 1:
        A = bf16(rng.standard_normal((Din // pool_group, r)))
    cb = orc.nf4_codebook()
    Wt = orc.dequantize(orc.quantize(W, cb, False), cb)
    dX, dA, dB = orc.backward(X, dY, Wt, A, B, r, alpha, pool_group)
    dyf = f64(dY)

    def loss(X_, A_, B_):
        Y, _ = orc.forward(X_, Wt, A_, B_, r, alpha, pool_group)
        return float(np.sum(dyf * Y))

    L0 = loss(X, A, B)

    def fd(arr, idx, which):
        old = f64(arr[idx])
        new = old + 0.5 if abs(old) < 4 else old * 1.5
        arr2 = arr.copy()
        arr2[idx] = bf16(new)
        h = f64(arr2[idx]) - old
        args = {"X": (arr2, A, B), "A": (X, arr2, B), "B": (X, A, arr2)}[which]
        return (loss(*args) - L0) / h

    for idx in [(0, 0), (2, 77), (1, 127)]:
        assert fd(X, idx, "X") == pytest.approx(dX[idx], rel=1e-9, abs=1e-11)
    for idx in [(0, 0), (A.shape[0] - 1, 1)]:
        assert fd(A, idx, "A") == pytest.approx(dA[idx], rel=1e-9, abs=1e-11)
    for idx in [(0, 0), (1, 7), (0, 5)]:
        assert fd(B, idx, "B") == pytest.approx(dB[idx], rel=1e-9, abs=1e-11)


def test_no_weight_gradient_and_shapes(orc):
    """The backward returns exactly (dX, dA, dB): nothing for the frozen W4."""
    rng = np.random.default_rng(31)
    W, X, A, B, dY = _problem(rng, 2, 64, 4, 1)
    cb = orc.nf4_codebook()
    Wt = orc.dequantize(orc.quantize(W, cb, False), cb)
    out = orc.backward(X, dY, Wt, A, B, 1, 1.0)
    assert len(out) == 3
    assert out[0].shape == (2, 64) and out[1].shape == (64, 1) and out[2].shape == (1, 4)


# ---------------------------------------------------------------- fp16 compute dtype
# The article's section 8.3 lets the layer's arithmetic run in FP16 as well as
# BF16; the oracle's layer functions read either format (fp64 arithmetic).

def test_fp16_decode_exhaustive(orc):
    """Every one of the 65536 binary16 patterns decodes to numpy's value."""
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = orc.fp16_decode(h)
    want = h.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def _both_formats(rng, shape, scale):
    """Values with at most 8 significant bits inside fp16's normal range: the
    same numbers in bf16 and in fp16 bit patterns."""
    mant = rng.integers(128, 256, shape) * rng.choice([-1, 1], shape)
    ex = rng.integers(-14, -6, shape)
    v = (mant * np.exp2(ex - 7.0) * scale).astype(np.float32)
    return v.view(np.uint32).astype(np.uint64) >> 16, v.astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("g", [1, 64])
def test_fp16_layer_equals_bf16_on_shared_values(orc, g):
    """On values both formats hold exactly, the fp16 layer equals the bf16
    layer bit for bit (same fp64 sums in the same order), for every output:
    y, T, dX, dA, dB and the merge; and it matches a float64 matmul."""
    rng = np.random.default_rng(3 + g)
    M, Din, Dout, r, alpha = 5, 128, 72, 8, 16.0
    xb, xh = _both_formats(rng, (M, Din), 1.0)
    wb, wh = _both_formats(rng, (Dout, Din), 1.0)
    ab, ah = _both_formats(rng, (Din // g, r), 1.0)
    bb, bh = _both_formats(rng, (r, Dout), 1.0)
    db, dh = _both_formats(rng, (M, Dout), 1.0)
    xb, wb, ab, bb, db = (a.astype(np.uint16) for a in (xb, wb, ab, bb, db))
    yb, Tb = orc.forward(xb, wb, ab, bb, r, alpha, g)
    yh, Th = orc.forward(xh, wh, ah, bh, r, alpha, g, dtype="fp16")
    assert np.array_equal(yb, yh) and np.array_equal(Tb, Th)
    for fb, fh in zip(orc.backward(xb, db, wb, ab, bb, r, alpha, g),
                      orc.backward(xh, dh, wh, ah, bh, r, alpha, g, dtype="fp16")):
        assert np.array_equal(fb, fh)
    assert np.array_equal(orc.merge(wb, ab, bb, r, alpha, g), orc.merge(wh, ah, bh, r, alpha, g, "fp16"))
    f = lambda h: h.view(np.float16).astype(np.float64)
    u = f(xh) if g == 1 else f(xh).reshape(M, Din // g, g).mean(axis=2)
    ref = f(xh) @ f(wh).T + (alpha / r) * (u @ f(ah)) @ f(bh)
    assert np.allclose(yh, ref, rtol=1e-12, atol=1e-12)


def test_fp16_layer_reads_fp16_values(orc):
    """Values bf16 cannot hold (11 significant bits): the fp16 forward matches
    a float64 matmul of the decoded fp16 inputs, and differs from reading the
    same bits as bf16."""
    rng = np.random.default_rng(9)
    M, Din, Dout, r, alpha = 3, 64, 40, 4, 8.0
    h = lambda shape: rng.standard_normal(shape).astype(np.float16).view(np.uint16)
    x, w, a, b = h((M, Din)), h((Dout, Din)), h((Din, r)), h((r, Dout))
    y, _ = orc.forward(x, w, a, b, r, alpha, dtype="fp16")
    f = lambda v: v.view(np.float16).astype(np.float64)
    ref = f(x) @ f(w).T + (alpha / r) * (f(x) @ f(a)) @ f(b)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    yb, _ = orc.forward(x, w, a, b, r, alpha)
    assert not np.allclose(yb, y)


# ---------------------------------------------------------------- backward over several column chunks

@pytest.mark.parametrize("pool_group", [1, 64])
def test_backward_multichunk(orc, pool_group):
    """Din = 640 and Dout = 2112 run the backward's dX over three input
    chunks (the last one ragged) and dB over three output chunks (ragged), at
    M = 3.  Three facts from the chain rule ("大模型量化从0到1（十）" 12.4) pin
    every entry:

    - finite differences at each chunk's first and last column;
    - Euler's identity: L = sum(dY * y) is linear and homogeneous in x, so
      L = <dX, x> exactly;
    - the adapter part of L is linear and homogeneous in A and in B, so
      L - L(B = 0) = <dA, A> = <dB, B>.

    A wrong chunk bound leaves some entries unwritten or summed twice, which
    breaks one of them."""
    rng = np.random.default_rng(41 + pool_group)
    M, Din, Dout, r, alpha = 3, 640, 2112, 3, 7.0
    W, X, A, B, dY = _problem(rng, M, Din, Dout, r)
    if pool_group > 1:
        A = bf16(rng.standard_normal((Din // pool_group, r)))
    cb = orc.nf4_codebook()
    Wt = orc.dequantize(orc.quantize(W, cb, True), cb)
    dX, dA, dB = orc.backward(X, dY, Wt, A, B, r, alpha, pool_group)
    dyf = f64(dY)

    def loss(X_, A_, B_):
        Y, _ = orc.forward(X_, Wt, A_, B_, r, alpha, pool_group)
        return float(np.sum(dyf * Y))

    L0 = loss(X, A, B)
    L_base = loss(X, A, np.zeros_like(B))
    assert L0 == pytest.approx(float(np.sum(dX * f64(X))), rel=1e-10)
    assert L0 - L_base == pytest.approx(float(np.sum(dB * f64(B))), rel=1e-9)
    assert L0 - L_base == pytest.approx(float(np.sum(dA * f64(A))), rel=1e-9)

    def fd(arr, idx, which):
        old = f64(arr[idx])
        new = old + 0.5 if abs(old) < 4 else old * 1.5
        arr2 = arr.copy()
        arr2[idx] = bf16(new)
        h = f64(arr2[idx]) - old
        args = {"X": (arr2, A, B), "A": (X, arr2, B), "B": (X, A, arr2)}[which]
        return (loss(*args) - L0) / h

    for m, k in [(0, 0), (1, 255), (2, 256), (0, 511), (1, 512), (2, 639)]:
        assert fd(X, (m, k), "X") == pytest.approx(dX[m, k], rel=1e-8, abs=1e-9)
    a_rows = [0, A.shape[0] - 1] + ([63, 64, 600] if pool_group == 1 else [4])
    for k in a_rows:
        assert fd(A, (k, k % r), "A") == pytest.approx(dA[k, k % r], rel=1e-8, abs=1e-9)
    for j, n in [(0, 0), (1, 1023), (2, 1024), (0, 2047), (1, 2048), (2, 2111)]:
        assert fd(B, (j, n), "B") == pytest.approx(dB[j, n], rel=1e-8, abs=1e-9)


@pytest.mark.parametrize("pool_group", [1, 64])
def test_backward_multichunk_B_zero_is_plain_matmul(orc, pool_group):
    """B = 0 at the multi-chunk sizes: dX = dY . dequant(W4) as numpy's matmul
    computes it, dA = 0, and dB = s (u A)^T dY with u = x or pool(x)."""
    rng = np.random.default_rng(51 + pool_group)
    M, Din, Dout, r, alpha = 4, 640, 2112, 2, 6.0
    W, X, A, B, dY = _problem(rng, M, Din, Dout, r)
    if pool_group > 1:
        A = bf16(rng.standard_normal((Din // pool_group, r)))
    B[:] = 0
    cb = orc.nf4_codebook()
    Wt = orc.dequantize(orc.quantize(W, cb, False), cb)
    dX, dA, dB = orc.backward(X, dY, Wt, A, B, r, alpha, pool_group)
    np.testing.assert_allclose(dX, f64(dY) @ f64(Wt), rtol=1e-12, atol=1e-12)
    assert np.all(dA == 0)
    u = f64(X) if pool_group == 1 else f64(X).reshape(M, -1, pool_group).mean(axis=2)
    np.testing.assert_allclose(dB, (alpha / r) * (u @ f64(A)).T @ f64(dY), rtol=1e-12, atol=1e-12)
