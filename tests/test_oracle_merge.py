"""Pins for the oracle's adapter merge, W_eff = dequant(W4) + (alpha/r) A B
("从 LoRA 到 QLoRA、QA-LoRA" section 2; bitsandbytes article (CSDN) 12.10,
merging the adapter into the weight for deployment), stored [Dout, Din].
The pooled form shares (A_p B)/g across a group's inputs (same blog,
section 5)."""
import numpy as np

from conftest import floats, read_golden
from test_oracle_layer import bf16, f64


def test_merge_worked_lora_example(orc):
    """Zero base: the merged weight is the printed dW (transposed to the
    stored orientation), up to the bf16 rounding of B."""
    g = read_golden("lora_worked_example.txt")
    Din, Dout, r = int(g["Din"]), int(g["Dout"]), int(g["r"])
    A = bf16(np.array(floats(g["A"])).reshape(Din, r))
    B = bf16(np.array(floats(g["B"])).reshape(r, Dout))
    dW = np.array(floats(g["dW"])).reshape(Din, Dout)
    W = orc.merge(np.zeros((Dout, Din), np.uint16), A, B, r, alpha=r)
    np.testing.assert_array_equal(W, (f64(A) @ f64(B)).T)
    np.testing.assert_allclose(W, dW.T, rtol=2 ** -8, atol=0)


def test_merge_pooled_group_updates(orc):
    """Din=4 in groups of 2: inputs 0-1 get group1_update, 2-3 group2_update."""
    g = read_golden("pooled_adapter_example.txt")
    gs = int(g["group_size"])
    A = bf16(np.array(floats(g["A"])).reshape(-1, 1))
    B = bf16(np.array(floats(g["B"])).reshape(1, -1))
    Din, Dout = int(g["Din"]), int(g["Dout"])
    W = orc.merge(np.zeros((Dout, Din), np.uint16), A, B, 1, alpha=1, pool_group=gs)
    u1, u2 = np.array(floats(g["group1_update"])), np.array(floats(g["group2_update"]))
    expect = np.stack([u1, u1, u2, u2]).T                  # [Dout, Din]
    np.testing.assert_allclose(W, expect, rtol=2 ** -7, atol=0)


def test_merge_adds_to_base_and_scales(orc):
    """B = 0 returns the base exactly; the adapter term scales as alpha/r."""
    rng = np.random.default_rng(3)
    Dout, Din, r = 6, 128, 3
    Wt = bf16(rng.standard_normal((Dout, Din)))
    A = bf16(rng.standard_normal((Din, r)))
    B = bf16(rng.standard_normal((r, Dout)))
    np.testing.assert_array_equal(orc.merge(Wt, A, np.zeros_like(B), r, 5.0), f64(Wt))
    d1 = orc.merge(Wt, A, B, r, 1.0) - f64(Wt)
    d4 = orc.merge(Wt, A, B, r, 4.0) - f64(Wt)
    np.testing.assert_allclose(d4, 4 * d1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(d1, (f64(A) @ f64(B)).T / r, rtol=1e-12, atol=1e-12)


def test_merged_weight_reproduces_the_forward(orc):
    """x W_eff^T equals the layer forward, plain and pooled (the merge's
    purpose: the adapter folded into the weight)."""
    rng = np.random.default_rng(4)
    M, Din, Dout, r = 3, 128, 8, 2
    X = bf16(rng.standard_normal((M, Din)))
    Wt = bf16(rng.standard_normal((Dout, Din)) * 0.1)
    B = bf16(rng.standard_normal((r, Dout)))
    for g in (1, 64):
        A = bf16(rng.standard_normal((Din // g, r)))
        y, _ = orc.forward(X, Wt, A, B, r, 3.0, pool_group=g)
        W = orc.merge(Wt, A, B, r, 3.0, pool_group=g)
        np.testing.assert_allclose(f64(X) @ W.T, y, rtol=1e-12, atol=1e-12)
