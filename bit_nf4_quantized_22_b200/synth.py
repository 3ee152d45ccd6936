"""Seeded synthetic inputs for the layer (weights, activations, adapters,
upstream gradients).  Used alike by the tests, the benchmark and the smoke
check; it holds none of the layer's arithmetic.

Generator: numpy PCG64 seeded with 20261202 + 1000*config + 10*linear + tensor
(tensor ids: W=0, x=1, A=2, B=3, dY=4).  Values are drawn in fp32; bf16
tensors are the round-to-nearest-even bf16 of those draws, returned as uint16
bit patterns (numpy has no bf16).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BASE_SEED = 20261202
TID = {"W": 0, "x": 1, "A": 2, "B": 3, "dY": 4}


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng(config: int, linear: int, tensor: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(BASE_SEED + 1000 * config + 10 * linear + TID[tensor]))


@dataclass
class LinearSpec:
    """One QLoRA linear of a workload."""
    name: str
    Din: int
    Dout: int
    r: int
    alpha: float
    double_quant: bool
    w_dist: str = "normal"      # "normal" or "t5"
    w_scale: float = 0.02
    pool_group: int = 1


def fp16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> IEEE binary16 bit patterns, round to nearest even."""
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def draw(spec: LinearSpec, M: int, config: int, linear: int = 0, which=("W", "x", "A", "B", "dY"),
         fmt: str = "bf16"):
    """Arrays for one linear: W fp32 [Dout, Din]; x [M, Din], A [Din/g, r],
    B [r, Dout], dY [M, Dout] as 16-bit patterns of `fmt` ("bf16" or "fp16",
    the layer's compute dtype), rounded from the same fp32 draws."""
    bf16_bits = globals()["bf16_bits"] if fmt == "bf16" else fp16_bits
    out = {}
    if "W" in which:
        g = rng(config, linear, "W")
        if spec.w_dist == "t5":
            w = g.standard_t(5, size=(spec.Dout, spec.Din)).astype(np.float32)
        else:
            w = g.standard_normal(size=(spec.Dout, spec.Din), dtype=np.float32)
        out["W"] = (w * np.float32(spec.w_scale)).astype(np.float32)
    if "x" in which:
        out["x"] = bf16_bits(rng(config, linear, "x").standard_normal((M, spec.Din), dtype=np.float32))
    if "A" in which:
        a = rng(config, linear, "A").standard_normal((spec.Din // spec.pool_group, spec.r), dtype=np.float32)
        out["A"] = bf16_bits(a * np.float32(1.0 / np.sqrt(spec.r)))
    if "B" in which:
        b = rng(config, linear, "B").standard_normal((spec.r, spec.Dout), dtype=np.float32)
        out["B"] = bf16_bits(b * np.float32(0.01))
    if "dY" in which:
        out["dY"] = bf16_bits(rng(config, linear, "dY").standard_normal((M, spec.Dout), dtype=np.float32))
    return out


# The five workloads: shapes, distributions and adapter settings.
CONFIGS = {
    1: dict(name="single linear 256x256, M=16, no double quant",
            linears=[LinearSpec("linear", 256, 256, 8, 16.0, False)], M=[16], passes="fwd+bwd"),
    2: dict(name="decode-shaped 7B projection 4096x4096, M in {1,16}",
            linears=[LinearSpec("proj", 4096, 4096, 16, 32.0, True)], M=[1, 16], passes="fwd"),
    3: dict(name="training-shaped 7B up-projection 4096->11008, M=4096",
            linears=[LinearSpec("up", 4096, 11008, 64, 128.0, True, "t5")], M=[4096],
            passes="fwd+bwd"),
    4: dict(name="7B decoder layer, 7 linears, M=2048",
            linears=[LinearSpec(n, di, do, 16, 32.0, True) for n, di, do in (
                ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                ("gate", 4096, 11008), ("up", 4096, 11008), ("down", 11008, 4096))],
            M=[2048], passes="quantize+fwd+bwd"),
    5: dict(name="70B MLP linears 8192<->28672, M in {1,16,8192}, + pooled adapter",
            linears=[LinearSpec("up", 8192, 28672, 64, 16.0, True, w_scale=0.015),
                     LinearSpec("down", 28672, 8192, 64, 16.0, True, w_scale=0.015),
                     LinearSpec("up_pooled", 8192, 28672, 64, 16.0, True, w_scale=0.015,
                                pool_group=64)],
            M=[1, 16, 8192], passes="fwd+bwd"),
}
