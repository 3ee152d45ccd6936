"""The codebooks handed to the library (16-entry fp32 host tables).

The NF4 table is built by the library's ``nf4_codebook`` ("QLoRA：用4比特行李箱装下整个大模型"
chapter 3; bitsandbytes article (CSDN) section 6.2), the FP4 table by its
``fp4_codebook`` (sections 6.4-6.5: a 4-bit float-style layout, read as E2M1
divided by 6); this module only calls them.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import check, load

# mean of the outermost interval-midpoint probabilities for 16 and 15 pieces
# (QLORA_NF4_DELTA in include/qlora.h)
DEFAULT_DELTA = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


def nf4_codebook(delta: float = DEFAULT_DELTA) -> torch.Tensor:
    """fp32 CPU tensor of the 16 sorted levels."""
    out = (ctypes.c_float * 16)()
    check(load().nf4_codebook(float(delta), out), "nf4_codebook")
    return torch.tensor(list(out), dtype=torch.float32)


def fp4_codebook() -> torch.Tensor:
    """fp32 CPU tensor of the 16 FP4 levels (ascending, -0 before +0)."""
    out = (ctypes.c_float * 16)()
    check(load().fp4_codebook(out), "fp4_codebook")
    return torch.tensor(list(out), dtype=torch.float32)
