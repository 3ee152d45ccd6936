"""The NF4 codebook handed to the library (a 16-entry fp32 host table).

Levels are standard-normal quantiles of equal-probability pieces of the CDF,
normalised to [-1, 1], with 8 positive levels, 7 negative levels and an
exact 0 ("QLoRA：用4比特行李箱装下整个大模型" chapter 3; bitsandbytes article (CSDN)
section 6.2).  Probabilities run evenly from the tail probability ``delta``
to 1/2 (9 points on the positive side, 8 on the negative side, the 1/2 point
of each side being the shared zero); every quantile is divided by
Phi^-1(delta) so the extremes are exactly -1 and +1.
"""
from __future__ import annotations

import torch

# mean of the outermost interval-midpoint probabilities for 16 and 15 pieces
DEFAULT_DELTA = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


def nf4_codebook(delta: float = DEFAULT_DELTA) -> torch.Tensor:
    """fp32 CPU tensor of the 16 sorted levels."""
    d = torch.tensor(delta, dtype=torch.float64)
    z = torch.special.ndtri(d)
    pos = delta + (0.5 - delta) * torch.arange(8, dtype=torch.float64) / 8.0
    neg = delta + (0.5 - delta) * torch.arange(7, dtype=torch.float64) / 7.0
    v = torch.cat([torch.special.ndtri(pos) / z, -torch.special.ndtri(neg) / z,
                   torch.zeros(1, dtype=torch.float64)])
    v, _ = torch.sort(v)
    return v.to(torch.float32).contiguous()
