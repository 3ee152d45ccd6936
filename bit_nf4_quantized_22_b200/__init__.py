"""QLoRA linear layer on B200 (sm_100a): NF4 + double quantization + LoRA.

The compute lives in libqlora.so (CUDA kernels behind a C ABI,
include/qlora.h); this package is its thin Python binding.
"""
from ._lib import QLoRAError, EXPORTS, STATUS_NONFINITE, STATUS_TIMEOUT  # noqa: F401
from .api import (NF4Weight, QLoRALinearFn, backward, check_codebook, dequantize,  # noqa: F401
                  forward, forward_noalloc, load, quantize, workspace_size, merge)
from .codebook import DEFAULT_DELTA, fp4_codebook, nf4_codebook  # noqa: F401
