"""Failure detection on the GPU without a fault: a bounded pipeline wait that
can never complete gives up, reports QLORA_STATUS_TIMEOUT in the status word,
and leaves the context usable (a normal quantize runs bit-exact right after)."""
import ctypes
import time

import numpy as np
import pytest
import torch

from bit_nf4_quantized_22_b200._lib import QLORA_EINVAL, QLORA_OK, STATUS_TIMEOUT

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(orc, qlib):
    lib = qlib.load()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    t0 = time.time()
    assert lib.qlora_selftest_wait_timeout(ctypes.c_void_p(status.data_ptr()), stream) == QLORA_OK
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert int(status.item()) & STATUS_TIMEOUT
    assert elapsed < 30.0
    # the context still works: a quantize right after is bit-exact
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((64, 256)) * 0.05).astype(np.float32)
    w = qlib.quantize(torch.from_numpy(W).cuda(), double_quant=True)
    torch.cuda.synchronize()
    ref = orc.quantize(W, orc.nf4_codebook(), True)
    assert np.array_equal(w.packed.cpu().numpy(), ref.packed)


def test_selftest_rejects_null_status(qlib):
    lib = qlib.load()
    assert lib.qlora_selftest_wait_timeout(None, None) == QLORA_EINVAL
