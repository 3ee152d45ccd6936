"""qlora_forward_noalloc checked against qlora_forward.

qlora_forward_noalloc is the forward pass for callers that cannot allocate
device memory: code that runs where cudaMalloc is not allowed or not wanted
(inside another allocator's arena, in a service that must not grow its
device footprint after start-up) and so has no workspace to pass.  It runs
the same kernels as qlora_forward with the library's fixed scratch array in
place of the caller's workspace.

Each case calls the new entry point through the C ABI twice in a row (the
second call starts from whatever the first left in the shared scratch) and
compares both results with qlora_forward's, within the parity tolerance the
other tests use.  A request larger than the array must be refused before
anything is enqueued.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import assert_close, dev_bf16, host_f64
from bit_nf4_quantized_22_b200 import synth
from bit_nf4_quantized_22_b200._lib import QLORA_EWORKSPACE, QLORA_OK
from bit_nf4_quantized_22_b200.synth import LinearSpec

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, q, x, w, A, B, r, alpha, pool, y, T):
    cb = (ctypes.c_float * 16)(*q.nf4_codebook().tolist())
    wc = w.c_struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.qlora_forward_noalloc(_ptr(x), x.shape[0], ctypes.byref(wc), cb, _ptr(A), _ptr(B),
                                     r, float(alpha), pool, _ptr(y), _ptr(T), None, stream)


@pytest.mark.parametrize("M,Din,Dout,r,dq,pool", [
    (1, 4096, 4096, 16, True, 1),      # decode, GEMV path
    (16, 4096, 4096, 16, True, 1),
    (5, 512, 136, 8, False, 64),       # pooled adapter
    (64, 512, 264, 8, True, 1),        # tensor-core path
])
def test_noalloc_matches_forward(qlib, M, Din, Dout, r, dq, pool):
    lib = qlib.load()
    spec = LinearSpec("na", Din, Dout, r, 2.0 * r, dq, pool_group=pool)
    a = synth.draw(spec, M, 21, Din + M)
    w = qlib.quantize(torch.from_numpy(a["W"]).cuda(), double_quant=dq)
    x, A, B = dev_bf16(a["x"]), dev_bf16(a["A"]), dev_bf16(a["B"])
    y_ref, T_ref = qlib.forward(x, w, A, B, spec.alpha, pool)
    torch.cuda.synchronize()
    ys = [torch.full((M, Dout), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    Ts = [torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
    free = []
    for y, T in zip(ys, Ts):
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        assert _noalloc(lib, qlib, x, w, A, B, r, spec.alpha, pool, y, T) == QLORA_OK
        torch.cuda.synchronize()
        assert_close(host_f64(y), host_f64(y_ref), "y (no-alloc vs workspace forward)")
        assert_close(host_f64(T), host_f64(T_ref), "T (no-alloc vs workspace forward)")
    # the second call finds the kernels loaded and allocates nothing: the
    # device's free memory is the same before and after it
    assert torch.cuda.mem_get_info()[0] == free[1]


def test_noalloc_refuses_oversize_request(qlib):
    """M = 8192 on the 8192 -> 28672 projection needs far more scratch than
    the fixed array holds: refused, output untouched."""
    lib = qlib.load()
    M, Din, Dout, r = 8192, 8192, 28672, 64
    w = qlib.NF4Weight.empty(Dout, Din, True)
    x = torch.zeros(M, Din, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(Din, r, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(r, Dout, dtype=torch.bfloat16, device="cuda")
    y = torch.full((M, Dout), 7.0, dtype=torch.bfloat16, device="cuda")
    assert qlib.workspace_size(M, w, r, 1, 0) > (8 << 20)
    assert _noalloc(lib, qlib, x, w, A, B, r, 16.0, 1, y, None) == QLORA_EWORKSPACE
    torch.cuda.synchronize()
    assert bool(torch.all(y == 7.0))


def test_noalloc_decode_limits(qlib):
    """The stated limits: on the 8192 -> 28672 projection (r = 64) M = 1 fits
    the fixed array and M = 16 does not (refused, output untouched)."""
    lib = qlib.load()
    Din, Dout, r = 8192, 28672, 64
    w = qlib.NF4Weight.empty(Dout, Din, True)
    A = torch.zeros(Din, r, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(r, Dout, dtype=torch.bfloat16, device="cuda")
    assert qlib.workspace_size(1, w, r, 1, 0) <= (8 << 20)
    assert qlib.workspace_size(16, w, r, 1, 0) > (8 << 20)
    x = torch.zeros(16, Din, dtype=torch.bfloat16, device="cuda")
    y = torch.full((16, Dout), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, qlib, x, w, A, B, r, 16.0, 1, y, None) == QLORA_EWORKSPACE
    torch.cuda.synchronize()
    assert bool(torch.all(y == 7.0))
