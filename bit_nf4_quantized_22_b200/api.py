"""Python binding of the QLoRA layer library.

Argument marshalling only: every function hands device pointers, sizes and
the current CUDA stream to the C ABI (include/qlora.h) and every step of the
computation runs in the library's CUDA kernels.  PyTorch provides device
memory (tensors, the workspace) and streams.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from .codebook import nf4_codebook

BLOCK = 64
DQ_GROUP = 256
# double-quantization codes of the block scales (QLORA_DQ_* in qlora.h)
DQ_VARIANTS = {"u8": 1, "s8": 2, "mean": 3, "f8": 4}


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _cb_host(codebook: torch.Tensor | None) -> ctypes.Array:
    cb = nf4_codebook() if codebook is None else codebook.detach().to("cpu", torch.float32)
    arr = (ctypes.c_float * 16)(*cb.tolist())
    return arr


def _need(t: torch.Tensor, dtype, name: str, dims: int):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.dim() != dims:
        raise TypeError(f"{name}: expected a {dims}-D {dtype} tensor")
    if not t.is_cuda:
        raise TypeError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise TypeError(f"{name}: must be contiguous")


@dataclass
class NF4Weight:
    """A quantized frozen weight Wt:[rows = Dout, cols = Din] (device buffers)."""
    rows: int
    cols: int
    double_quant: bool
    packed: torch.Tensor                   # uint8 [rows*cols/2]
    absmax: torch.Tensor | None = None     # fp32 [nb]
    codes: torch.Tensor | None = None      # uint8 [nb] (int8 two's complement for "mean")
    steps: torch.Tensor | None = None      # fp32 [ceil(nb/256)]
    block: int = BLOCK                     # weights per first-level scale (32, 64, 128, 256)
    dq_variant: str = "u8"                 # code of the scales: "u8", "s8", "mean" or "f8"
    means: torch.Tensor | None = None      # fp32 [ceil(nb/256)] group means ("mean")
    # the layer calls' 16-bit dtype (x, A, B, dY, y, dX, merged weight)
    compute_dtype: torch.dtype = torch.bfloat16

    @staticmethod
    def empty(rows: int, cols: int, double_quant: bool, device="cuda", block: int = BLOCK,
              dq_variant: str = "u8") -> "NF4Weight":
        nb = rows * cols // block
        packed = torch.empty(rows * cols // 2, dtype=torch.uint8, device=device)
        if double_quant:
            if dq_variant not in DQ_VARIANTS:
                raise ValueError(f"dq_variant: one of {sorted(DQ_VARIANTS)}")
            ng = (nb + DQ_GROUP - 1) // DQ_GROUP
            means = torch.empty(ng, dtype=torch.float32, device=device) if dq_variant == "mean" else None
            return NF4Weight(rows, cols, True, packed,
                             codes=torch.empty(nb, dtype=torch.uint8, device=device),
                             steps=torch.empty(ng, dtype=torch.float32, device=device), block=block,
                             dq_variant=dq_variant, means=means)
        return NF4Weight(rows, cols, False, packed,
                         absmax=torch.empty(nb, dtype=torch.float32, device=device), block=block)

    def c_struct(self) -> _lib.NF4WeightC:
        return _lib.NF4WeightC(
            self.rows, self.cols, self.block,
            DQ_VARIANTS[self.dq_variant] if self.double_quant else 0, DQ_GROUP,
            _DTYPE_CODES[self.compute_dtype],
            self.packed.data_ptr(),
            self.absmax.data_ptr() if self.absmax is not None else None,
            self.codes.data_ptr() if self.codes is not None else None,
            self.steps.data_ptr() if self.steps is not None else None,
            self.means.data_ptr() if self.means is not None else None)

    @property
    def nbytes(self) -> int:
        n = self.packed.numel()
        for t in (self.absmax, self.codes, self.steps, self.means):
            if t is not None:
                n += t.numel() * t.element_size()
        return n


def load():
    """Load libqlora.so; raises if it is missing (no fallback exists)."""
    return _lib.load()


def check_codebook(codebook: torch.Tensor) -> int:
    return load().qlora_check_codebook(_cb_host(codebook))


def quantize(W: torch.Tensor, double_quant: bool = True, codebook: torch.Tensor | None = None,
             status: torch.Tensor | None = None, out: NF4Weight | None = None,
             block: int = BLOCK, dq_variant: str = "u8",
             compute_dtype: torch.dtype = torch.bfloat16) -> NF4Weight:
    """nf4_quantize on W (fp32 [Dout, Din], CUDA) in blocks of `block` weights
    (32, 64, 128 or 256; the layer calls need 64); with double quantization
    the block scales take the `dq_variant` code ("u8", "s8", "mean" or "f8").
    `compute_dtype` (bf16 or fp16) is the dtype the layer calls then use."""
    _need(W, torch.float32, "W", 2)
    if compute_dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("compute_dtype: torch.bfloat16 or torch.float16")
    rows, cols = W.shape
    q = out if out is not None else NF4Weight.empty(rows, cols, double_quant, W.device, block,
                                                    dq_variant)
    if out is None:
        q.compute_dtype = compute_dtype
    qc = q.c_struct()
    rc = load().nf4_quantize(_ptr(W), ctypes.byref(qc), _cb_host(codebook), _ptr(status), _stream())
    _lib.check(rc, "nf4_quantize")
    return q


_DTYPE_CODES = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}


def dequantize(q: NF4Weight, codebook: torch.Tensor | None = None,
               out: torch.Tensor | None = None, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """The dequantized weight [rows, cols] in the compute dtype (bf16, fp16 or fp32)."""
    if dtype not in _DTYPE_CODES:
        raise TypeError(f"dtype: one of {list(_DTYPE_CODES)}")
    out = out if out is not None else torch.empty(q.rows, q.cols, dtype=dtype,
                                                  device=q.packed.device)
    if out.dtype != dtype:
        raise TypeError("out: dtype does not match")
    qc = q.c_struct()
    if dtype == torch.bfloat16:
        rc = load().nf4_dequantize(ctypes.byref(qc), _cb_host(codebook), _ptr(out), _stream())
    else:
        rc = load().nf4_dequantize_dtype(ctypes.byref(qc), _cb_host(codebook), _DTYPE_CODES[dtype],
                                         _ptr(out), _stream())
    _lib.check(rc, "nf4_dequantize")
    return out


def merge(q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float, pool_group: int = 1,
          codebook: torch.Tensor | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 [Dout, Din] weight with the adapter folded in (qlora_merge)."""
    r = B.shape[0]
    out = out if out is not None else torch.empty(q.rows, q.cols, dtype=q.compute_dtype,
                                                  device=q.packed.device)
    qc = q.c_struct()
    rc = load().qlora_merge(ctypes.byref(qc), _cb_host(codebook), _ptr(A), _ptr(B), r,
                            float(alpha), pool_group, _ptr(out), _stream())
    _lib.check(rc, "qlora_merge")
    return out


def workspace_size(M: int, q: NF4Weight, r: int, pool_group: int = 1, which: int = 0) -> int:
    qc = q.c_struct()
    return int(load().qlora_workspace_size(M, ctypes.byref(qc), r, pool_group, which))


def _workspace(nbytes: int, device, ws: torch.Tensor | None):
    if nbytes == 0:
        return None, 0
    if ws is not None and ws.numel() >= nbytes:
        return ws, ws.numel()
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


def forward(x: torch.Tensor, q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
            pool_group: int = 1, codebook: torch.Tensor | None = None, save_T: bool = True,
            workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
            out: torch.Tensor | None = None):
    """y = x dequant(W4) + (alpha/r) (u A) B.  Returns (y bf16 [M, Dout], T fp32 [M, r] or None)."""
    _need(x, q.compute_dtype, "x", 2)
    _need(A, q.compute_dtype, "A", 2)
    _need(B, q.compute_dtype, "B", 2)
    M = x.shape[0]
    r = A.shape[1]
    y = out if out is not None else torch.empty(M, q.rows, dtype=q.compute_dtype, device=x.device)
    T = torch.empty(M, r, dtype=torch.float32, device=x.device) if save_T else None
    ws, nbytes = _workspace(workspace_size(M, q, r, pool_group, 0), x.device, workspace)
    qc = q.c_struct()
    rc = load().qlora_forward(_ptr(x), M, ctypes.byref(qc), _cb_host(codebook), _ptr(A), _ptr(B),
                              r, float(alpha), pool_group, _ptr(y), _ptr(T), _ptr(ws), nbytes,
                              _ptr(status), _stream())
    _lib.check(rc, "qlora_forward")
    return y, T


def backward(x: torch.Tensor | None, dy: torch.Tensor, q: NF4Weight, A: torch.Tensor,
             B: torch.Tensor, alpha: float, pool_group: int = 1, T: torch.Tensor | None = None,
             need_dx: bool = True, need_dA: bool = True, need_dB: bool = True,
             codebook: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
             status: torch.Tensor | None = None):
    """Returns (dX bf16 [M, Din] | None, dA fp32 | None, dB fp32 | None); W4 gets none."""
    _need(dy, q.compute_dtype, "dy", 2)
    _need(A, q.compute_dtype, "A", 2)
    _need(B, q.compute_dtype, "B", 2)
    M = dy.shape[0]
    r = A.shape[1]
    dev = dy.device
    dX = torch.empty(M, q.cols, dtype=q.compute_dtype, device=dev) if need_dx else None
    dA = torch.empty(A.shape[0], r, dtype=torch.float32, device=dev) if need_dA else None
    dB = torch.empty(r, q.rows, dtype=torch.float32, device=dev) if need_dB else None
    ws, nbytes = _workspace(workspace_size(M, q, r, pool_group, 1), dev, workspace)
    qc = q.c_struct()
    rc = load().qlora_backward(_ptr(x), _ptr(dy), M, ctypes.byref(qc), _cb_host(codebook),
                               _ptr(A), _ptr(B), r, float(alpha), pool_group, _ptr(T), _ptr(dX),
                               _ptr(dA), _ptr(dB), _ptr(ws), nbytes, _ptr(status), _stream())
    _lib.check(rc, "qlora_backward")
    return dX, dA, dB


def forward_noalloc(x: torch.Tensor, q: NF4Weight, A: torch.Tensor, B: torch.Tensor,
                    alpha: float, pool_group: int = 1, codebook: torch.Tensor | None = None,
                    out: torch.Tensor | None = None, T_out: torch.Tensor | None = None,
                    status: torch.Tensor | None = None):
    """qlora_forward_noalloc: the forward with the library's built-in scratch
    array instead of a workspace.  The caller passes the outputs (`out`,
    `T_out`); when omitted they are created here, which allocates."""
    _need(x, q.compute_dtype, "x", 2)
    _need(A, q.compute_dtype, "A", 2)
    _need(B, q.compute_dtype, "B", 2)
    M, r = x.shape[0], A.shape[1]
    y = out if out is not None else torch.empty(M, q.rows, dtype=q.compute_dtype, device=x.device)
    qc = q.c_struct()
    rc = load().qlora_forward_noalloc(_ptr(x), M, ctypes.byref(qc), _cb_host(codebook), _ptr(A),
                                      _ptr(B), r, float(alpha), pool_group, _ptr(y), _ptr(T_out),
                                      _ptr(status), _stream())
    _lib.check(rc, "qlora_forward_noalloc")
    return y, T_out


class QLoRALinearFn(torch.autograd.Function):
    """Autograd wrapper: gradients for x, A and B; none for the frozen W4."""

    @staticmethod
    def forward(ctx, x, A, B, q: NF4Weight, alpha: float, pool_group: int):
        y, T = forward(x, q, A, B, alpha, pool_group)
        ctx.save_for_backward(x, A, B, T)
        ctx.q, ctx.alpha, ctx.pool = q, alpha, pool_group
        return y

    @staticmethod
    def backward(ctx, dy):
        x, A, B, T = ctx.saved_tensors
        dX, dA, dB = backward(x, dy.contiguous(), ctx.q, A, B, ctx.alpha, ctx.pool, T=T,
                              need_dx=ctx.needs_input_grad[0], need_dA=ctx.needs_input_grad[1],
                              need_dB=ctx.needs_input_grad[2])
        return (dX, None if dA is None else dA.to(A.dtype), None if dB is None else dB.to(B.dtype),
                None, None, None)
