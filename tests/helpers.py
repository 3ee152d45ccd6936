"""Shared helpers for the GPU parity tests."""
import numpy as np
import torch

from bit_nf4_quantized_22_b200 import synth

# Tolerance for floating-point outputs (y, dX, dA, dB) against the fp64
# oracle: relative Frobenius error <= 5e-3 and |err| <= 2e-2 (|ref| + 1)
# per element.
REL_FRO = 5e-3
ELEM = 2e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def host_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return synth.bf16_to_f32(host_bits(t)).astype(np.float64)
    return t.detach().cpu().numpy().astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    denom = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / denom if denom > 0 else np.linalg.norm(got - ref)
    worst = np.max(err - ELEM * (np.abs(ref) + 1)) if err.size else -1
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert worst <= 0, f"{what}: element error exceeds {ELEM}(|ref|+1) by {worst:.3e}"
    return rel


def unpack(packed: np.ndarray) -> np.ndarray:
    out = np.empty(packed.size * 2, dtype=np.int64)
    out[0::2] = packed >> 4
    out[1::2] = packed & 15
    return out
