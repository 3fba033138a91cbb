"""Shared helpers of the GPU parity tests: moving bf16 bit patterns to and
from the device, and the floating-point acceptance rule.

Acceptance for GEMM outputs (bf16 in, fp32 accumulate): per element
|y - y_ref| <= 2^-7 * sum_k |w'_rk| |x_kt|, and relative Frobenius error
||Y - Y_ref||_F / ||Y_ref||_F <= 5e-3.  Values, metadata and index maps are
compared bit for bit.
"""
import numpy as np
import torch

import workloads as wl

DEV = "cuda:0"
ELEM_TOL = 2.0 ** -7
FROB_TOL = 5e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> a torch.bfloat16 CUDA tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def to_dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).astype(np.int32)).to(DEV)


def to_dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).astype(np.uint8)).to(DEV)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> uint16 bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def words(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy().view(np.uint32)


def values_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return wl.bf16_to_f32(bits(t)).astype(np.float64)
    return t.float().cpu().numpy().astype(np.float64)


def assert_gemm_close(y_gpu: np.ndarray, y_ref: np.ndarray, y_abs: np.ndarray, what: str = ""):
    err = np.abs(y_gpu - y_ref)
    bound = ELEM_TOL * y_abs
    bad = err > bound
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} elements over 2^-7*sum|w||x|; worst excess "
        f"{float((err - bound).max()):.3e} at {np.unravel_index(np.argmax(err - bound), err.shape)}")
    ref_norm = np.linalg.norm(y_ref)
    if ref_norm > 0:
        rel = np.linalg.norm(y_gpu - y_ref) / ref_norm
        assert rel <= FROB_TOL, f"{what}: relative Frobenius error {rel:.3e}"


def bf16_rne_of(y: np.ndarray) -> np.ndarray:
    """bf16 bits of exactly representable float32 values (integer tests)."""
    return wl.bf16_bits(y.astype(np.float32))
