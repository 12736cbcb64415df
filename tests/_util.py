"""Helpers shared by the GPU parity tests: moving bit patterns between numpy and torch."""
import numpy as np
import torch


def to_dev_bits(a: np.ndarray, dtype=torch.bfloat16, device="cuda") -> torch.Tensor:
    """uint16 numpy bit patterns -> a torch tensor of `dtype` (bf16/fp16) on the device."""
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(dtype).to(device)


def bits(t: torch.Tensor) -> np.ndarray:
    """A 16-bit torch tensor -> its uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |v| (0 at v = 0): the largest error that the
    round-to-nearest conversion of an exact result to a bf16 output can add."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.ldexp(1.0, (e - 8).astype(np.int64)), 0.0)


def matmul_tolerance(y_ref: np.ndarray, bound: np.ndarray, tol: float = 2e-3) -> np.ndarray:
    """Per-element tolerance of a bf16 W4A16 product: tol * sum_k |Wdeq| |x| for the fp32
    arithmetic, plus half a bf16 ulp of the result for rounding it to the bf16 output (bf16
    keeps 8 significant bits, so that half ulp alone can reach 2^-8 relative)."""
    return tol * bound + bf16_half_ulp(y_ref)
