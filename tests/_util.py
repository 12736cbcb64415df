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
