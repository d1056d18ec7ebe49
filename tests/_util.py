"""Small helpers shared by the GPU tests (conversions only, no method arithmetic)."""
import numpy as np
import torch


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits_of(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> its uint16 bit patterns."""
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def rand_bf16(shape, scale=1.0, seed=0, device="cuda"):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).to(device)


def zeros_err(device="cuda"):
    return torch.zeros(1, dtype=torch.int32, device=device)
