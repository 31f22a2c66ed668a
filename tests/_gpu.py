"""Device-side helpers for the GPU tests (marshalling numpy inputs to torch)."""
import numpy as np
import torch


def to_dev(x: np.ndarray) -> torch.Tensor:
    """uint16 arrays are bf16 bit patterns; float32 arrays stay fp32."""
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
