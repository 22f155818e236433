"""Small helpers shared by the tests: torch bf16 tensors -> float64 numpy (exact)."""
import numpy as np
import torch


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy()
