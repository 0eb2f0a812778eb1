"""Shared helpers for the tests: tensor <-> numpy marshalling and error metrics."""
import numpy as np
import torch


def to_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> contiguous uint16 numpy array of its bit patterns."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def err_stats(got: np.ndarray, want: np.ndarray):
    e = np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))
    return float(e.max()), float(e.mean())


# Tolerances stated for the outputs of bf16 inputs with fp32 accumulation, and for the
# rotated q/k as the kernels computed them (fp32, before any rounding).
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
ROT_ABS = 1e-3
