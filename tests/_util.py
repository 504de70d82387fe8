"""Helpers shared by the GPU parity tests (comparison metrics only)."""

import numpy as np
import torch


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def rel_err(got, ref) -> float:
    """max |got − ref| / max |ref| (the workloads' tolerance metric)."""
    g, r = to_np(got), to_np(ref)
    denom = np.max(np.abs(r))
    return float(np.max(np.abs(g - r)) / (denom if denom > 0 else 1.0))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (RNE) and back, through torch."""
    return torch.from_numpy(np.asarray(x, np.float64)).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
