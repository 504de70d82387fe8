"""Conversion helper for the oracle: any CPU tensor or array to a float64 numpy array."""

from __future__ import annotations

import numpy as np


def f64(x) -> np.ndarray:
    """Widen ``x`` (numpy array, torch tensor of any float dtype incl. bf16, or nested list)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover - torch is always present in this image
        pass
    return np.asarray(x, dtype=np.float64)
