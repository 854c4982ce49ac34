"""Helpers shared by the GPU parity tests."""
import numpy as np
import torch

from sparse_long_context_04_b200 import build as _build
from sparse_long_context_04_b200 import dsa as D


def ensure_lib():
    _build.build()
    D.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def indexer_close(gpu: np.ndarray, ref: np.ndarray, rel=1e-2, abs_=1e-3):
    """|g - o| <= abs + rel*|o| elementwise (the indexer tolerance)."""
    err = np.abs(gpu.astype(np.float64) - ref)
    bad = err > abs_ + rel * np.abs(ref)
    return not bad.any(), float(err.max()) if err.size else 0.0, int(bad.sum())
