"""Helpers of the GPU tests: moving bf16 bit patterns between numpy and the device."""
import numpy as np
import pytest
import torch

from kv_cache_serving_ws_b200 import native as ws


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    ws.lib()   # raises when libws.so is missing: no fallback


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).cpu().numpy()


# Attention tolerance on bf16 N(0,1) inputs (max |err|, mean |err|), as fixed for this path.
ATOL_MAX = 1e-2
ATOL_MEAN = 1e-3
