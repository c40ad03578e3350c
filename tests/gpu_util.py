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
# Stressed scores (queries scaled x4, rising key scales): the weights concentrate on a few
# keys, whose P carry bf16 rounding (2^-9 relative), and outputs reach |out| ~ 4.  The
# bound is 2e-2 for the computation plus the output's own bf16 rounding: half a unit in
# the last place of the oracle value, 2^(floor(log2 |out|) - 8) (0.0156 for |out| in [4, 8)).
STRESSED_MAX = 2e-2
STRESSED_MEAN = 2e-3


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place of each |x| (normal range; 0 for x == 0)."""
    _, e = np.frexp(np.abs(x))          # |x| = m * 2^e, m in [0.5, 1): ulp = 2^(e - 8)
    return np.where(x == 0, 0.0, np.ldexp(1.0, e - 9))


def check_stressed(got: np.ndarray, want: np.ndarray):
    """Element-wise |got - want| <= STRESSED_MAX + half_ulp_bf16(want), mean <= STRESSED_MEAN."""
    assert np.all(np.isfinite(got))
    d = np.abs(got - want)
    excess = d - (STRESSED_MAX + half_ulp_bf16(want))
    assert excess.max() <= 0 and d.mean() <= STRESSED_MEAN, (float(d.max()), float(excess.max()), float(d.mean()))
    return float(d.max()), float(d.mean())
