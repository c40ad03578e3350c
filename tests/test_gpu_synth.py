"""The device input generator reproduces the numpy generator bit for bit."""
import numpy as np
import pytest
import torch

from gpu_util import from_dev, require_gpu
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth


@pytest.mark.gpu
@pytest.mark.parametrize("n,offset", [(1, 0), (4097, 0), (1_000_003, 0), (65536, 123_456_789)])
def test_device_generator_matches_numpy(n, offset):
    require_gpu()
    k = synth.stream_key(7, synth.KIND_MISC, unit=n, layer=3)
    t = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    ws.synth_fill(t, k, offset)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(t), synth.normal_tensor(k, (n,), offset=offset))
