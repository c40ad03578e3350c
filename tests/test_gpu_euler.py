"""Euler kernel vs the oracle: bit-exact, through the C ABI."""
import os

import numpy as np
import pytest
import torch

from gpu_util import from_dev, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from kv_cache_serving_ws_b200.workloads import V02, key
from oracle import ws_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _run(xb, vb, dt):
    x, v = to_dev(xb), to_dev(vb)
    assert ws.ws_flow_step(x, v, dt, check=False) == ws.WS_OK
    torch.cuda.synchronize()
    return from_dev(x)


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 7, 8, 9, 4097, 1_000_003])
@pytest.mark.parametrize("dt", [0.25, 0.1, -0.37, 0.0])
def test_euler_bit_exact_random_patterns(n, dt):
    require_gpu()
    rng = np.random.default_rng(n)
    xb = rng.integers(0, 2 ** 16, size=n, dtype=np.uint32).astype(np.uint16)   # every pattern: NaN, inf, subnormal
    vb = rng.integers(0, 2 ** 16, size=n, dtype=np.uint32).astype(np.uint16)
    assert np.array_equal(_run(xb, vb, dt), orc.euler_step(xb, vb, dt))


@pytest.mark.gpu
def test_euler_every_x_pattern():
    require_gpu()
    rng = np.random.default_rng(1)
    vs = np.concatenate([[0x0000, 0x8000, 0x0001, 0x7F7F, 0xFF7F, 0x3F80, 0xBF80, 0x7F80, 0x7FC0],
                         rng.integers(0, 2 ** 16, size=55, dtype=np.uint32)]).astype(np.uint16)
    xb = np.tile(np.arange(2 ** 16, dtype=np.uint32).astype(np.uint16), len(vs))
    vb = np.repeat(vs, 2 ** 16)
    assert np.array_equal(_run(xb, vb, 0.25), orc.euler_step(xb, vb, 0.25))


@pytest.mark.gpu
def test_euler_golden_cases():
    require_gpu()
    with open(os.path.join(GOLDEN, "euler_cases.txt")) as f:
        rows = [[c.strip() for c in ln.split("|", 4)] for ln in f if ln.strip() and not ln.startswith("#")]
    for xh, vh, dt, want, _ in rows:
        got = _run(np.array([int(xh, 16)], np.uint16), np.array([int(vh, 16)], np.uint16), float(dt))
        assert int(got[0]) == int(want, 16), (xh, vh, dt, hex(int(got[0])))


@pytest.mark.gpu
def test_euler_in_place_alias_and_guards():
    require_gpu()
    rng = np.random.default_rng(2)
    n, pad = 10_007, 64
    buf = rng.integers(0, 2 ** 16, size=n + 2 * pad, dtype=np.uint32).astype(np.uint16)
    t = to_dev(buf)
    mid = t[pad:pad + n]
    assert ws.ws_flow_step(mid, mid, 0.5, check=False) == ws.WS_OK        # x == v
    torch.cuda.synchronize()
    got = from_dev(t)
    assert np.array_equal(got[:pad], buf[:pad]) and np.array_equal(got[pad + n:], buf[pad + n:])
    assert np.array_equal(got[pad:pad + n], orc.euler_step(buf[pad:pad + n], buf[pad:pad + n], 0.5))


@pytest.mark.gpu
def test_euler_unit_latent_four_steps():
    """A whole 640x368 unit latent (Nq*H*D elements), 4 steps of dt = 0.25 with fresh velocities."""
    require_gpu()
    w = V02
    n = w.n_query * w.n_heads * w.head_dim
    x0 = synth.normal_tensor(key(w, synth.KIND_X, w.unit), (n,))
    x = to_dev(x0)
    want = x0
    for s in range(4):
        vb = synth.normal_tensor(key(w, synth.KIND_VEL, w.unit, 0, s), (n,))
        assert ws.ws_flow_step(x, to_dev(vb), 0.25, check=False) == ws.WS_OK
        want = orc.euler_step(want, vb, 0.25)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(x), want)
