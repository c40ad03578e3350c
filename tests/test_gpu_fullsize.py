"""Parity at the full sizes of the pages' workloads, in the launch configuration the
benchmark uses (automatic split count): every query row of four heads, plus 256
(head, row) samples from eight other heads, against the oracle, which computes each
(head, row) on its own."""
import numpy as np
import pytest

from gpu_util import ATOL_MAX, ATOL_MEAN, dev_f64, require_gpu
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200.workloads import FULL, RING, V02, GpuSession
from oracle_side import oracle_cache


def _sampled_parity(w, layer, step, heads, other_heads=8, other_rows=32, seed=0):
    g = GpuSession(w)
    g.prefill()
    q, kn, vn = g.step_inputs(layer, step)
    out = g.attention(layer, q, kn, vn)
    assert ws.ws_sync(g.h, check=False) == ws.WS_OK
    got = dev_f64(out)
    g.close()
    assert np.all(np.isfinite(got))
    rng = np.random.default_rng(seed)
    cache, qb, knb, vnb = oracle_cache(w, layer, heads, step)
    st, want = cache.unit_attention(0, w.unit, qb, knb, vnb)          # every row
    assert st == 0
    errs = [np.abs(got[:, heads] - want).reshape(-1)]
    others = sorted(rng.choice([h for h in range(w.n_heads) if h not in heads], size=other_heads,
                               replace=False).tolist())
    rows2 = sorted(rng.choice(w.n_query, size=other_rows, replace=False).tolist())
    cache, qb, knb, vnb = oracle_cache(w, layer, others, step)
    st, want = cache.unit_attention(0, w.unit, qb, knb, vnb, rows=rows2)
    assert st == 0
    errs.append(np.abs(got[rows2][:, others] - want).reshape(-1))
    d = np.concatenate(errs)
    assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (float(d.max()), float(d.mean()))


@pytest.mark.gpu
def test_v02_unit_32_history_sampled():
    """924 query rows x 40 heads over 33 units of 956 tokens (31548 keys)."""
    require_gpu()
    _sampled_parity(V02, 0, 0, heads=[0, 13, 26, 39], seed=3)


@pytest.mark.gpu
def test_ring_128_history_wrapped_sampled():
    """129-slot ring after ~8 wraps (current unit 1000 in slot 97), 123324 keys."""
    require_gpu()
    _sampled_parity(RING, 0, 0, heads=[5, 15, 25, 35], seed=4)


@pytest.mark.gpu
def test_full_unit_step_one_layer_sampled():
    """40-layer, 64-unit-history cache (~50 GB); layer 23 at Euler step 2."""
    require_gpu()
    _sampled_parity(FULL, 23, 2, heads=[0, 11, 22, 33], seed=5)
