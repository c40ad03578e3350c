"""The R-split invariant on the GPU: heads are independent, so attention over a cache
holding all H heads equals, head for head, attention over R caches holding H/R heads
each (the head slices of the same data).  With one CTA per lane (no item is cut
between CTAs) every item is computed by the same code in the same key order, so the
outputs must be bit-identical; with the automatic decomposition the cut points
differ and the results agree within the attention tolerance."""
import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, from_dev, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth

L, H, D, NV, NA, NC, U = 1, 8, 128, 250, 6, 12, 5
NQ = NV + NA


def _bits(kind, shape, u):
    return synth.normal_tensor(synth.stream_key(55, kind, u), shape)


def _run(heads, splits):
    """Attention of unit U (after U committed units) over a cache of the given heads."""
    _, h = ws.ws_cache_create(ws.make_config(L, len(heads), D, NV, NA, NC, U))
    cs, ls, qs = (L, NC, H, D), (L, NQ, H, D), (NQ, H, D)
    for u in range(U + 1):
        k, v = _bits(synth.KIND_COND_K, cs, u)[:, :, heads], _bits(synth.KIND_COND_V, cs, u)[:, :, heads]
        ws.ws_cache_append(h, u, ws.WS_SEG_COND, to_dev(k), to_dev(v))
        if u < U:
            k, v = _bits(synth.KIND_COMMIT_K, ls, u)[:, :, heads], _bits(synth.KIND_COMMIT_V, ls, u)[:, :, heads]
            ws.ws_cache_append(h, u, ws.WS_SEG_LATENT, to_dev(k), to_dev(v))
    q, kn, vn = (_bits(kd, qs, U)[:, heads] for kd in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
    out = torch.empty((NQ, len(heads), D), dtype=torch.bfloat16, device="cuda")
    ws.ws_cache_set_splits(h, splits)
    ws.ws_unit_attention(h, 0, U, to_dev(q), to_dev(kn), to_dev(vn), out)
    assert ws.ws_sync(h, check=False) == ws.WS_OK
    got = from_dev(out)
    ws.ws_cache_destroy(h)
    return got


@pytest.mark.gpu
@pytest.mark.parametrize("R", [2, 4, 8])
def test_head_split_is_bit_identical_without_cut_items(R):
    require_gpu()
    full = _run(list(range(H)), splits=1)
    g = H // R
    parts = [_run(list(range(r * g, (r + 1) * g)), splits=1) for r in range(R)]
    assert np.array_equal(np.concatenate(parts, axis=1), full)


@pytest.mark.gpu
def test_head_split_within_tolerance_with_automatic_splits():
    require_gpu()
    from oracle.ws_oracle import bf16_to_f64
    full = bf16_to_f64(_run(list(range(H)), splits=0))
    parts = bf16_to_f64(np.concatenate([_run([0, 1, 2], 0), _run([3, 4, 5, 6, 7], 0)], axis=1))
    d = np.abs(parts - full)
    assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN
