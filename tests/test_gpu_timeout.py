"""Failure detection without a GPU fault: a test hook leaves out one V load per
CTA, every CTA's bounded wait runs out, the kernel leaves cleanly (copies drained,
TMEM freed), ws_sync reports WS_ERR_DEVICE_TIMEOUT, and the next call on the same
cache is correct again."""
import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, dev_f64, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc


@pytest.mark.gpu
def test_bounded_wait_runs_out_is_reported_and_the_context_stays_usable(monkeypatch):
    require_gpu()
    monkeypatch.setenv("WS_WAIT_TIMEOUT_MS", "200")     # read when the cache is created
    cfg = orc.Config(1, 8, 64, 252, 8, 64, 4)
    _, h = ws.ws_cache_create(ws.make_config(1, 8, 64, 252, 8, 64, 4))
    o = orc.UnitCache(cfg)
    bits = lambda kind, shape, u=0: synth.normal_tensor(synth.stream_key(31, kind, u), shape)
    cs, ls, qs = (1, 64, 8, 64), (1, 260, 8, 64), (260, 8, 64)
    for u in range(5):
        k, v = bits(synth.KIND_COND_K, cs, u), bits(synth.KIND_COND_V, cs, u)
        ws.ws_cache_append(h, u, ws.WS_SEG_COND, to_dev(k), to_dev(v))
        o.append(u, orc.SEG_COND, k, v)
        if u < 4:
            k, v = bits(synth.KIND_COMMIT_K, ls, u), bits(synth.KIND_COMMIT_V, ls, u)
            ws.ws_cache_append(h, u, ws.WS_SEG_LATENT, to_dev(k), to_dev(v))
            o.append(u, orc.SEG_LATENT, k, v)
    q, kn, vn = (bits(kd, qs, 4) for kd in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
    out = torch.empty(qs, dtype=torch.bfloat16, device="cuda")
    assert ws.ws_sync(h, check=False) == ws.WS_OK

    ws.ws_debug_inject_stall(h, 1)
    assert ws.ws_unit_attention(h, 0, 4, to_dev(q), to_dev(kn), to_dev(vn), out, check=False) == ws.WS_OK
    assert ws.ws_sync(h, check=False) == ws.WS_ERR_DEVICE_TIMEOUT
    assert ws.ws_sync(h, check=False) == ws.WS_OK       # the status word was cleared

    ws.ws_debug_inject_stall(h, -1)
    assert ws.ws_unit_attention(h, 0, 4, to_dev(q), to_dev(kn), to_dev(vn), out, check=False) == ws.WS_OK
    assert ws.ws_sync(h, check=False) == ws.WS_OK
    st, want = o.unit_attention(0, 4, q, kn, vn)
    d = np.abs(dev_f64(out) - want)
    assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN
    ws.ws_cache_destroy(h)


@pytest.mark.gpu
def test_inject_hook_validates_its_argument():
    require_gpu()
    _, h = ws.ws_cache_create(ws.make_config(1, 1, 64, 4, 0, 0, 0))
    assert ws.ws_debug_inject_stall(h, -2, check=False) == ws.WS_ERR_ARG
    # a NULL cache addresses the no-alloc calls' hook: -1 (off) is accepted, -2 is not
    assert ws.ws_debug_inject_stall(None, -2, check=False) == ws.WS_ERR_ARG
    assert ws.ws_debug_inject_stall(None, -1, check=False) == ws.WS_OK
    ws.ws_cache_destroy(h)


@pytest.mark.gpu
def test_timeout_during_an_in_kernel_merge_leaves_no_stale_counters(monkeypatch):
    """A call long enough to merge its cut items inside the kernel (6 CTAs x 171
    key tiles over 8 items of 128 tiles) stalls at CTA-local tile 150: some CTAs
    have already counted their piece of a cut item, the others never will.  ws_sync
    reports the timeout and clears the counters with the status word; the next call
    merges every item correctly (a stale count would make a CTA merge before the
    other piece was written)."""
    require_gpu()
    monkeypatch.setenv("WS_WAIT_TIMEOUT_MS", "200")
    H, D, Nv, Na, U = 8, 128, 250, 6, 63
    Nq = Nv + Na
    cfg = orc.Config(1, H, D, Nv, Na, 0, U)
    _, h = ws.ws_cache_create(ws.make_config(1, H, D, Nv, Na, 0, U))
    o = orc.UnitCache(cfg)
    bits = lambda kind, shape, u=0: synth.normal_tensor(synth.stream_key(37, kind, u), shape)
    cs, ls, qs = (1, 0, H, D), (1, Nq, H, D), (Nq, H, D)
    for u in range(U + 1):
        k, v = bits(synth.KIND_COND_K, cs, u), bits(synth.KIND_COND_V, cs, u)
        ws.ws_cache_append(h, u, ws.WS_SEG_COND, to_dev(k), to_dev(v))
        o.append(u, orc.SEG_COND, k, v)
        if u < U:
            k, v = bits(synth.KIND_COMMIT_K, ls, u), bits(synth.KIND_COMMIT_V, ls, u)
            ws.ws_cache_append(h, u, ws.WS_SEG_LATENT, to_dev(k), to_dev(v))
            o.append(u, orc.SEG_LATENT, k, v)
    q, kn, vn = (bits(kd, qs, U) for kd in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
    out = torch.empty(qs, dtype=torch.bfloat16, device="cuda")
    ws.ws_cache_set_splits(h, 6)
    assert ws.ws_sync(h, check=False) == ws.WS_OK

    ws.ws_debug_inject_stall(h, 150)
    assert ws.ws_unit_attention(h, 0, U, to_dev(q), to_dev(kn), to_dev(vn), out, check=False) == ws.WS_OK
    assert ws.ws_sync(h, check=False) == ws.WS_ERR_DEVICE_TIMEOUT
    prof_split = ws.ws_profile_read(h)["last_n_split"]
    assert prof_split == 6

    ws.ws_debug_inject_stall(h, -1)
    for _ in range(2):                                   # and once more on clean counters
        assert ws.ws_unit_attention(h, 0, U, to_dev(q), to_dev(kn), to_dev(vn), out, check=False) == ws.WS_OK
        assert ws.ws_sync(h, check=False) == ws.WS_OK
        st, want = o.unit_attention(0, U, q, kn, vn)
        d = np.abs(dev_f64(out) - want)
        assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (float(d.max()), float(d.mean()))
    ws.ws_cache_destroy(h)
