"""ws_attention_noalloc -- attention for callers that cannot allocate device memory
(frameworks that own every allocation, real-time loops that may not take the
allocator's locks) -- gives the same result as ws_unit_attention on the same keys,
and matches the fp64 oracle on sampled heads, for calls in a row that reuse its
shared scratch array with different shapes, the last one long enough to merge its
cut items inside the kernel.  A call whose bounded wait runs out is reported by
ws_attention_noalloc_sync, and the next call is correct again.
Kept in a file of its own, collected last."""
import os

import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, from_dev, require_gpu
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc


def _oracle_heads(q, kv, heads):
    """fp64 oracle over the caller's planes for a few heads: q [Nq][H][D], kv [2][H][Nk][D]."""
    qb = orc.bf16_to_f64(from_dev(q))
    kvb = from_dev(kv)
    k = orc.bf16_to_f64(kvb[0]).transpose(1, 0, 2)        # [Nk][H][D]
    v = orc.bf16_to_f64(kvb[1]).transpose(1, 0, 2)
    return orc.attention_rows(qb, k, v, heads=heads)


def _reference_and_keys(cfg, layer, seed):
    """Run ws_unit_attention on a small cache and return (q, out, kv planes [2][H][Nk][D])."""
    L, H, D, Nv, Na, Nc, U = cfg
    Nq = Nv + Na
    _, h = ws.ws_cache_create(ws.make_config(L, H, D, Nv, Na, Nc, U))
    def bits(kind, shape, u=0, l=0):                 # the device twin of the seeded generator
        t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        ws.synth_fill(t, synth.stream_key(seed, kind, u, l))
        return t
    unit = U + 1
    for u in range(unit + 1):
        ws.ws_cache_append(h, u, ws.WS_SEG_COND, bits(synth.KIND_COND_K, (L, Nc, H, D), u),
                           bits(synth.KIND_COND_V, (L, Nc, H, D), u))
        if u < unit:
            ws.ws_cache_append(h, u, ws.WS_SEG_LATENT, bits(synth.KIND_COMMIT_K, (L, Nq, H, D), u),
                               bits(synth.KIND_COMMIT_V, (L, Nq, H, D), u))
    q = bits(synth.KIND_Q, (Nq, H, D), unit, layer)
    kn = bits(synth.KIND_K_NEW, (Nq, H, D), unit, layer)
    vn = bits(synth.KIND_V_NEW, (Nq, H, D), unit, layer)
    out = torch.empty_like(q)
    ws.ws_unit_attention(h, layer, unit, q, kn, vn, out)
    # the visible keys (units unit-U .. unit), read back from the cache
    ks, vs = [], []
    for u in range(unit - U, unit + 1):
        for seg, n in ((ws.WS_SEG_COND, Nc), (ws.WS_SEG_LATENT, Nq)):
            kb = torch.empty((n, H, D), dtype=torch.bfloat16, device="cuda")
            vb = torch.empty_like(kb)
            ws.ws_cache_read(h, layer, u, seg, kb, vb)
            ks.append(kb)
            vs.append(vb)
    assert ws.ws_sync(h, check=False) == ws.WS_OK
    ws.ws_cache_destroy(h)
    k = torch.cat(ks).permute(1, 0, 2)          # [H][Nk][D]
    v = torch.cat(vs).permute(1, 0, 2)
    kv = torch.stack([k, v]).contiguous()       # [2][H][Nk][D]
    return q, out, kv


@pytest.mark.gpu
def test_noalloc_matches_unit_attention_on_two_calls_in_a_row():
    require_gpu()
    cases = [((2, 6, 128, 250, 4, 16, 3), 1, 21),   # D = 128, key ranges cut between CTAs
             ((1, 5, 64, 300, 7, 9, 2), 0, 22),     # D = 64, other shapes: reuses the same scratch
             # 40 heads x 256 key tiles over 148 CTAs (69 iterations each): cut items are
             # merged inside the kernel, with the arrival counters in the static array
             ((1, 40, 128, 250, 6, 0, 127), 0, 23)]
    for cfg, layer, seed in cases:
        q, ref, kv = _reference_and_keys(cfg, layer, seed)
        _, H, D, Nv, Na, _, _ = cfg
        Nq, Nk = Nv + Na, kv.shape[2]
        out = torch.full_like(q, float("nan"))
        assert ws.ws_attention_noalloc(q, kv, out, Nq, Nk, H, D, check=False) == ws.WS_OK
        torch.cuda.synchronize()
        assert ws.ws_attention_noalloc_sync(check=False) == ws.WS_OK
        got = out.to(torch.float64).cpu().numpy()
        want = ref.to(torch.float64).cpu().numpy()
        assert np.all(np.isfinite(got))
        d = np.abs(got - want)
        assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (cfg, float(d.max()), float(d.mean()))
        # and against the oracle itself on two heads (first and last)
        heads = [0, H - 1]
        d = np.abs(got[:, heads] - _oracle_heads(q, kv, heads))
        assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (cfg, float(d.max()), float(d.mean()))
    # the entry point allocates no device memory: after the calls above (module and
    # scratch already loaded), more calls leave the device's free memory as it was
    # (any cudaMalloc takes at least a 2 MiB page)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert ws.ws_attention_noalloc(q, kv, out, Nq, Nk, H, D, check=False) == ws.WS_OK
    torch.cuda.synchronize()
    assert ws.ws_attention_noalloc_sync(check=False) == ws.WS_OK
    assert free0 - torch.cuda.mem_get_info()[0] < (1 << 20)


@pytest.mark.gpu
def test_noalloc_reports_a_wait_that_ran_out_then_recovers():
    """The stall hook (NULL cache: the no-alloc calls) leaves out one V load per CTA,
    so every CTA's bounded wait (200 ms here) runs out; ws_attention_noalloc_sync
    reports WS_ERR_DEVICE_TIMEOUT once, and the next call matches the oracle."""
    require_gpu()
    H, D, Nq, Nk = 4, 128, 300, 1000
    key = lambda kind: synth.stream_key(29, kind, 0, 0)
    q = torch.empty((Nq, H, D), dtype=torch.bfloat16, device="cuda")
    kv = torch.empty((2, H, Nk, D), dtype=torch.bfloat16, device="cuda")
    ws.synth_fill(q, key(synth.KIND_Q))
    ws.synth_fill(kv, key(synth.KIND_K_NEW))
    out = torch.empty_like(q)
    old = os.environ.get("WS_WAIT_TIMEOUT_MS")
    os.environ["WS_WAIT_TIMEOUT_MS"] = "200"
    try:
        ws.ws_debug_inject_stall(None, 0)
        assert ws.ws_attention_noalloc(q, kv, out, Nq, Nk, H, D, check=False) == ws.WS_OK
        assert ws.ws_attention_noalloc_sync(check=False) == ws.WS_ERR_DEVICE_TIMEOUT
        assert ws.ws_attention_noalloc_sync(check=False) == ws.WS_OK       # read once, then cleared
    finally:
        ws.ws_debug_inject_stall(None, -1)
        if old is None:
            os.environ.pop("WS_WAIT_TIMEOUT_MS", None)
        else:
            os.environ["WS_WAIT_TIMEOUT_MS"] = old
    assert ws.ws_attention_noalloc(q, kv, out, Nq, Nk, H, D, check=False) == ws.WS_OK
    assert ws.ws_attention_noalloc_sync(check=False) == ws.WS_OK
    got = out.to(torch.float64).cpu().numpy()
    d = np.abs(got - _oracle_heads(q, kv, range(H)))
    assert np.all(np.isfinite(got))
    assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (float(d.max()), float(d.mean()))


@pytest.mark.gpu
def test_noalloc_rejects_bad_arguments_before_any_launch():
    require_gpu()
    t = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    assert ws.ws_attention_noalloc(t, t, t, 0, 8, 1, 64, check=False) == ws.WS_ERR_ARG
    assert ws.ws_attention_noalloc(t, t, t, 1, 8, 1, 96, check=False) == ws.WS_ERR_UNSUPPORTED
    odd = torch.zeros(80, dtype=torch.bfloat16, device="cuda")[1:65]
    assert ws.ws_attention_noalloc(odd, t, t, 1, 1, 1, 64, check=False) == ws.WS_ERR_ALIGN
    # partials of 4096 query tiles x 64 heads cannot fit the 48 MiB array
    assert ws.ws_attention_noalloc(t, t, t, 4096 * 128, 1 << 20, 64, 128, check=False) == ws.WS_ERR_UNSUPPORTED
    # a stream of another device than the current one (only with two GPUs)
    if torch.cuda.device_count() > 1:
        with torch.cuda.device(1):
            other = torch.cuda.Stream()
        assert ws.ws_attention_noalloc(t, t, t, 1, 1, 1, 64, stream=other, check=False) == ws.WS_ERR_ARG


@pytest.mark.gpu
def test_noalloc_on_a_second_device_after_the_first():
    """Kernel attributes (the shared-memory opt-in) and the scratch address are kept per
    device: a call on device 1 after calls on device 0 gives the same bytes.  Needs two
    GPUs; skipped otherwise."""
    require_gpu()
    if torch.cuda.device_count() < 2:
        pytest.skip("one GPU visible")
    H, D, Nq, Nk = 3, 128, 260, 700
    key = lambda kind: synth.stream_key(31, kind, 0, 0)
    outs = []
    for dev in (0, 1):
        with torch.cuda.device(dev):
            q = torch.empty((Nq, H, D), dtype=torch.bfloat16, device=f"cuda:{dev}")
            kv = torch.empty((2, H, Nk, D), dtype=torch.bfloat16, device=f"cuda:{dev}")
            ws.synth_fill(q, key(synth.KIND_Q))
            ws.synth_fill(kv, key(synth.KIND_K_NEW))
            out = torch.empty_like(q)
            stream = torch.cuda.current_stream()
            assert ws.ws_attention_noalloc(q, kv, out, Nq, Nk, H, D, stream=stream, check=False) == ws.WS_OK
            assert ws.ws_attention_noalloc_sync(stream=stream, check=False) == ws.WS_OK
            outs.append(out.cpu())
    assert torch.equal(outs[0], outs[1])
