"""Independent caches driven from different CUDA streams at the same time, and the
multi-unit paths on stressed queries.  Each cache owns its workspace, status word
and merge counters, so interleaved launches on two streams must give each cache
the oracle's results."""
import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, check_stressed, dev_f64, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc


class Side:
    """One cache, its oracle and its stream."""

    def __init__(self, cfg, seed, stream):
        self.cfg, self.seed, self.stream = cfg, seed, stream
        self.o = orc.UnitCache(cfg)
        _, self.h = ws.ws_cache_create(ws.make_config(cfg.n_layers, cfg.n_heads, cfg.head_dim, cfg.n_video,
                                                      cfg.n_audio, cfg.n_cond, cfg.history_units))

    def bits(self, kind, shape, u, layer=0):
        return synth.normal_tensor(synth.stream_key(self.seed, kind, u, layer), shape)

    def unit(self, u, commit=True):
        # device buffers allocated on this side's stream: the caching allocator
        # reuses them only behind this stream's own work
        c = self.cfg
        cs, ls = (c.n_layers, c.n_cond, c.n_heads, c.head_dim), (c.n_layers, c.n_query, c.n_heads, c.head_dim)
        with torch.cuda.stream(self.stream):
            k, v = self.bits(synth.KIND_COND_K, cs, u), self.bits(synth.KIND_COND_V, cs, u)
            ws.ws_cache_append(self.h, u, ws.WS_SEG_COND, to_dev(k), to_dev(v), stream=self.stream)
            self.o.append(u, orc.SEG_COND, k, v)
            if commit:
                k, v = self.bits(synth.KIND_COMMIT_K, ls, u), self.bits(synth.KIND_COMMIT_V, ls, u)
                ws.ws_cache_append(self.h, u, ws.WS_SEG_LATENT, to_dev(k), to_dev(v), stream=self.stream)
                self.o.append(u, orc.SEG_LATENT, k, v)

    def inputs(self, u, layer, q_scale=None):
        c = self.cfg
        s = (c.n_query, c.n_heads, c.head_dim)
        q = self.bits(synth.KIND_Q, s, u, layer)
        if q_scale is not None:
            q = q_scale(q)
        return q, self.bits(synth.KIND_K_NEW, s, u, layer), self.bits(synth.KIND_V_NEW, s, u, layer)


def _check(got, want, max_tol=ATOL_MAX, mean_tol=ATOL_MEAN):
    d = np.abs(got - want)
    assert np.all(np.isfinite(got))
    assert d.max() <= max_tol and d.mean() <= mean_tol, (float(d.max()), float(d.mean()))


@pytest.mark.gpu
def test_two_caches_on_two_streams_interleaved():
    require_gpu()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    # a: 7 heads x 22 key tiles over 2 CTAs, 77 iterations each: cut items merged in-kernel
    a = Side(orc.Config(2, 7, 128, 250, 6, 16, 9), 81, s1)
    b = Side(orc.Config(2, 3, 64, 130, 3, 5, 3), 82, s2)        # short calls: separate merge launches
    for u in range(10):
        a.unit(u, commit=u < 9)
        if u < 4:
            b.unit(u, commit=u < 3)
    ws.ws_cache_set_splits(a.h, 2)
    outs, wants = [], []
    for layer in range(2):                                       # launches alternate between the streams
        for side, u in ((a, 9), (b, 3)):
            q, kn, vn = side.inputs(u, layer)
            with torch.cuda.stream(side.stream):
                out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
                dq, dk, dv = to_dev(q), to_dev(kn), to_dev(vn)
                ws.ws_unit_attention(side.h, layer, u, dq, dk, dv, out, stream=side.stream)
            st, want = side.o.unit_attention(layer, u, q, kn, vn)
            assert st == orc.OK
            outs.append((side, out))
            wants.append(want)
    torch.cuda.synchronize()
    for (side, out), want in zip(outs, wants):
        assert ws.ws_sync(side.h, stream=side.stream, check=False) == ws.WS_OK
        _check(dev_f64(out), want)
    ws.ws_cache_destroy(a.h)
    ws.ws_cache_destroy(b.h)


@pytest.mark.gpu
def test_prefill_and_sessions_on_stressed_queries():
    """Queries scaled by 4 (logit std 4): the reference max moves often; multi-unit and
    multi-session calls keep the stressed-query tolerance of the single-unit path."""
    require_gpu()
    times4 = lambda bits: orc.f64_to_bf16(orc.bf16_to_f64(bits) * 4.0)
    cfg = orc.Config(1, 4, 128, 250, 6, 8, 5)
    _, h = ws.ws_pool_create(ws.make_config(1, 4, 128, 250, 6, 8, 5), 2)
    pool = orc.SessionPool(cfg, 2)
    bits = lambda s, kind, shape, u: synth.normal_tensor(synth.stream_key(90 + s, kind, u), shape)
    cs = (1, 8, 4, 128)
    for s in range(2):
        for u in range(4 + s):
            k, v = bits(s, synth.KIND_COND_K, cs, u), bits(s, synth.KIND_COND_V, cs, u)
            ws.ws_session_append(h, s, u, ws.WS_SEG_COND, to_dev(k), to_dev(v))
            assert pool.sessions[s].append(u, orc.SEG_COND, k, v) == orc.OK
    # session 0: a 4-unit prefill stretch; session 1: a 5-unit one; one launch
    sessions, units = [0] * 4 + [1] * 5, list(range(4)) + list(range(5))
    shape = (9, 256, 4, 128)
    q = times4(bits(7, synth.KIND_Q, shape, 0))
    kn, vn = bits(7, synth.KIND_K_NEW, shape, 0), bits(7, synth.KIND_V_NEW, shape, 0)
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    ws.ws_session_attention(h, 0, sessions, units, to_dev(q), to_dev(kn), to_dev(vn), out)
    assert ws.ws_sync(h, check=False) == ws.WS_OK
    st, want = pool.session_attention(0, sessions, units, q, kn, vn)
    assert st == orc.OK
    check_stressed(dev_f64(out), want)
    ws.ws_cache_destroy(h)
