"""Multi-unit (prefill) block-causal attention on the GPU vs the oracle: several query
units in one launch, each over its own window of units, whole units outside a window
never loaded; status codes identical to the oracle's."""
import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, dev_f64, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc


class PrefillPair:
    def __init__(self, cfg, seed):
        self.cfg, self.seed = cfg, seed
        self.o = orc.UnitCache(cfg)
        _, self.h = ws.ws_cache_create(ws.make_config(cfg.n_layers, cfg.n_heads, cfg.head_dim, cfg.n_video,
                                                      cfg.n_audio, cfg.n_cond, cfg.history_units))

    def bits(self, kind, shape, unit=0, layer=0):
        return synth.normal_tensor(synth.stream_key(self.seed, kind, unit, layer), shape)

    def cond(self, u):
        c = self.cfg
        s = (c.n_layers, c.n_cond, c.n_heads, c.head_dim)
        k, v = self.bits(synth.KIND_COND_K, s, u), self.bits(synth.KIND_COND_V, s, u)
        assert ws.ws_cache_append(self.h, u, ws.WS_SEG_COND, to_dev(k), to_dev(v), check=False) == 0
        assert self.o.append(u, orc.SEG_COND, k, v) == 0

    def commit(self, u):
        c = self.cfg
        s = (c.n_layers, c.n_query, c.n_heads, c.head_dim)
        k, v = self.bits(synth.KIND_COMMIT_K, s, u), self.bits(synth.KIND_COMMIT_V, s, u)
        assert ws.ws_cache_append(self.h, u, ws.WS_SEG_LATENT, to_dev(k), to_dev(v), check=False) == 0
        assert self.o.append(u, orc.SEG_LATENT, k, v) == 0

    def prefill(self, layer, u_first, n, splits=0, rows=None, heads=None, expect=orc.OK):
        c = self.cfg
        s = (n, c.n_query, c.n_heads, c.head_dim)
        q = self.bits(synth.KIND_Q, s, u_first, layer)
        kn = self.bits(synth.KIND_K_NEW, s, u_first, layer)
        vn = self.bits(synth.KIND_V_NEW, s, u_first, layer)
        ws.ws_cache_set_splits(self.h, splits)
        out = torch.empty(s, dtype=torch.bfloat16, device="cuda")
        st_g = ws.ws_prefill_attention(self.h, layer, u_first, n, to_dev(q), to_dev(kn), to_dev(vn), out,
                                       check=False)
        st_o, want = self.o.prefill_attention(layer, u_first, n, q, kn, vn, rows=rows, heads=heads)
        assert st_g == st_o == expect, (st_g, st_o, expect)
        if expect != orc.OK:
            return None
        assert ws.ws_sync(self.h, check=False) == ws.WS_OK
        got = dev_f64(out)
        if rows is not None:
            got = got[:, rows]
        if heads is not None:
            got = got[:, :, heads]
        d = np.abs(got - want)
        assert np.all(np.isfinite(got))
        assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (float(d.max()), float(d.mean()))
        return d

    def close(self):
        ws.ws_cache_destroy(self.h)


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_prefill_from_scratch_and_mid_stream(head_dim, splits):
    require_gpu()
    cfg = orc.Config(n_layers=2, n_heads=3, head_dim=head_dim, n_video=130, n_audio=3, n_cond=5, history_units=5)
    p = PrefillPair(cfg, seed=40 + head_dim + splits)
    for u in range(4):                                   # prompt prefill: units 0..3 at once
        p.cond(u)
    p.prefill(1, 0, 4, splits=splits)
    for u in range(4):
        p.commit(u)
    for u in range(4, 6):                                # a later stretch: units 4..5, windows reach back to unit 0
        p.cond(u)
    p.prefill(0, 4, 2, splits=splits)
    p.close()


@pytest.mark.gpu
def test_prefill_status_codes_match_the_oracle():
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=64, n_video=20, n_audio=0, n_cond=3, history_units=3)
    p = PrefillPair(cfg, seed=7)
    for u in range(4):
        p.cond(u)
    p.prefill(0, 2, 3, expect=orc.ERR_NOT_READY)
    p.prefill(0, 1, 2, expect=orc.ERR_UNIT_ORDER)
    p.prefill(0, 1, 3)
    p.cond(4)                                            # takes unit 0's slot
    p.prefill(0, 1, 4, expect=orc.ERR_EVICTED)
    p.prefill(0, 0, 5, expect=orc.ERR_EVICTED)
    p.prefill(0, 4, 1)
    p.close()


@pytest.mark.gpu
def test_prefill_sixty_four_units():
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=128, n_video=40, n_audio=2, n_cond=6, history_units=63)
    p = PrefillPair(cfg, seed=8)
    for u in range(64):
        p.cond(u)
    p.prefill(0, 0, 64)
    p.cond(64)
    p.cond(65)
    c = cfg
    s = (65, c.n_query, c.n_heads, c.head_dim)
    z = torch.zeros(s, dtype=torch.bfloat16, device="cuda")
    assert ws.ws_prefill_attention(p.h, 0, 1, 65, z, z, z, z, check=False) == ws.WS_ERR_UNSUPPORTED
    p.close()


@pytest.mark.gpu
def test_prefill_v02_shapes_sampled():
    """16 units of the 640x368 stream at once (14784 query rows x 40 heads), 32-unit window."""
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=40, head_dim=128, n_video=920, n_audio=4, n_cond=32, history_units=32)
    p = PrefillPair(cfg, seed=9)
    for u in range(16):
        p.cond(u)
    rng = np.random.default_rng(9)
    rows = sorted(rng.choice(cfg.n_query, size=24, replace=False).tolist() + [0, cfg.n_query - 1])
    p.prefill(0, 0, 16, rows=rows, heads=[0, 21, 39])
    p.close()
