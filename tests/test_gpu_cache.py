"""Cache append / commit / readback / slot table on the GPU vs the oracle's cache
model: bit-exact bytes, identical slot table and identical status codes."""
import numpy as np
import pytest
import torch

from gpu_util import from_dev, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc


def _pair(cfg, seg, seed, unit):
    n = cfg.n_cond if seg == orc.SEG_COND else cfg.n_query
    shape = (cfg.n_layers, n, cfg.n_heads, cfg.head_dim)
    kk = synth.KIND_COND_K if seg == orc.SEG_COND else synth.KIND_COMMIT_K
    kv = synth.KIND_COND_V if seg == orc.SEG_COND else synth.KIND_COMMIT_V
    return (synth.normal_tensor(synth.stream_key(seed, kk, unit), shape),
            synth.normal_tensor(synth.stream_key(seed, kv, unit), shape))


class Twin:
    """The same operations on the GPU library and on the oracle model."""

    def __init__(self, cfg):
        self.cfg = cfg
        self.ocache = orc.UnitCache(cfg)
        self.wcfg = ws.make_config(cfg.n_layers, cfg.n_heads, cfg.head_dim, cfg.n_video, cfg.n_audio, cfg.n_cond,
                                   cfg.history_units)
        _, self.h = ws.ws_cache_create(self.wcfg)

    def append(self, unit, seg, seed=3):
        k, v = _pair(self.cfg, seg, seed, unit)
        a = ws.ws_cache_append(self.h, unit, seg, to_dev(k), to_dev(v), check=False)
        b = self.ocache.append(unit, seg, k, v)
        assert a == b, (unit, seg, a, b)
        return a

    def attention(self, layer, unit, seed=5):
        c = self.cfg
        qs = (c.n_query, c.n_heads, c.head_dim)
        bits = [synth.normal_tensor(synth.stream_key(seed, kind, unit, layer), qs)
                for kind in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW)]
        dev = [to_dev(b) for b in bits]
        out = torch.empty_like(dev[0])
        a = ws.ws_unit_attention(self.h, layer, unit, *dev, out, check=False)
        b, _ = self.ocache.unit_attention(layer, unit, *bits, rows=[], heads=[])
        assert a == b, (layer, unit, a, b)

    def check_state(self):
        torch.cuda.synchronize()
        assert ws.ws_cache_slot_table(self.h) == self.ocache.slot_table()
        c = self.cfg
        units = sorted(set(u for u in self.ocache.slot_table() if u >= 0))
        probe = units + [u - c.slots for u in units if u - c.slots >= 0] + [max(units, default=0) + 1]
        for u in probe:
            for layer in range(c.n_layers):
                for seg, n in ((orc.SEG_COND, c.n_cond), (orc.SEG_LATENT, c.n_query)):
                    pad = 16
                    kbuf = torch.full((n * c.n_heads * c.head_dim + 2 * pad,), 7, dtype=torch.int16, device="cuda")
                    vbuf = torch.full_like(kbuf, 9)
                    ko, vo = kbuf[pad:pad + n * c.n_heads * c.head_dim], vbuf[pad:pad + n * c.n_heads * c.head_dim]
                    a = ws.ws_cache_read(self.h, layer, u, seg, ko, vo, check=False)
                    st, k, v = self.ocache.read(layer, u, seg)
                    assert a == st, (u, layer, seg, a, st)
                    torch.cuda.synchronize()
                    kb, vb = kbuf.cpu().numpy(), vbuf.cpu().numpy()
                    assert (kb[:pad] == 7).all() and (kb[-pad:] == 7).all()    # guards untouched
                    assert (vb[:pad] == 9).all() and (vb[-pad:] == 9).all()
                    if st == orc.OK and n > 0:
                        assert np.array_equal(from_dev(ko), k.reshape(-1))
                        assert np.array_equal(from_dev(vo), v.reshape(-1))

    def close(self):
        ws.ws_cache_destroy(self.h)


@pytest.mark.gpu
def test_tiny_workload_prefill_bit_exact():
    require_gpu()
    cfg = orc.Config(1, 8, 64, 252, 8, 64, 4)
    t = Twin(cfg)
    for u in range(4):
        t.append(u, orc.SEG_COND)
        t.append(u, orc.SEG_LATENT)
    t.append(4, orc.SEG_COND)
    t.attention(0, 4)
    t.check_state()
    t.close()


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
def test_ring_wraps_gaps_and_status_codes(head_dim):
    require_gpu()
    cfg = orc.Config(n_layers=2, n_heads=3, head_dim=head_dim, n_video=5, n_audio=2, n_cond=3, history_units=3)
    t = Twin(cfg)
    rng = np.random.default_rng(head_dim)
    u = 0
    t.attention(0, 0)                                    # nothing appended yet: NOT_READY on both
    for _ in range(30):
        r = rng.random()
        if r < 0.45:
            u += int(rng.choice([1, 1, 2, 3]))
            t.append(u, orc.SEG_COND)
        elif r < 0.6:
            t.append(max(0, u - int(rng.integers(0, 3))), orc.SEG_COND)   # older or same unit
        elif r < 0.85:
            t.append(max(0, u - int(rng.integers(0, 6))), orc.SEG_LATENT)
        else:
            t.attention(int(rng.integers(0, 2)), u - int(rng.integers(0, 2)))
    t.check_state()
    t.close()


@pytest.mark.gpu
def test_no_conditioning_tokens():
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=64, n_video=9, n_audio=0, n_cond=0, history_units=2)
    t = Twin(cfg)
    for u in range(5):
        t.append(u, orc.SEG_COND)
        t.append(u, orc.SEG_LATENT)
    t.check_state()
    t.close()


@pytest.mark.gpu
def test_argument_errors_leave_state_unchanged():
    require_gpu()
    cfg = orc.Config(1, 2, 64, 4, 0, 2, 1)
    t = Twin(cfg)
    t.append(0, orc.SEG_COND)
    k, v = _pair(cfg, orc.SEG_COND, 3, 1)
    kd, vd = to_dev(k), to_dev(v)
    odd = torch.zeros(kd.numel() + 8, dtype=torch.bfloat16, device="cuda")[1:1 + kd.numel()]
    assert ws.ws_cache_append(t.h, 1, orc.SEG_COND, odd, vd, check=False) == ws.WS_ERR_ALIGN
    assert ws.ws_cache_append(t.h, 1, 7, kd, vd, check=False) == ws.WS_ERR_ARG
    assert ws.ws_cache_append(t.h, -3, orc.SEG_COND, kd, vd, check=False) == ws.WS_ERR_ARG
    t.check_state()
    info = ws.ws_cache_get_info(t.h)
    assert info["newest_unit"] == 0 and info["slots"] == 2 and info["tokens_per_unit"] == 6
    assert info["cache_bytes"] == 1 * 2 * 2 * 2 * 6 * 64 * 2
    assert ws.ws_sync(t.h, check=False) == ws.WS_OK
    t.close()


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
def test_latent_write_inside_the_attention_launch(head_dim):
    """The single-SM kernel writes the call's latent K/V itself: one launch per call
    (no separate write), and the written rows equal k_new / v_new bit for bit, over
    a ragged unit (Nq = 133) with the ring wrapped."""
    require_gpu()
    cfg = orc.Config(n_layers=2, n_heads=3, head_dim=head_dim, n_video=130, n_audio=3, n_cond=5, history_units=2)
    t = Twin(cfg)
    for u in range(6):
        t.append(u, orc.SEG_COND)
        if u < 5:
            t.append(u, orc.SEG_LATENT)
    ws.ws_profile_enable(t.h, True)
    t.attention(1, 5)
    t.attention(0, 5)
    torch.cuda.synchronize()
    prof = ws.ws_profile_read(t.h)
    ws.ws_profile_enable(t.h, False)
    assert prof["last_kernel"] == 1
    assert prof["latent_write_launches"] == 0 and prof["attention_launches"] == 2
    t.check_state()
    t.close()
