"""Block-causal unit attention on the GPU (tcgen05 kernel, through the C ABI) vs the
fp64 oracle, element by element, at sizes the oracle finishes in seconds: several
query tiles with a ragged tail, several key tiles with partial tiles, rings with
gaps and uncommitted units, both head sizes, every split count."""
import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, check_stressed, dev_f64, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from kv_cache_serving_ws_b200.workloads import TINY, V01, GpuSession
from oracle import ws_oracle as orc
from oracle_side import oracle_cache


class Pair:
    def __init__(self, cfg, seed=11):
        self.cfg, self.seed = cfg, seed
        self.o = orc.UnitCache(cfg)
        wc = ws.make_config(cfg.n_layers, cfg.n_heads, cfg.head_dim, cfg.n_video, cfg.n_audio, cfg.n_cond,
                            cfg.history_units)
        _, self.h = ws.ws_cache_create(wc)

    def _bits(self, kind, shape, unit, layer=0):
        return synth.normal_tensor(synth.stream_key(self.seed, kind, unit, layer), shape)

    def cond(self, u):
        c = self.cfg
        s = (c.n_layers, c.n_cond, c.n_heads, c.head_dim)
        k, v = self._bits(synth.KIND_COND_K, s, u), self._bits(synth.KIND_COND_V, s, u)
        assert ws.ws_cache_append(self.h, u, ws.WS_SEG_COND, to_dev(k), to_dev(v), check=False) == 0
        assert self.o.append(u, orc.SEG_COND, k, v) == 0

    def commit(self, u):
        c = self.cfg
        s = (c.n_layers, c.n_query, c.n_heads, c.head_dim)
        k, v = self._bits(synth.KIND_COMMIT_K, s, u), self._bits(synth.KIND_COMMIT_V, s, u)
        assert ws.ws_cache_append(self.h, u, ws.WS_SEG_LATENT, to_dev(k), to_dev(v), check=False) == 0
        assert self.o.append(u, orc.SEG_LATENT, k, v) == 0

    def attend(self, layer, u, q_scale=None, splits=0):
        c = self.cfg
        s = (c.n_query, c.n_heads, c.head_dim)
        q = self._bits(synth.KIND_Q, s, u, layer)
        if q_scale is not None:
            q = q_scale(q)
        kn, vn = self._bits(synth.KIND_K_NEW, s, u, layer), self._bits(synth.KIND_V_NEW, s, u, layer)
        ws.ws_cache_set_splits(self.h, splits)
        out = torch.empty(s, dtype=torch.bfloat16, device="cuda")
        assert ws.ws_unit_attention(self.h, layer, u, to_dev(q), to_dev(kn), to_dev(vn), out, check=False) == 0
        assert ws.ws_sync(self.h, check=False) == ws.WS_OK
        st, want = self.o.unit_attention(layer, u, q, kn, vn)
        assert st == 0
        return dev_f64(out), want

    def close(self):
        ws.ws_cache_destroy(self.h)


def _check(got, want, max_tol=ATOL_MAX, mean_tol=ATOL_MEAN):
    assert np.all(np.isfinite(got))
    d = np.abs(got - want)
    assert d.max() <= max_tol and d.mean() <= mean_tol, (float(d.max()), float(d.mean()))
    return float(d.max()), float(d.mean())


def _times4(bits):
    """q * 4: adds 2 to the bf16 exponent (exact for these magnitudes)."""
    f = orc.bf16_to_f64(bits) * 4.0
    return orc.f64_to_bf16(f)


@pytest.mark.gpu
@pytest.mark.parametrize("splits", [0, 1, 2, 5, 13])
def test_tiny_workload_all_heads_all_rows(splits):
    require_gpu()
    w = TINY
    p = Pair(orc.Config(w.n_layers, w.n_heads, w.head_dim, w.n_video, w.n_audio, w.n_cond, w.history_units),
             seed=w.seed)
    for u in w.history():
        p.cond(u)
        p.commit(u)
    p.cond(w.unit)
    got, want = p.attend(0, w.unit, splits=splits)
    _check(got, want)
    p.close()


@pytest.mark.gpu
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_v01_workload_all_heads_all_rows(splits):
    """40 heads x 128, 256 query rows, 17 units of 288 tokens (4896 keys)."""
    require_gpu()
    w = V01
    g = GpuSession(w)
    g.prefill()
    ws.ws_cache_set_splits(g.h, splits)
    q, kn, vn = g.step_inputs(0)
    out = g.attention(0, q, kn, vn)
    assert ws.ws_sync(g.h, check=False) == 0
    cache, qb, knb, vnb = oracle_cache(w, 0, range(w.n_heads))
    st, want = cache.unit_attention(0, w.unit, qb, knb, vnb)
    assert st == 0
    _check(dev_f64(out), want)
    g.close()


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("splits", [0, 1, 4])
def test_ragged_tiles_gaps_and_uncommitted_units(head_dim, splits):
    """Nq = 133 (two query tiles, the second ragged), T = 138 (key runs end mid-tile),
    a gap in the unit sequence and an uncommitted unit (conditioning rows only)."""
    require_gpu()
    cfg = orc.Config(n_layers=2, n_heads=3, head_dim=head_dim, n_video=130, n_audio=3, n_cond=5, history_units=4)
    p = Pair(cfg, seed=head_dim + splits)
    for u in (0, 1, 2, 4, 5, 6):            # unit 3 never arrives
        p.cond(u)
        if u not in (5,):                   # unit 5 keeps only its conditioning rows
            if u != 6:
                p.commit(u)
    got, want = p.attend(1, 6, splits=splits)
    _check(got, want)
    # the same unit at the other layer, then a stressed query (logit std 4)
    got, want = p.attend(0, 6, splits=splits)
    _check(got, want)
    got, want = p.attend(0, 6, q_scale=_times4, splits=splits)
    check_stressed(got, want)
    p.close()


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
def test_single_unit_no_history_no_conditioning(head_dim):
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=head_dim, n_video=1, n_audio=0, n_cond=0, history_units=0)
    p = Pair(cfg)
    p.cond(0)
    got, want = p.attend(0, 0)
    # one key: its weight is 1, so out = v_new exactly (a bf16 value times 1, rounded to bf16)
    assert np.all(np.isfinite(got))
    assert np.array_equal(got, want), float(np.abs(got - want).max())
    p.close()


@pytest.mark.gpu
def test_wrapped_ring_many_tiles_and_determinism():
    """A ring that has wrapped (newest slot mid-buffer): two key runs per query."""
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=4, head_dim=128, n_video=200, n_audio=4, n_cond=16, history_units=5)
    p = Pair(cfg)
    for u in range(9):
        p.cond(u)
        p.commit(u)
    p.cond(9)
    got1, want = p.attend(0, 9, splits=0)
    _check(got1, want)
    got2, _ = p.attend(0, 9, splits=0)
    assert np.array_equal(got1, got2)            # same inputs, same launch: same bits
    p.close()


@pytest.mark.gpu
@pytest.mark.parametrize("splits,heads", [(12, 1), (3, 2)])
def test_long_history_items_merged_inside_the_kernel(splits, heads):
    """Long items (a 512-unit window, 1 024 key tiles per head) cut into many pieces,
    with at least 64 iterations per CTA: the cut items are merged inside the
    attention kernel (12 pieces also exceed the merge's register-held (max, sum)
    cache).  One query block, 256 rows."""
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=heads, head_dim=128, n_video=250, n_audio=6, n_cond=0, history_units=511)
    p = Pair(cfg, seed=23)
    for u in range(511):
        p.cond(u)
        p.commit(u)
    p.cond(511)
    got, want = p.attend(0, 511, splits=splits)
    _check(got, want)
    p.close()


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim,splits,slope", [(128, 0, 0.25), (128, 3, 0.25), (64, 0, 0.25), (128, 0, 4.0)])
def test_rising_scores_move_the_reference_max(head_dim, splits, slope):
    """Keys scaled by 1 + slope*u for unit u: a row's scores rise tile after tile.
    With slope 1/4 (scale 1 to 4) the P of a later tile against the earlier reference
    max often sums past 255 (the row then moves its reference to the row max) or
    exceeds 2^8 (the lazy move).  With slope 4 (scale up to 49) the scores climb by
    far more than 128 in log2 units, so a P left against an old reference would
    overflow to inf: only the check on the P sum, and the move it triggers, keep the
    output finite.  The tolerance is that of the other stressed-score tests."""
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=4, head_dim=head_dim, n_video=250, n_audio=6, n_cond=8, history_units=12)
    p = Pair(cfg, seed=31)
    scaled = lambda bits, f: orc.f64_to_bf16(orc.bf16_to_f64(bits) * f)
    for u in range(13):
        f = 1.0 + slope * u
        cs = (1, cfg.n_cond, cfg.n_heads, head_dim)
        k, v = scaled(p._bits(synth.KIND_COND_K, cs, u), f), p._bits(synth.KIND_COND_V, cs, u)
        assert ws.ws_cache_append(p.h, u, ws.WS_SEG_COND, to_dev(k), to_dev(v), check=False) == 0
        assert p.o.append(u, orc.SEG_COND, k, v) == 0
        if u < 12:
            ls = (1, cfg.n_query, cfg.n_heads, head_dim)
            k, v = scaled(p._bits(synth.KIND_COMMIT_K, ls, u), f), p._bits(synth.KIND_COMMIT_V, ls, u)
            assert ws.ws_cache_append(p.h, u, ws.WS_SEG_LATENT, to_dev(k), to_dev(v), check=False) == 0
            assert p.o.append(u, orc.SEG_LATENT, k, v) == 0
    got, want = p.attend(0, 12, splits=splits)
    check_stressed(got, want)
    p.close()
