"""Keys the query must not see never reach its output, even when they hold inf or
NaN: the rows of a partial key tile past the end of a visible run (stale latent rows
of a slot whose unit kept only its conditioning, a neighbouring session's rows, a
later unit of a prefill) are loaded with the tile, but the block-causal rule
("通义实验室发布 Wan-Streamer v0.2…", remio.ai, section
为什么端到端模型对级联式 AI 智能体构成挑战: a chunk sees only what is already
available) gives them no weight.  The oracle excludes them by definition, so the
GPU output must be finite and match it element by element."""
import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, dev_f64, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc

INF, NAN = np.uint16(0x7F80), np.uint16(0x7FC0)


def poisoned(bits, token_axis):
    """V-style poison: every third token row +inf, the next one NaN."""
    b = np.array(bits, copy=True)
    idx = [slice(None)] * b.ndim
    for t in range(b.shape[token_axis]):
        if t % 3 == 2:
            continue
        idx[token_axis] = t
        b[tuple(idx)] = INF if t % 3 == 0 else NAN
    return b


def nan_rows(bits, token_axis, every=5):
    """K-style poison: every `every`-th token row NaN."""
    b = np.array(bits, copy=True)
    idx = [slice(None)] * b.ndim
    for t in range(0, b.shape[token_axis], every):
        idx[token_axis] = t
        b[tuple(idx)] = NAN
    return b


def _check(got, want):
    assert np.all(np.isfinite(got)), "a non-finite value leaked from a key row the query cannot see"
    d = np.abs(got - want)
    assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (float(d.max()), float(d.mean()))


class Pair:
    """A GPU cache and the oracle's, fed the same bytes."""

    def __init__(self, cfg, seed):
        self.cfg, self.seed = cfg, seed
        self.o = orc.UnitCache(cfg)
        _, self.h = ws.ws_cache_create(ws.make_config(cfg.n_layers, cfg.n_heads, cfg.head_dim, cfg.n_video,
                                                      cfg.n_audio, cfg.n_cond, cfg.history_units))

    def bits(self, kind, shape, unit, layer=0):
        return synth.normal_tensor(synth.stream_key(self.seed, kind, unit, layer), shape)

    def append(self, u, seg, k, v):
        assert ws.ws_cache_append(self.h, u, seg, to_dev(k), to_dev(v), check=False) == 0
        assert self.o.append(u, seg, k, v) == 0

    def cond(self, u, poison=False):
        c = self.cfg
        s = (c.n_layers, c.n_cond, c.n_heads, c.head_dim)
        k, v = self.bits(synth.KIND_COND_K, s, u), self.bits(synth.KIND_COND_V, s, u)
        if poison:
            k, v = nan_rows(k, 1), poisoned(v, 1)
        self.append(u, orc.SEG_COND, k, v)

    def commit(self, u, poison=False):
        c = self.cfg
        s = (c.n_layers, c.n_query, c.n_heads, c.head_dim)
        k, v = self.bits(synth.KIND_COMMIT_K, s, u), self.bits(synth.KIND_COMMIT_V, s, u)
        if poison:
            k, v = nan_rows(k, 1), poisoned(v, 1)
        self.append(u, orc.SEG_LATENT, k, v)

    def attend(self, layer, u, splits):
        c = self.cfg
        s = (c.n_query, c.n_heads, c.head_dim)
        q, kn, vn = (self.bits(kind, s, u, layer) for kind in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
        ws.ws_cache_set_splits(self.h, splits)
        out = torch.empty(s, dtype=torch.bfloat16, device="cuda")
        assert ws.ws_unit_attention(self.h, layer, u, to_dev(q), to_dev(kn), to_dev(vn), out, check=False) == 0
        assert ws.ws_sync(self.h, check=False) == ws.WS_OK
        st, want = self.o.unit_attention(layer, u, q, kn, vn)
        assert st == 0
        return dev_f64(out), want

    def close(self):
        ws.ws_cache_destroy(self.h)


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("n_cond", [40, 48, 5])
@pytest.mark.parametrize("splits", [0, 3])
def test_stale_latent_rows_after_a_conditioning_only_slot(head_dim, n_cond, splits):
    """Ring of 4 slots, 124 latent tokens per unit.  Unit 0 commits poisoned K/V
    (NaN key rows, inf and NaN value rows); unit 4 takes its slot with a
    conditioning slice only, so the slot's latent rows still hold unit 0's poison.
    Unit 5 sees unit 4's conditioning rows and nothing after them: its run ends
    n_cond rows into a key tile (mid 16-key step for 40 and 5, on a step boundary
    for 48)."""
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=3, head_dim=head_dim, n_video=120, n_audio=4, n_cond=n_cond,
                     history_units=3)
    p = Pair(cfg, seed=101 + n_cond)
    for u in range(4):
        p.cond(u)
        p.commit(u, poison=(u == 0))
    p.cond(4)                      # slot 0: conditioning of unit 4, unit 0's poisoned latent rows after it
    p.cond(5)
    got, want = p.attend(0, 5, splits)
    _check(got, want)
    p.close()


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("splits", [0, 2])
def test_stale_latent_rows_after_a_multi_tile_run(head_dim, splits):
    """A run of a full slot and a conditioning-only slot (204 rows: the second tile
    ends 76 rows in), followed by the stale, poisoned latent rows of the evicted
    unit 1."""
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=head_dim, n_video=120, n_audio=4, n_cond=40,
                     history_units=3)
    p = Pair(cfg, seed=131)
    for u in range(5):
        p.cond(u)
        p.commit(u, poison=(u == 1))
    p.cond(5)                      # unit 5 evicts unit 1 from slot 1 and is never committed
    p.cond(6)
    got, want = p.attend(0, 6, splits)
    _check(got, want)
    p.close()


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("splits", [0, 4])
def test_neighbouring_session_rows_are_not_seen(head_dim, splits):
    """Two sessions in one pool.  Session 0's window ends at the last row of its
    rows (a partial tile: 3 x 164 rows), and session 1's first slot, right after,
    holds poisoned conditioning and latent rows.  Session 0 alone, and session 0
    batched with a clean query of session 1's later unit, must match the oracle."""
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=head_dim, n_video=120, n_audio=4, n_cond=40,
                     history_units=2)
    o = orc.SessionPool(cfg, 2)
    _, h = ws.ws_pool_create(ws.make_config(1, 2, head_dim, 120, 4, 40, 2), 2)
    key = lambda s, kind, u, layer=0: synth.stream_key(151 + 10 * s, kind, u, layer)
    cs, ls = (1, 40, 2, head_dim), (1, 124, 2, head_dim)

    def feed(s, u, commit, poison):
        ck, cv = synth.normal_tensor(key(s, synth.KIND_COND_K, u), cs), synth.normal_tensor(key(s, synth.KIND_COND_V, u), cs)
        if poison:
            ck, cv = nan_rows(ck, 1), poisoned(cv, 1)
        assert ws.ws_session_append(h, s, u, ws.WS_SEG_COND, to_dev(ck), to_dev(cv), check=False) == 0
        assert o.sessions[s].append(u, orc.SEG_COND, ck, cv) == 0
        if commit:
            lk, lv = synth.normal_tensor(key(s, synth.KIND_COMMIT_K, u), ls), synth.normal_tensor(key(s, synth.KIND_COMMIT_V, u), ls)
            if poison:
                lk, lv = nan_rows(lk, 1), poisoned(lv, 1)
            assert ws.ws_session_append(h, s, u, ws.WS_SEG_LATENT, to_dev(lk), to_dev(lv), check=False) == 0
            assert o.sessions[s].append(u, orc.SEG_LATENT, lk, lv) == 0

    for u in range(3):
        feed(0, u, commit=(u < 2), poison=False)     # session 0: units 0-2, unit 2 in its last slot
    feed(1, 0, commit=True, poison=True)             # session 1, slot 0: right after session 0's rows
    feed(1, 1, commit=False, poison=False)
    ws.ws_cache_set_splits(h, splits)
    for sessions, units in (([0], [2]), ([0, 1], [2, 1])):
        n = len(sessions)
        shape = (n, 124, 2, head_dim)
        q, kn, vn = (synth.normal_tensor(key(9, kind, n), shape)
                     for kind in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
        out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        assert ws.ws_session_attention(h, 0, sessions, units, to_dev(q), to_dev(kn), to_dev(vn), out,
                                       check=False) == 0
        assert ws.ws_sync(h, check=False) == ws.WS_OK
        st, want = o.session_attention(0, sessions, units, q, kn, vn)
        assert st == 0
        got = dev_f64(out)
        # session 1's unit 1 sees its own poisoned unit 0: only session 0's rows are checked
        _check(got[0], want[0])
    ws.ws_cache_destroy(h)


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("splits", [0, 3])
def test_prefill_earlier_units_do_not_see_a_poisoned_later_unit(head_dim, splits):
    """A prefill of units 0-3 from an empty ring.  Unit 3's conditioning slice is
    poisoned; query units 0-2 end their windows before it (unit 2's run ends 108
    rows into its last key tile, 4 rows before the poison), so their outputs must be
    finite and match the oracle."""
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=head_dim, n_video=120, n_audio=4, n_cond=40,
                     history_units=3)
    p = Pair(cfg, seed=171)
    for u in range(4):
        p.cond(u, poison=(u == 3))
    shape = (4, 124, 2, head_dim)
    q, kn, vn = (p.bits(kind, shape, 99) for kind in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
    ws.ws_cache_set_splits(p.h, splits)
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    assert ws.ws_prefill_attention(p.h, 0, 0, 4, to_dev(q), to_dev(kn), to_dev(vn), out, check=False) == 0
    assert ws.ws_sync(p.h, check=False) == ws.WS_OK
    st, want = p.o.prefill_attention(0, 0, 4, q, kn, vn)
    assert st == 0
    got = dev_f64(out)
    _check(got[:3], want[:3])
    p.close()
