"""Concurrent sessions on the GPU vs the oracle's SessionPool: one pool allocation,
several independent rings, query units of several sessions in one attention launch;
status codes, slot tables and cache bytes identical to the oracle's."""
import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, dev_f64, from_dev, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc


class PoolPair:
    def __init__(self, cfg, n_sessions, seed):
        self.cfg, self.seed, self.n = cfg, seed, n_sessions
        self.o = orc.SessionPool(cfg, n_sessions)
        _, self.h = ws.ws_pool_create(ws.make_config(cfg.n_layers, cfg.n_heads, cfg.head_dim, cfg.n_video,
                                                     cfg.n_audio, cfg.n_cond, cfg.history_units), n_sessions)

    def bits(self, kind, shape, s, unit=0, layer=0):
        # every session draws its own stream: the seed differs per session
        return synth.normal_tensor(synth.stream_key(self.seed * 100 + s, kind, unit, layer), shape)

    def cond(self, s, u):
        c = self.cfg
        shape = (c.n_layers, c.n_cond, c.n_heads, c.head_dim)
        k, v = self.bits(synth.KIND_COND_K, shape, s, u), self.bits(synth.KIND_COND_V, shape, s, u)
        st_g = ws.ws_session_append(self.h, s, u, ws.WS_SEG_COND, to_dev(k), to_dev(v), check=False)
        st_o = self.o.sessions[s].append(u, orc.SEG_COND, k, v)
        assert st_g == st_o, (st_g, st_o)

    def commit(self, s, u):
        c = self.cfg
        shape = (c.n_layers, c.n_query, c.n_heads, c.head_dim)
        k, v = self.bits(synth.KIND_COMMIT_K, shape, s, u), self.bits(synth.KIND_COMMIT_V, shape, s, u)
        st_g = ws.ws_session_append(self.h, s, u, ws.WS_SEG_LATENT, to_dev(k), to_dev(v), check=False)
        st_o = self.o.sessions[s].append(u, orc.SEG_LATENT, k, v)
        assert st_g == st_o, (st_g, st_o)

    def stream(self, s, units):
        for u in units:
            self.cond(s, u)
            self.commit(s, u)

    def reset(self, s):
        assert ws.ws_session_reset(self.h, s, check=False) == self.o.reset(s)

    def attend(self, layer, sessions, units, splits=0, rows=None, heads=None, expect=orc.OK):
        c = self.cfg
        n = len(sessions)
        shape = (n, c.n_query, c.n_heads, c.head_dim)
        key = 7 * layer + 1000 * len(sessions) + sum(units)
        q = synth.normal_tensor(synth.stream_key(self.seed, synth.KIND_Q, key, layer), shape)
        kn = synth.normal_tensor(synth.stream_key(self.seed, synth.KIND_K_NEW, key, layer), shape)
        vn = synth.normal_tensor(synth.stream_key(self.seed, synth.KIND_V_NEW, key, layer), shape)
        ws.ws_cache_set_splits(self.h, splits)
        out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        st_g = ws.ws_session_attention(self.h, layer, sessions, units, to_dev(q), to_dev(kn), to_dev(vn), out,
                                       check=False)
        st_o, want = self.o.session_attention(layer, sessions, units, q, kn, vn, rows=rows, heads=heads)
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

    def check_tables(self):
        for s in range(self.n):
            assert ws.ws_session_slot_table(self.h, s) == self.o.sessions[s].slot_table(), s

    def close(self):
        ws.ws_cache_destroy(self.h)


@pytest.mark.gpu
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("splits", [0, 2])
def test_sessions_batched_in_one_launch(head_dim, splits):
    require_gpu()
    cfg = orc.Config(n_layers=2, n_heads=3, head_dim=head_dim, n_video=130, n_audio=3, n_cond=5, history_units=3)
    p = PoolPair(cfg, 4, seed=50 + head_dim)
    p.stream(0, range(0, 9))                 # wrapped twice
    p.cond(0, 9)
    p.stream(1, [0])                         # young session: window not full
    p.cond(1, 1)
    p.stream(2, range(200, 203))             # starts at unit 200
    p.cond(2, 203)
    p.check_tables()
    p.attend(1, [0, 1, 2], [9, 1, 203], splits=splits)
    p.attend(0, [2, 0], [203, 9], splits=splits)          # another layer, other order, session 1 left out
    p.cond(1, 2)
    p.attend(1, [1, 1, 0], [1, 2, 9], splits=splits)      # a two-unit prefill stretch beside a streaming unit
    p.check_tables()
    p.close()


@pytest.mark.gpu
def test_session_status_codes_match_the_oracle():
    require_gpu()
    cfg = orc.Config(n_layers=1, n_heads=2, head_dim=64, n_video=20, n_audio=0, n_cond=3, history_units=3)
    p = PoolPair(cfg, 3, seed=3)
    for u in range(3):
        p.cond(0, u)
    p.cond(1, 5)
    p.attend(0, [0, 1], [2, 5])
    p.attend(0, [0, 1, 0], [2, 5, 2], expect=orc.ERR_ARG)
    p.attend(0, [0, 0], [1, 1], expect=orc.ERR_ARG)
    p.attend(0, [0, 0], [0, 2], expect=orc.ERR_ARG)
    p.attend(0, [0, 3], [2, 0], expect=orc.ERR_ARG)
    p.attend(0, [0, 2], [2, 0], expect=orc.ERR_NOT_READY)
    p.attend(0, [1, 0], [5, 1], expect=orc.ERR_UNIT_ORDER)
    p.attend(0, [0, 0, 0], [0, 1, 2])
    p.attend(0, [2, 0], [0, 1], expect=orc.ERR_NOT_READY)
    p.cond(0, 3)
    p.cond(0, 4)                             # unit 4 takes unit 0's slot
    p.attend(0, [0, 0, 0, 0], [1, 2, 3, 4], expect=orc.ERR_EVICTED)
    p.reset(0)
    p.check_tables()
    p.attend(0, [0], [4], expect=orc.ERR_NOT_READY)
    p.cond(0, 100)                           # a new conversation at any unit index
    p.attend(0, [0, 1], [100, 5])
    zc = torch.zeros((cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
    assert ws.ws_session_append(p.h, 3, 0, ws.WS_SEG_COND, zc, zc, check=False) == ws.WS_ERR_ARG
    assert ws.ws_session_append(p.h, -1, 0, ws.WS_SEG_COND, zc, zc, check=False) == ws.WS_ERR_ARG
    assert ws.ws_session_reset(p.h, 3, check=False) == ws.WS_ERR_ARG
    p.close()


@pytest.mark.gpu
def test_sessions_do_not_touch_each_others_rows():
    """Cache bytes of every session read back bit for bit after interleaved appends,
    prefills and batched calls in the other sessions."""
    require_gpu()
    cfg = orc.Config(n_layers=2, n_heads=2, head_dim=64, n_video=30, n_audio=2, n_cond=4, history_units=2)
    p = PoolPair(cfg, 3, seed=9)
    p.stream(0, range(0, 5))
    p.stream(2, range(10, 12))
    p.cond(0, 5)
    p.cond(2, 12)
    p.attend(1, [0, 2], [5, 12])
    p.stream(1, range(0, 2))
    p.cond(1, 2)
    p.attend(0, [1], [2])
    for s in range(3):
        for u in p.o.sessions[s].slot_table():
            if u < 0:
                continue
            for layer in range(cfg.n_layers):
                for seg, n in ((ws.WS_SEG_COND, cfg.n_cond), (ws.WS_SEG_LATENT, cfg.n_query)):
                    st_o, k_o, v_o = p.o.sessions[s].read(layer, u, seg)
                    k = torch.empty((n, cfg.n_heads, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
                    v = torch.empty_like(k)
                    st_g = ws.ws_session_read(p.h, s, layer, u, seg, k, v, check=False)
                    assert st_g == st_o, (s, u, layer, seg)
                    if st_o == orc.OK:
                        assert np.array_equal(from_dev(k), k_o) and np.array_equal(from_dev(v), v_o)
    p.close()


@pytest.mark.gpu
def test_eight_sessions_at_v02_shapes_sampled():
    """Eight conversations of the 640x368 stream (8-unit windows, histories of 1..8
    units) in one launch: 7392 query rows x 40 heads.  The device generator fills the
    GPU side; the oracle sees three of the heads (heads are independent), sampled rows."""
    require_gpu()
    from kv_cache_serving_ws_b200.workloads import gen_heads
    H, D, Nv, Na, Nc, U = 40, 128, 920, 4, 32, 8
    Nq = Nv + Na
    heads = [0, 17, 39]
    _, h = ws.ws_pool_create(ws.make_config(1, H, D, Nv, Na, Nc, U), 8)
    pool = orc.SessionPool(orc.Config(1, len(heads), D, Nv, Na, Nc, U), 8)
    key = lambda s, kind, u: synth.stream_key(600 + s, kind, u, 0)
    cs, ls = (1, Nc, H, D), (1, Nq, H, D)
    ck, cv = (torch.empty(cs, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    lk, lv = (torch.empty(ls, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    units = []
    for s in range(8):
        first = 5 * s + 1
        hist = list(range(first, first + 1 + s))
        for u in hist + [hist[-1] + 1]:
            ws.synth_fill(ck, key(s, synth.KIND_COND_K, u))
            ws.synth_fill(cv, key(s, synth.KIND_COND_V, u))
            ws.ws_session_append(h, s, u, ws.WS_SEG_COND, ck, cv)
            assert pool.sessions[s].append(u, orc.SEG_COND, gen_heads(key(s, synth.KIND_COND_K, u), cs, heads, 0)[None],
                                           gen_heads(key(s, synth.KIND_COND_V, u), cs, heads, 0)[None]) == orc.OK
            if u in hist:
                ws.synth_fill(lk, key(s, synth.KIND_COMMIT_K, u))
                ws.synth_fill(lv, key(s, synth.KIND_COMMIT_V, u))
                ws.ws_session_append(h, s, u, ws.WS_SEG_LATENT, lk, lv)
                assert pool.sessions[s].append(
                    u, orc.SEG_LATENT, gen_heads(key(s, synth.KIND_COMMIT_K, u), ls, heads, 0)[None],
                    gen_heads(key(s, synth.KIND_COMMIT_V, u), ls, heads, 0)[None]) == orc.OK
        units.append(hist[-1] + 1)
    qs = (Nq, H, D)
    q, kn, vn = (torch.empty((8,) + qs, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    oq, okn, ovn = [], [], []
    for s in range(8):
        for t, o, kind in ((q, oq, synth.KIND_Q), (kn, okn, synth.KIND_K_NEW), (vn, ovn, synth.KIND_V_NEW)):
            ws.synth_fill(t[s], key(s, kind, units[s]))
            o.append(gen_heads(key(s, kind, units[s]), qs, heads))
    out = torch.empty_like(q)
    ws.ws_session_attention(h, 0, list(range(8)), units, q, kn, vn, out)
    assert ws.ws_sync(h, check=False) == ws.WS_OK
    rng = np.random.default_rng(4)
    rows = sorted(rng.choice(Nq, size=12, replace=False).tolist() + [0, Nq - 1])
    st, want = pool.session_attention(0, list(range(8)), units, np.stack(oq), np.stack(okn), np.stack(ovn), rows=rows)
    assert st == orc.OK
    got = dev_f64(out)[:, rows][:, :, heads]
    d = np.abs(got - want)
    assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (float(d.max()), float(d.mean()))
    ws.ws_cache_destroy(h)
