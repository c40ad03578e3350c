"""The unit program (one CUDA graph per unit) against the direct calls and the oracle.

The program records the same entry points the direct path calls, so a unit
replayed from the graph must leave bit-identical outputs, latent and cache
bytes, and the same slot table; each unit's attention outputs and latent are
also checked against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, dev_f64, from_dev, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc

CFG = orc.Config(n_layers=2, n_heads=3, head_dim=64, n_video=130, n_audio=3, n_cond=5, history_units=3)
STEPS = 2
DT = 0.25
N_LAT = 4000


def bits(seed, kind, shape, unit, layer=0, step=0):
    return synth.normal_tensor(synth.stream_key(seed, kind, unit, layer, step), shape)


class UnitData:
    """Host bit patterns of one unit's inputs."""

    def __init__(self, seed, u):
        c = CFG
        cs = (c.n_layers, c.n_cond, c.n_heads, c.head_dim)
        ls = (c.n_layers, c.n_query, c.n_heads, c.head_dim)
        qs = (STEPS, c.n_layers, c.n_query, c.n_heads, c.head_dim)
        self.cond_k = bits(seed, synth.KIND_COND_K, cs, u)
        self.cond_v = bits(seed, synth.KIND_COND_V, cs, u)
        self.q = bits(seed, synth.KIND_Q, qs, u)
        self.k_new = bits(seed, synth.KIND_K_NEW, qs, u)
        self.v_new = bits(seed, synth.KIND_V_NEW, qs, u)
        self.commit_k = bits(seed, synth.KIND_COMMIT_K, ls, u)
        self.commit_v = bits(seed, synth.KIND_COMMIT_V, ls, u)
        self.vel = bits(seed, synth.KIND_VEL, (STEPS, N_LAT), u)
        self.x = bits(seed, synth.KIND_X, (N_LAT,), u)


def new_cache():
    c = CFG
    _, h = ws.ws_cache_create(ws.make_config(c.n_layers, c.n_heads, c.head_dim, c.n_video, c.n_audio, c.n_cond,
                                             c.history_units))
    return h


def run_direct(h, u, d):
    c = CFG
    x = to_dev(d.x)
    out = torch.empty((STEPS, c.n_layers, c.n_query, c.n_heads, c.head_dim), dtype=torch.bfloat16, device="cuda")
    q, kn, vn, vel = to_dev(d.q), to_dev(d.k_new), to_dev(d.v_new), to_dev(d.vel)
    ws.ws_cache_append(h, u, ws.WS_SEG_COND, to_dev(d.cond_k), to_dev(d.cond_v))
    for s in range(STEPS):
        for l in range(c.n_layers):
            ws.ws_unit_attention(h, l, u, q[s, l], kn[s, l], vn[s, l], out[s, l])
        ws.ws_flow_step(x, vel[s], DT)
    ws.ws_cache_append(h, u, ws.WS_SEG_LATENT, to_dev(d.commit_k), to_dev(d.commit_v))
    torch.cuda.synchronize()
    return out, x


class Program:
    """Fixed device buffers of a unit program, refilled per unit."""

    def __init__(self, h, session=0):
        c = CFG
        e = lambda *s: torch.empty(s, dtype=torch.bfloat16, device="cuda")
        self.cond_k = e(c.n_layers, c.n_cond, c.n_heads, c.head_dim)
        self.cond_v = e(c.n_layers, c.n_cond, c.n_heads, c.head_dim)
        self.q = e(STEPS, c.n_layers, c.n_query, c.n_heads, c.head_dim)
        self.k_new, self.v_new, self.out = e(*self.q.shape), e(*self.q.shape), e(*self.q.shape)
        self.commit_k = e(c.n_layers, c.n_query, c.n_heads, c.head_dim)
        self.commit_v = e(*self.commit_k.shape)
        self.vel = e(STEPS, N_LAT)
        self.x = e(N_LAT)
        _, self.g = ws.ws_unit_graph_create(h, STEPS, DT, self.cond_k, self.cond_v, self.q, self.k_new, self.v_new,
                                            self.out, self.x, self.vel, self.commit_k, self.commit_v,
                                            session=session)

    def load(self, d):
        for name in ("cond_k", "cond_v", "q", "k_new", "v_new", "commit_k", "commit_v", "vel", "x"):
            getattr(self, name).copy_(to_dev(getattr(d, name)))

    def close(self):
        ws.ws_unit_graph_destroy(self.g)


def cache_bytes(h, units):
    c = CFG
    got = []
    for u in units:
        for l in range(c.n_layers):
            for seg, n in ((ws.WS_SEG_COND, c.n_cond), (ws.WS_SEG_LATENT, c.n_query)):
                k = torch.empty((n, c.n_heads, c.head_dim), dtype=torch.bfloat16, device="cuda")
                v = torch.empty_like(k)
                ws.ws_cache_read(h, l, u, seg, k, v)
                got.append(from_dev(k))
                got.append(from_dev(v))
    torch.cuda.synchronize()
    return got


@pytest.mark.gpu
def test_unit_program_matches_direct_calls_and_oracle():
    """Units 0..9 (ring of 4 slots wraps twice): graph == direct, bit for bit; both within
    tolerance of the oracle; after the window fills, every unit updates the graph in place."""
    require_gpu()
    seed = 77
    h_direct, h_graph = new_cache(), new_cache()
    prog = Program(h_graph)
    oc = orc.UnitCache(CFG)
    c = CFG
    for u in range(10):
        d = UnitData(seed, u)
        out_d, x_d = run_direct(h_direct, u, d)
        prog.load(d)
        ws.ws_unit_graph_launch(prog.g, u)
        torch.cuda.synchronize()
        assert ws.ws_sync(h_graph, check=False) == ws.WS_OK
        assert ws.ws_sync(h_direct, check=False) == ws.WS_OK
        assert np.array_equal(from_dev(prog.out), from_dev(out_d)), u
        assert np.array_equal(from_dev(prog.x), from_dev(x_d)), u
        assert ws.ws_cache_slot_table(h_graph) == ws.ws_cache_slot_table(h_direct)

        # oracle: the same unit, step by step
        assert oc.append(u, orc.SEG_COND, d.cond_k, d.cond_v) == orc.OK
        x = d.x
        for s in range(STEPS):
            for l in range(c.n_layers):
                st, want = oc.unit_attention(l, u, d.q[s, l], d.k_new[s, l], d.v_new[s, l])
                assert st == orc.OK
                err = np.abs(dev_f64(prog.out[s, l]) - want)
                assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (u, s, l, float(err.max()))
            x = orc.euler_step(x, d.vel[s], DT)
        assert oc.append(u, orc.SEG_LATENT, d.commit_k, d.commit_v) == orc.OK
        assert np.array_equal(from_dev(prog.x), x), u
        assert ws.ws_cache_slot_table(h_graph) == oc.slot_table()

    resident = [u for u in oc.slot_table() if u >= 0]
    for a, b in zip(cache_bytes(h_graph, resident), cache_bytes(h_direct, resident)):
        assert np.array_equal(a, b)
    stats = ws.ws_unit_graph_get_stats(prog.g)
    assert stats["launches"] == 10
    assert stats["nodes"] >= 1 + STEPS * c.n_layers * 2 + STEPS + 1
    # units 3..9 see full windows of identical structure: recorded graphs differ in parameters only
    assert stats["updates"] >= 6, stats
    prog.close()
    ws.ws_cache_destroy(h_direct)
    ws.ws_cache_destroy(h_graph)


@pytest.mark.gpu
def test_unit_program_errors_leave_the_cache_unchanged():
    require_gpu()
    h = new_cache()
    prog = Program(h)
    d = UnitData(5, 0)
    prog.load(d)
    ws.ws_unit_graph_launch(prog.g, 0)
    ws.ws_unit_graph_launch(prog.g, 1)
    torch.cuda.synchronize()
    table = ws.ws_cache_slot_table(h)
    info = ws.ws_cache_get_info(h)
    # a unit older than the newest one: refused before anything is recorded or launched
    assert ws.ws_unit_graph_launch(prog.g, 0, check=False) == ws.WS_ERR_UNIT_ORDER
    assert ws.ws_unit_graph_launch(prog.g, -1, check=False) == ws.WS_ERR_ARG
    assert ws.ws_cache_slot_table(h) == table
    assert ws.ws_cache_get_info(h)["newest_unit"] == info["newest_unit"] == 1
    assert ws.ws_unit_graph_get_stats(prog.g)["launches"] == 2
    # and the program keeps working
    ws.ws_unit_graph_launch(prog.g, 2)
    assert ws.ws_sync(h, check=False) == ws.WS_OK
    prog.close()
    ws.ws_cache_destroy(h)


@pytest.mark.gpu
def test_unit_program_rejects_bad_buffers():
    require_gpu()
    h = new_cache()
    prog = Program(h)
    z = prog.q
    bad = z.view(-1)[1:]                                   # 2-byte offset: not 16-byte aligned
    st, _ = ws.ws_unit_graph_create(h, STEPS, DT, prog.cond_k, prog.cond_v, bad, prog.k_new, prog.v_new, prog.out,
                                    prog.x, prog.vel, prog.commit_k, prog.commit_v, check=False)
    assert st == ws.WS_ERR_ALIGN
    st, _ = ws.ws_unit_graph_create(h, 0, DT, prog.cond_k, prog.cond_v, z, prog.k_new, prog.v_new, prog.out,
                                    prog.x, prog.vel, prog.commit_k, prog.commit_v, check=False)
    assert st == ws.WS_ERR_ARG
    prog.close()
    ws.ws_cache_destroy(h)


@pytest.mark.gpu
def test_unit_program_on_one_session_of_a_pool():
    """A program on session 1 of a two-session pool gives, bit for bit, what direct calls
    on a plain cache give; session 0's stream in the same pool is left as it was."""
    require_gpu()
    c = CFG
    h_direct = new_cache()
    _, pool = ws.ws_pool_create(ws.make_config(c.n_layers, c.n_heads, c.head_dim, c.n_video, c.n_audio, c.n_cond,
                                               c.history_units), 2)
    other = UnitData(999, 50)
    ws.ws_session_append(pool, 0, 50, ws.WS_SEG_COND, to_dev(other.cond_k), to_dev(other.cond_v))
    ws.ws_session_append(pool, 0, 50, ws.WS_SEG_LATENT, to_dev(other.commit_k), to_dev(other.commit_v))
    prog = Program(pool, session=1)
    for u in range(6):
        d = UnitData(31, u)
        out_d, x_d = run_direct(h_direct, u, d)
        prog.load(d)
        ws.ws_unit_graph_launch(prog.g, u)
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(prog.out), from_dev(out_d)), u
        assert np.array_equal(from_dev(prog.x), from_dev(x_d)), u
    assert ws.ws_session_slot_table(pool, 1) == ws.ws_cache_slot_table(h_direct)
    assert ws.ws_session_slot_table(pool, 0) == [-1, -1, 50, -1]
    for l in range(c.n_layers):
        k = torch.empty((c.n_query, c.n_heads, c.head_dim), dtype=torch.bfloat16, device="cuda")
        v = torch.empty_like(k)
        ws.ws_session_read(pool, 0, l, 50, ws.WS_SEG_LATENT, k, v)
        assert np.array_equal(from_dev(k), other.commit_k[l]) and np.array_equal(from_dev(v), other.commit_v[l])
    prog.close()
    ws.ws_cache_destroy(pool)
    ws.ws_cache_destroy(h_direct)
