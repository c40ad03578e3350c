"""CPU checks of the C-ABI library: it loads, exports every symbol its headers
declare, validates arguments on the host before touching the GPU, and its
visible-row planner agrees with the oracle's cache model."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from kv_cache_serving_ws_b200 import native as ws
from oracle import ws_oracle as orc


def _exports(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    return {line.split()[-1] for line in out.splitlines() if line.strip()}


def test_library_exports_every_declared_symbol():
    declared = ws.header_symbols()
    assert len(declared) >= 12
    exported = _exports(ws.LIB_PATH)
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    lib = ws.lib()
    for s in declared:
        assert hasattr(lib, s)


def test_synth_library_exports_its_symbol():
    declared = ws.header_symbols(os.path.join(ws.ROOT, "include", "ws_synth.h"))
    assert declared == ["ws_synth_fill_normal_bf16"]
    assert set(declared) <= _exports(ws.SYNTH_PATH)


def test_status_strings():
    for code in range(-9, 1):
        assert ws.status_string(code) not in ("", "unknown status")
    assert ws.status_string(-100) == "unknown status"


def test_host_validation_without_gpu():
    lib = ws.lib()
    cfg = ws.make_config(1, 8, 64, 252, 8, 64, 4)
    h = ctypes.c_void_p()
    assert lib.ws_cache_create(None, ctypes.byref(cfg), None) == ws.WS_ERR_ARG
    assert lib.ws_cache_create(ctypes.byref(h), None, None) == ws.WS_ERR_ARG
    for bad in (dict(n_layers=0), dict(n_heads=0), dict(n_video=0, n_audio=0), dict(n_cond=-1),
                dict(history_units=-1), dict(head_dim=0)):
        c = ws.make_config(**{**dict(n_layers=1, n_heads=8, head_dim=64, n_video=252, n_audio=8, n_cond=64,
                                     history_units=4), **bad})
        assert lib.ws_cache_create(ctypes.byref(h), ctypes.byref(c), None) == ws.WS_ERR_ARG, bad
    c = ws.make_config(1, 8, 96, 252, 8, 64, 4)
    assert lib.ws_cache_create(ctypes.byref(h), ctypes.byref(c), None) == ws.WS_ERR_UNSUPPORTED
    # huge ring: C*T past 2^31 rows
    c = ws.make_config(1, 1, 64, 1 << 20, 0, 0, 4096)
    assert lib.ws_cache_create(ctypes.byref(h), ctypes.byref(c), None) == ws.WS_ERR_ARG
    # calls on a NULL handle
    assert lib.ws_cache_append(None, 0, 0, 16, 16, None) == ws.WS_ERR_ARG
    assert lib.ws_unit_attention(None, 0, 0, 16, 16, 16, 16, None) == ws.WS_ERR_ARG
    assert lib.ws_cache_read(None, 0, 0, 0, 16, 16, None) == ws.WS_ERR_ARG
    assert lib.ws_sync(None, None) == ws.WS_ERR_ARG
    assert lib.ws_cache_set_splits(None, 1) == ws.WS_ERR_ARG
    assert lib.ws_cache_destroy(None) == ws.WS_OK
    # Euler: sizes and pointers are checked before any launch
    assert lib.ws_flow_step(None, None, ctypes.c_float(0.25), 0, None) == ws.WS_OK
    assert lib.ws_flow_step(None, None, ctypes.c_float(0.25), -1, None) == ws.WS_ERR_ARG
    assert lib.ws_flow_step(None, 16, ctypes.c_float(0.25), 8, None) == ws.WS_ERR_ARG
    assert lib.ws_flow_step(18, 16, ctypes.c_float(0.25), 8, None) == ws.WS_ERR_ALIGN
    assert lib.ws_flow_step(16, 24, ctypes.c_float(0.25), 8, None) == ws.WS_ERR_ALIGN


def _oracle_history(rng, cfg, n_ops):
    """A random history: new units with gaps, re-appends, commits of random resident units."""
    cache = orc.UnitCache(cfg)
    cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
    ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
    zc, zl = np.zeros(cs, np.uint16), np.zeros(ls, np.uint16)
    u = int(rng.integers(0, 50))
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.55:
            u += int(rng.choice([1, 1, 1, 2, 3]))
            assert cache.append(u, orc.SEG_COND, zc, zc) == orc.OK
        elif r < 0.9 and cache.newest >= 0:
            uu = cache.newest - int(rng.integers(0, cfg.history_units + 1))
            cache.append(uu, orc.SEG_LATENT, zl, zl)
        elif cache.newest >= 0:
            layer = int(rng.integers(0, cfg.n_layers))
            qs = (cfg.n_query, cfg.n_heads, cfg.head_dim)
            z = np.zeros(qs, np.uint16)
            assert cache.unit_attention(layer, cache.newest, z, z, z, rows=[], heads=[])[0] == orc.OK
    return cache


@pytest.mark.parametrize("seed", range(12))
def test_planner_matches_oracle_visible_keys(seed):
    rng = np.random.default_rng(seed)
    cfg = orc.Config(n_layers=3, n_heads=1, head_dim=4, n_video=int(rng.integers(1, 6)),
                     n_audio=int(rng.integers(0, 3)), n_cond=int(rng.integers(0, 4)),
                     history_units=int(rng.integers(0, 7)))
    cache = _oracle_history(rng, cfg, 40)
    unit = cache.newest
    C, T, L = cfg.slots, cfg.tokens_per_unit, cfg.n_layers
    slot_unit = cache.slot_table()
    for layer in range(L):
        ready = []
        for s in range(C):
            for l in range(L):
                u = slot_unit[s]
                ready.append(u >= 0 and u in cache.units and l in cache.units[u].lat_k)
        wcfg = ws.make_config(cfg.n_layers, cfg.n_heads, cfg.head_dim, cfg.n_video, cfg.n_audio, cfg.n_cond,
                              cfg.history_units)
        st, runs = ws.ws_plan_visible(wcfg, slot_unit, ready, layer, unit)
        assert st == ws.WS_OK
        got = []
        for b, n in runs:
            for row in range(b, b + n):
                s, t = divmod(row, T)
                got.append((slot_unit[s], "cond" if t < cfg.n_cond else "latent", t))
        # oracle: visible units and which of their segments exist (the query unit's latent always does)
        want = []
        for u in cache.visible_units(unit):
            want += [(u, "cond", t) for t in range(cfg.n_cond)]
            if u == unit or layer in cache.units[u].lat_k:
                want += [(u, "latent", cfg.n_cond + t) for t in range(cfg.n_query)]
        assert sorted(got) == sorted(want)
        # runs are maximal: consecutive runs never touch
        for (b0, n0), (b1, _) in zip(runs, runs[1:]):
            assert b0 + n0 < b1


def test_planner_reports_too_many_runs():
    cfg = ws.make_config(1, 1, 64, 1, 0, 1, 9)
    slot_unit = list(range(10))
    st, _ = ws.ws_plan_visible(cfg, slot_unit, [0] * 10, 0, 9, max_runs=3)
    assert st == ws.WS_ERR_UNSUPPORTED
    st, runs = ws.ws_plan_visible(cfg, slot_unit, [0] * 10, 0, 9)
    # units 0..8 contribute their conditioning row only; unit 9 (the query's own) both rows
    assert st == ws.WS_OK and runs == [(2 * s, 1) for s in range(9)] + [(18, 2)]
