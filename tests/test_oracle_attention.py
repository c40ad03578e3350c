"""Pins of the oracle's attention and cache model against things other than itself:
brute-force full-sequence masked attention (pure Python loops), a torch float64 SDPA
witness, closed forms, softmax row sums, R-way splits, and the ring's closed form."""
import math
import os

import numpy as np
import pytest
import torch

from kv_cache_serving_ws_b200 import synth
from oracle import ws_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cfg(**kw):
    base = dict(n_layers=2, n_heads=2, head_dim=4, n_video=3, n_audio=1, n_cond=2, history_units=2)
    base.update(kw)
    return orc.Config(**base)


def _bits(seed, kind, shape, unit=0, layer=0, step=0):
    return synth.normal_tensor(synth.stream_key(seed, kind, unit, layer, step), shape)


def _fill(cache, cfg, units, seed=1, commit=True, skip_latent=()):
    """Append COND for every unit, and commit latents for all but the last (and not those in skip_latent)."""
    for u in units:
        cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
        assert cache.append(u, orc.SEG_COND, _bits(seed, synth.KIND_COND_K, cs, u),
                            _bits(seed, synth.KIND_COND_V, cs, u)) == orc.OK
        if commit and u != units[-1] and u not in skip_latent:
            ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
            assert cache.append(u, orc.SEG_LATENT, _bits(seed, synth.KIND_COMMIT_K, ls, u),
                                _bits(seed, synth.KIND_COMMIT_V, ls, u)) == orc.OK


# ------------------------------------------------------------ brute force --

def _brute_force(cfg, seq, q_unit, layer, q_rows):
    """Full-sequence attention by the definition, with pure-Python loops.

    seq: list of (unit, kind, k[D]..., v[D]...) for every token of every unit in
    arrival order, kind in {"cond", "latent"}.  The dense block-causal mask is
    M[i, j] = u(j) <= u(i) and u(j) >= u(i) - U.  Query rows are the latent tokens
    of q_unit.  Returns out[row][head][d].
    """
    U = cfg.history_units
    D = cfg.head_dim
    out = []
    for qi in q_rows:                             # qi: per-head query vectors of one latent token
        row = []
        for h in range(cfg.n_heads):
            logits, vals = [], []
            for (u, _kind, kvec, vvec) in seq:
                if u <= q_unit and u >= q_unit - U:
                    s = sum(qi[h][d] * kvec[h][d] for d in range(D)) / math.sqrt(D)
                    logits.append(s)
                    vals.append(vvec[h])
            m = max(logits)
            w = [math.exp(s - m) for s in logits]
            z = sum(w)
            row.append([sum(w[j] * vals[j][d] for j in range(len(w))) / z for d in range(D)])
        out.append(row)
    return np.array(out)


@pytest.mark.parametrize("U,units,q_unit_layer", [(2, [0, 1, 2, 3, 4], 1), (1, [0, 1, 2], 0),
                                                   (3, [0, 1], 1), (0, [5, 6], 0), (2, [0, 1, 3, 4], 1)])
def test_incremental_equals_full_recomputation(U, units, q_unit_layer):
    cfg = _cfg(history_units=U)
    cache = orc.UnitCache(cfg)
    _fill(cache, cfg, units)
    u = units[-1]
    layer = q_unit_layer
    qs = (cfg.n_query, cfg.n_heads, cfg.head_dim)
    q = _bits(1, synth.KIND_Q, qs, u, layer)
    kn = _bits(1, synth.KIND_K_NEW, qs, u, layer)
    vn = _bits(1, synth.KIND_V_NEW, qs, u, layer)
    st, out = cache.unit_attention(layer, u, q, kn, vn)
    assert st == orc.OK

    # independent full sequence: every unit's tokens, in arrival order
    seq = []
    for uu in units:
        cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
        ck = orc.bf16_to_f64(_bits(1, synth.KIND_COND_K, cs, uu))[layer]
        cv = orc.bf16_to_f64(_bits(1, synth.KIND_COND_V, cs, uu))[layer]
        seq += [(uu, "cond", ck[t], cv[t]) for t in range(cfg.n_cond)]
        if uu == u:
            lk, lv = orc.bf16_to_f64(kn), orc.bf16_to_f64(vn)
        else:
            ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
            lk = orc.bf16_to_f64(_bits(1, synth.KIND_COMMIT_K, ls, uu))[layer]
            lv = orc.bf16_to_f64(_bits(1, synth.KIND_COMMIT_V, ls, uu))[layer]
        seq += [(uu, "latent", lk[t], lv[t]) for t in range(cfg.n_query)]
    want = _brute_force(cfg, seq, u, layer, orc.bf16_to_f64(q))
    assert np.max(np.abs(out - want)) <= 1e-12


def test_torch_sdpa_witness_float64():
    cfg = _cfg(n_heads=3, head_dim=8, n_video=5, n_audio=2, n_cond=3, history_units=2)
    cache = orc.UnitCache(cfg)
    units = [0, 1, 2, 3]
    _fill(cache, cfg, units, seed=9)
    qs = (cfg.n_query, cfg.n_heads, cfg.head_dim)
    q = _bits(9, synth.KIND_Q, qs, 3)
    kn = _bits(9, synth.KIND_K_NEW, qs, 3)
    vn = _bits(9, synth.KIND_V_NEW, qs, 3)
    st, out = cache.unit_attention(0, 3, q, kn, vn)
    assert st == orc.OK
    # build the full sequence (including unit 0, which the mask must hide) and mask it in torch
    ks, vs, owner = [], [], []
    for uu in units:
        cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
        ks.append(orc.bf16_to_f64(_bits(9, synth.KIND_COND_K, cs, uu))[0])
        vs.append(orc.bf16_to_f64(_bits(9, synth.KIND_COND_V, cs, uu))[0])
        owner += [uu] * cfg.n_cond
        if uu == 3:
            ks.append(orc.bf16_to_f64(kn)); vs.append(orc.bf16_to_f64(vn))
        else:
            ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
            ks.append(orc.bf16_to_f64(_bits(9, synth.KIND_COMMIT_K, ls, uu))[0])
            vs.append(orc.bf16_to_f64(_bits(9, synth.KIND_COMMIT_V, ls, uu))[0])
        owner += [uu] * cfg.n_query
    K = torch.from_numpy(np.concatenate(ks)).permute(1, 0, 2)      # [H, Nk, D]
    V = torch.from_numpy(np.concatenate(vs)).permute(1, 0, 2)
    Q = torch.from_numpy(orc.bf16_to_f64(q)).permute(1, 0, 2)      # [H, Nq, D]
    owner = torch.tensor(owner)
    mask = (owner <= 3) & (owner >= 3 - cfg.history_units)
    mask = mask[None, None, :].expand(1, Q.shape[1], -1)
    ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], attn_mask=mask)[0]
    assert np.max(np.abs(out - ref.permute(1, 0, 2).numpy())) <= 1e-12


def _parse_closed_forms():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "attention_closed_form.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case "):
                cur = {"name": line[5:], "k": [], "v": []}
                cases.append(cur)
                continue
            tag, nums = line.split(":", 1)
            vals = [float(x) for x in nums.split()]
            if tag in ("k", "v"):
                cur[tag].append(vals)
            else:
                cur[tag] = vals
    return cases


def test_golden_closed_forms():
    cases = _parse_closed_forms()
    assert len(cases) >= 3
    for c in cases:
        q = np.array(c["q"])[None, None, :]
        k = np.array(c["k"])[:, None, :]
        v = np.array(c["v"])[:, None, :]
        out = orc.attention_rows(q, k, v)[0, 0]
        assert np.allclose(out, c["out"], rtol=0, atol=1e-14), (c["name"], out)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((7, 3, 16)) * 4
    k = rng.standard_normal((50, 3, 16))
    v = rng.standard_normal((50, 3, 16))
    _, p = orc.attention_rows(q, k, v, return_probs=True)
    assert np.max(np.abs(p.sum(-1) - 1.0)) <= 1e-12
    assert np.all(p >= 0)


@pytest.mark.parametrize("R", [2, 3, 7])
def test_r_split_rows_and_heads_bit_identical(R):
    cfg = _cfg(n_heads=7, head_dim=16, n_video=20, n_audio=3, n_cond=4, history_units=3)
    cache = orc.UnitCache(cfg)
    _fill(cache, cfg, [0, 1, 2, 3, 4], seed=2)
    qs = (cfg.n_query, cfg.n_heads, cfg.head_dim)
    q = _bits(2, synth.KIND_Q, qs, 4)
    kn = _bits(2, synth.KIND_K_NEW, qs, 4)
    vn = _bits(2, synth.KIND_V_NEW, qs, 4)
    st, full = cache.unit_attention(1, 4, q, kn, vn)
    assert st == orc.OK
    k, v, _ = cache.visible_kv(1, 4)
    qf = orc.bf16_to_f64(q)
    row_parts = np.array_split(np.arange(cfg.n_query), R)
    by_rows = np.concatenate([orc.attention_rows(qf[rp], k, v) for rp in row_parts], axis=0)
    assert np.array_equal(by_rows, full)
    head_parts = np.array_split(np.arange(cfg.n_heads), R)
    by_heads = np.concatenate([orc.attention_rows(qf[:, hp], k[:, hp], v[:, hp]) for hp in head_parts], axis=1)
    assert np.array_equal(by_heads, full)


def test_zero_query_gives_mean_of_visible_values():
    """q = 0 makes every logit 0, so out is the plain mean of the visible V rows:
    this pins the visible key set and its size (the window and the segments)."""
    cfg = _cfg(history_units=2)
    cache = orc.UnitCache(cfg)
    _fill(cache, cfg, [0, 1, 2, 3, 4], skip_latent=(2,))
    qs = (cfg.n_query, cfg.n_heads, cfg.head_dim)
    q = np.zeros(qs, np.uint16)
    kn = _bits(1, synth.KIND_K_NEW, qs, 4)
    vn = _bits(1, synth.KIND_V_NEW, qs, 4)
    st, out = cache.unit_attention(0, 4, q, kn, vn)
    assert st == orc.OK
    # visible: units 2, 3, 4; unit 2 has no committed latent
    cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
    ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
    rows = [orc.bf16_to_f64(_bits(1, synth.KIND_COND_V, cs, u))[0] for u in (2, 3, 4)]
    rows.append(orc.bf16_to_f64(_bits(1, synth.KIND_COMMIT_V, ls, 3))[0])
    rows.append(orc.bf16_to_f64(vn))
    allv = np.concatenate(rows)
    assert allv.shape[0] == 3 * cfg.n_cond + 2 * cfg.n_query
    want = allv.mean(axis=0)
    assert np.max(np.abs(out - want[None])) <= 1e-14


def test_constant_values_and_single_key():
    # all V rows equal c -> out = c
    rng = np.random.default_rng(1)
    q = rng.standard_normal((5, 2, 8))
    k = rng.standard_normal((30, 2, 8))
    v = np.full((30, 2, 8), 0.375)
    assert np.max(np.abs(orc.attention_rows(q, k, v) - 0.375)) <= 1e-15
    # the smallest cache: no conditioning, one latent token, no history -> out = v_new
    cfg = _cfg(n_video=1, n_audio=0, n_cond=0, history_units=0, n_layers=1)
    cache = orc.UnitCache(cfg)
    e = np.zeros((1, 0, cfg.n_heads, cfg.head_dim), np.uint16)
    assert cache.append(0, orc.SEG_COND, e, e) == orc.OK
    qs = (1, cfg.n_heads, cfg.head_dim)
    vn = _bits(4, synth.KIND_V_NEW, qs)
    st, out = cache.unit_attention(0, 0, _bits(4, synth.KIND_Q, qs), _bits(4, synth.KIND_K_NEW, qs), vn)
    assert st == orc.OK
    assert np.array_equal(out, orc.bf16_to_f64(vn))


def test_masked_units_do_not_leak():
    """Values far outside the window are huge; a mask error would show up at once."""
    cfg = _cfg(history_units=1)
    cache = orc.UnitCache(cfg)
    cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
    ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
    huge = np.full(cs, 0x4780, np.uint16)           # 65536
    huge_l = np.full(ls, 0x4780, np.uint16)
    small = np.full(cs, 0x3F80, np.uint16)          # 1
    small_l = np.full(ls, 0x3F80, np.uint16)
    assert cache.append(0, orc.SEG_COND, small, huge) == orc.OK
    assert cache.append(0, orc.SEG_LATENT, small_l, huge_l) == orc.OK
    for u in (1, 2):
        assert cache.append(u, orc.SEG_COND, small, small) == orc.OK
    assert cache.append(1, orc.SEG_LATENT, small_l, small_l) == orc.OK
    qs = (cfg.n_query, cfg.n_heads, cfg.head_dim)
    st, out = cache.unit_attention(1, 2, _bits(3, synth.KIND_Q, qs), np.full(qs, 0x3F80, np.uint16),
                                   np.full(qs, 0x3F80, np.uint16))
    assert st == orc.OK
    assert np.max(np.abs(out - 1.0)) <= 1e-15      # every visible value is 1


def test_ring_slot_table_closed_form():
    cfg = _cfg(history_units=3)                      # C = 4
    cache = orc.UnitCache(cfg)
    units = [0, 1, 2, 3, 4, 5, 7, 8, 9, 10, 13]
    _fill(cache, cfg, units, commit=False)
    C = cfg.slots
    want = [-1] * C
    for u in units:
        want[u % C] = u
    assert cache.slot_table() == want


def test_error_rules():
    cfg = _cfg(history_units=2)                      # C = 3
    cache = orc.UnitCache(cfg)
    qs = (cfg.n_query, cfg.n_heads, cfg.head_dim)
    z = np.zeros(qs, np.uint16)
    assert cache.unit_attention(0, 0, z, z, z)[0] == orc.ERR_NOT_READY   # nothing appended
    _fill(cache, cfg, [0, 1, 2, 3, 4], commit=False)
    cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
    ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
    zc, zl = np.zeros(cs, np.uint16), np.zeros(ls, np.uint16)
    assert cache.append(3, orc.SEG_COND, zc, zc) == orc.ERR_UNIT_ORDER
    assert cache.append(4, orc.SEG_COND, zc, zc) == orc.OK               # same unit again
    assert cache.append(1, orc.SEG_LATENT, zl, zl) == orc.ERR_EVICTED    # slot 1 now holds unit 4
    assert cache.append(2, orc.SEG_LATENT, zl, zl) == orc.OK
    assert cache.append(5, orc.SEG_LATENT, zl, zl) == orc.ERR_NOT_READY
    assert cache.unit_attention(0, 3, z, z, z)[0] == orc.ERR_UNIT_ORDER
    assert cache.unit_attention(0, 5, z, z, z)[0] == orc.ERR_NOT_READY
    assert cache.unit_attention(2, 4, z, z, z)[0] == orc.ERR_ARG         # layer out of range
    assert cache.read(0, 3, orc.SEG_LATENT)[0] == orc.ERR_NOT_READY
    assert cache.read(0, 0, orc.SEG_COND)[0] == orc.ERR_EVICTED
    assert cache.read(0, 4, orc.SEG_COND)[0] == orc.OK
    assert cache.append(-1, orc.SEG_COND, zc, zc) == orc.ERR_ARG


@pytest.mark.parametrize("U,n_prior,n_units", [(3, 0, 4), (5, 2, 4), (4, 1, 3), (2, 3, 1), (2, 3, 3), (0, 1, 3)])
def test_prefill_equals_full_recomputation_per_query_unit(U, n_prior, n_units):
    """A multi-unit query: every query unit's rows against the dense block-causal
    mask over the whole sequence (pure-Python brute force)."""
    cfg = _cfg(history_units=U)
    cache = orc.UnitCache(cfg)
    prior = list(range(n_prior))
    _fill(cache, cfg, prior + [n_prior], commit=True)           # committed history; unit n_prior: COND only
    qunits = list(range(n_prior, n_prior + n_units))
    for u in qunits[1:]:
        cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
        assert cache.append(u, orc.SEG_COND, _bits(1, synth.KIND_COND_K, cs, u),
                            _bits(1, synth.KIND_COND_V, cs, u)) == orc.OK
    layer = 1
    qs = (n_units, cfg.n_query, cfg.n_heads, cfg.head_dim)
    q = _bits(6, synth.KIND_Q, qs, n_prior, layer)
    kn = _bits(6, synth.KIND_K_NEW, qs, n_prior, layer)
    vn = _bits(6, synth.KIND_V_NEW, qs, n_prior, layer)
    st, out = cache.prefill_attention(layer, n_prior, n_units, q, kn, vn)
    # a unit inside some query window is gone once a later unit took its slot
    # (slot reuse after C = U + 1 units): a query unit itself, or a prior unit
    # of the first query unit's window
    u_last = n_prior + n_units - 1
    gone = n_units > cfg.slots or any(u + cfg.slots <= u_last for u in prior if u >= n_prior - U)
    if gone:
        assert st == orc.ERR_EVICTED
        return
    assert st == orc.OK
    seq = []
    for uu in prior + qunits:
        cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
        ck = orc.bf16_to_f64(_bits(1, synth.KIND_COND_K, cs, uu))[layer]
        cv = orc.bf16_to_f64(_bits(1, synth.KIND_COND_V, cs, uu))[layer]
        seq += [(uu, "cond", ck[t], cv[t]) for t in range(cfg.n_cond)]
        if uu in qunits:
            j = uu - n_prior
            lk, lv = orc.bf16_to_f64(kn[j]), orc.bf16_to_f64(vn[j])
        else:
            ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
            lk = orc.bf16_to_f64(_bits(1, synth.KIND_COMMIT_K, ls, uu))[layer]
            lv = orc.bf16_to_f64(_bits(1, synth.KIND_COMMIT_V, ls, uu))[layer]
        seq += [(uu, "latent", lk[t], lv[t]) for t in range(cfg.n_query)]
    for j, uq in enumerate(qunits):
        want = _brute_force(cfg, seq, uq, layer, orc.bf16_to_f64(q[j]))
        assert np.max(np.abs(out[j] - want)) <= 1e-12, uq


def test_prefill_error_rules():
    cfg = _cfg(history_units=3)                                  # C = 4
    cache = orc.UnitCache(cfg)
    _fill(cache, cfg, [0, 1, 2, 3], commit=False)
    qs = lambda n: np.zeros((n, cfg.n_query, cfg.n_heads, cfg.head_dim), np.uint16)
    assert cache.prefill_attention(0, 0, 4, qs(4), qs(4), qs(4))[0] == orc.OK           # from scratch
    assert cache.prefill_attention(0, 1, 3, qs(3), qs(3), qs(3))[0] == orc.OK           # unit 0 still resident
    assert cache.prefill_attention(0, 2, 3, qs(3), qs(3), qs(3))[0] == orc.ERR_NOT_READY # unit 4 not there yet
    assert cache.prefill_attention(0, 1, 2, qs(2), qs(2), qs(2))[0] == orc.ERR_UNIT_ORDER
    assert cache.prefill_attention(0, 1, 3, qs(4), qs(3), qs(3))[0] == orc.ERR_ARG       # shape
    assert cache.prefill_attention(0, 0, 65, qs(65), qs(65), qs(65))[0] == orc.ERR_UNSUPPORTED
    _fill(cache, cfg, [4], commit=False)                         # unit 4 takes unit 0's slot
    assert cache.prefill_attention(0, 1, 4, qs(4), qs(4), qs(4))[0] == orc.ERR_EVICTED   # 0 in unit 1's window
    assert cache.prefill_attention(0, 3, 2, qs(2), qs(2), qs(2))[0] == orc.ERR_EVICTED   # 0 in unit 3's window
    assert cache.prefill_attention(0, 4, 1, qs(1), qs(1), qs(1))[0] == orc.OK            # window 1..4
    assert cache.prefill_attention(0, 0, 5, qs(5), qs(5), qs(5))[0] == orc.ERR_EVICTED   # query unit 0 gone


# ------------------------------------------------------------- sessions --

def _session_seq(cfg, seed, units, layer, current=None):
    """Token sequence of one session for the brute force: committed units, and the
    query units' latent rows from `current` = {unit: (k_new, v_new)}."""
    seq = []
    for uu in units:
        cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
        ck = orc.bf16_to_f64(_bits(seed, synth.KIND_COND_K, cs, uu))[layer]
        cv = orc.bf16_to_f64(_bits(seed, synth.KIND_COND_V, cs, uu))[layer]
        seq += [(uu, "cond", ck[t], cv[t]) for t in range(cfg.n_cond)]
        if current and uu in current:
            lk, lv = (orc.bf16_to_f64(a) for a in current[uu])
        else:
            ls = (cfg.n_layers, cfg.n_query, cfg.n_heads, cfg.head_dim)
            lk = orc.bf16_to_f64(_bits(seed, synth.KIND_COMMIT_K, ls, uu))[layer]
            lv = orc.bf16_to_f64(_bits(seed, synth.KIND_COMMIT_V, ls, uu))[layer]
        seq += [(uu, "latent", lk[t], lv[t]) for t in range(cfg.n_query)]
    return seq


def test_sessions_each_see_only_their_own_window():
    """Three sessions at different points of their streams, batched in one call
    (one streaming unit, one two-unit prefill, one streaming unit after a ring
    wrap): every query unit equals the brute force over its own session's tokens."""
    cfg = _cfg(history_units=2)                                  # C = 3
    pool = orc.SessionPool(cfg, 4)
    seeds = {0: 11, 1: 12, 2: 13}
    hist = {0: list(range(0, 7)), 1: [0], 2: [40, 41]}           # session 0 wrapped twice
    for s, units in hist.items():
        _fill(pool.sessions[s], cfg, units, seed=seeds[s])
    cs = (cfg.n_layers, cfg.n_cond, cfg.n_heads, cfg.head_dim)
    assert pool.sessions[1].append(1, orc.SEG_COND, _bits(12, synth.KIND_COND_K, cs, 1),
                                   _bits(12, synth.KIND_COND_V, cs, 1)) == orc.OK
    sessions, units = [2, 1, 1, 0], [41, 0, 1, 6]
    layer = 1
    qs = (4, cfg.n_query, cfg.n_heads, cfg.head_dim)
    q, kn, vn = (_bits(9, kind, qs, 0, layer) for kind in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
    st, out = pool.session_attention(layer, sessions, units, q, kn, vn)
    assert st == orc.OK and out.shape == (4, cfg.n_query, cfg.n_heads, cfg.head_dim)
    for s in (0, 1, 2):
        js = [j for j in range(4) if sessions[j] == s]
        mine = {units[j]: (kn[j], vn[j]) for j in js}
        every = sorted(set(hist[s]) | set(mine))
        seq = _session_seq(cfg, seeds[s], every, layer, current=mine)
        for j in js:
            want = _brute_force(cfg, seq, units[j], layer, orc.bf16_to_f64(q[j]))
            assert np.max(np.abs(out[j] - want)) <= 1e-12, (s, units[j])
    # session 3 was never touched; the others' bookkeeping is their own
    assert pool.sessions[3].slot_table() == [-1, -1, -1]
    assert pool.sessions[0].slot_table() == [6, 4, 5]
    assert pool.sessions[2].slot_table() == [-1, 40, 41]


def test_sessions_batch_equals_separate_calls_bit_for_bit():
    """Routing pin: the batched call gives exactly what each session's own call gives
    (rows are independent in the definition)."""
    cfg = _cfg(history_units=3)
    a, b = orc.SessionPool(cfg, 3), orc.SessionPool(cfg, 3)
    for pool in (a, b):
        for s in range(3):
            _fill(pool.sessions[s], cfg, list(range(s, s + 4 + s)), seed=20 + s)
    units = [s + 3 + s for s in range(3)]
    qs = (3, cfg.n_query, cfg.n_heads, cfg.head_dim)
    q, kn, vn = (_bits(5, kind, qs) for kind in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
    st, out = a.session_attention(0, [0, 1, 2], units, q, kn, vn)
    assert st == orc.OK
    for s in range(3):
        st1, o1 = b.sessions[s].unit_attention(0, units[s], q[s], kn[s], vn[s])
        assert st1 == orc.OK and np.array_equal(o1, out[s])


def test_session_error_rules_and_reset():
    cfg = _cfg(history_units=3)                                  # C = 4
    pool = orc.SessionPool(cfg, 3)
    _fill(pool.sessions[0], cfg, [0, 1, 2], commit=False)
    _fill(pool.sessions[1], cfg, [5], commit=False)
    z = lambda n: np.zeros((n, cfg.n_query, cfg.n_heads, cfg.head_dim), np.uint16)
    call = lambda ss, uu: pool.session_attention(0, ss, uu, z(len(ss)), z(len(ss)), z(len(ss)))[0]
    assert call([0, 1], [2, 5]) == orc.OK
    assert call([1, 0], [5, 2]) == orc.OK                        # any session order
    assert call([0, 1, 0], [2, 5, 2]) == orc.ERR_ARG             # a session in two stretches
    assert call([0, 0], [1, 1]) == orc.ERR_ARG                   # same unit twice
    assert call([0, 0], [0, 2]) == orc.ERR_ARG                   # not consecutive
    assert call([0, 3], [2, 0]) == orc.ERR_ARG                   # no such session
    assert call([0, 1], [2, -1]) == orc.ERR_ARG
    assert call([0, 2], [2, 0]) == orc.ERR_NOT_READY             # session 2 empty
    assert call([1, 0], [5, 1]) == orc.ERR_UNIT_ORDER            # session 0's newest is 2
    assert call([0, 0, 0], [0, 1, 2]) == orc.OK                  # a prefill stretch
    assert call([2, 0], [0, 1]) == orc.ERR_NOT_READY             # first failing stretch decides
    assert call([0] * 65, list(range(65))) == orc.ERR_UNSUPPORTED
    _fill(pool.sessions[0], cfg, [3, 4], commit=False)           # unit 4 takes unit 0's slot
    assert call([0, 0, 0, 0], [1, 2, 3, 4]) == orc.ERR_EVICTED
    assert pool.reset(0) == orc.OK and pool.reset(3) == orc.ERR_ARG
    assert pool.sessions[0].slot_table() == [-1] * 4
    assert call([0], [4]) == orc.ERR_NOT_READY
    _fill(pool.sessions[0], cfg, [100], commit=False)            # a new conversation at any unit index
    assert call([0, 1], [100, 5]) == orc.OK
