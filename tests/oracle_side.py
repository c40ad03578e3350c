"""Oracle side of the workload tests: the fp64 oracle over a subset of heads and one layer."""
import numpy as np

from kv_cache_serving_ws_b200.workloads import Workload, gen_heads, key


def oracle_cache(w: Workload, layer: int, heads, step: int = 0, q_scale_bits=None):
    """Oracle side for a subset of heads and one layer: a UnitCache over those heads
    (heads are independent: the oracle's R-way head split is pinned bit-identical),
    filled with the same history, then the query unit's attention.  Returns
    (status, out [Nq, len(heads), D] float64)."""
    from oracle import ws_oracle as orc
    from kv_cache_serving_ws_b200.synth import KIND_COMMIT_K, KIND_COMMIT_V, KIND_COND_K, KIND_COND_V, \
        KIND_K_NEW, KIND_Q, KIND_V_NEW
    heads = list(heads)
    cfg = orc.Config(1, len(heads), w.head_dim, w.n_video, w.n_audio, w.n_cond, w.history_units)
    cache = orc.UnitCache(cfg)
    cs = (w.n_layers, w.n_cond, w.n_heads, w.head_dim)
    ls = (w.n_layers, w.n_query, w.n_heads, w.head_dim)
    for u in w.history() + [w.unit]:
        ck = gen_heads(key(w, KIND_COND_K, u), cs, heads, layer)[None]
        cv = gen_heads(key(w, KIND_COND_V, u), cs, heads, layer)[None]
        assert cache.append(u, orc.SEG_COND, ck, cv) == orc.OK
        if u != w.unit:
            lk = gen_heads(key(w, KIND_COMMIT_K, u), ls, heads, layer)[None]
            lv = gen_heads(key(w, KIND_COMMIT_V, u), ls, heads, layer)[None]
            assert cache.append(u, orc.SEG_LATENT, lk, lv) == orc.OK
    qs = (w.n_query, w.n_heads, w.head_dim)
    q = gen_heads(key(w, KIND_Q, w.unit, layer, step), qs, heads)
    if q_scale_bits is not None:
        q = q_scale_bits(q)
    kn = gen_heads(key(w, KIND_K_NEW, w.unit, layer, step), qs, heads)
    vn = gen_heads(key(w, KIND_V_NEW, w.unit, layer, step), qs, heads)
    return cache, q, kn, vn
