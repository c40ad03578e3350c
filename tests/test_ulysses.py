"""The Ulysses head-sharded step (sequence shard -> head shard -> attention ->
sequence shard) with gloo ranks on the CPU.  Each rank's attention is the fp64
oracle over that rank's head shard of the cache, fed with the head slices of the
conditioning and commit data; the assembled output of every rank must equal,
bit for bit, the single-GPU oracle over all heads on that rank's rows (heads and
rows are independent in the definition, pinned by the oracle's R-split test)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from kv_cache_serving_ws_b200.ulysses import UlyssesPlan, head_bounds, head_slice, video_bounds


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CFG = dict(n_layers=2, n_heads=4, head_dim=8, n_video=11, n_audio=3, n_cond=2, history_units=2)
UNITS = [0, 1, 2, 3]           # units 0..2 committed history, unit 3 the query unit (ring of 3 wraps)


def _data():
    from kv_cache_serving_ws_b200 import synth
    c = CFG
    nq = c["n_video"] + c["n_audio"]
    cs = (c["n_layers"], c["n_cond"], c["n_heads"], c["head_dim"])
    ls = (c["n_layers"], nq, c["n_heads"], c["head_dim"])
    qs = (nq, c["n_heads"], c["head_dim"])
    key = lambda kind, u, layer=0: synth.stream_key(33, kind, u, layer)
    d = {"cond": {u: (synth.normal_tensor(key(synth.KIND_COND_K, u), cs), synth.normal_tensor(key(synth.KIND_COND_V, u), cs))
                  for u in UNITS},
         "commit": {u: (synth.normal_tensor(key(synth.KIND_COMMIT_K, u), ls),
                        synth.normal_tensor(key(synth.KIND_COMMIT_V, u), ls)) for u in UNITS[:-1]},
         "q": {l: tuple(synth.normal_tensor(key(k, UNITS[-1], l), qs)
                        for k in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW)) for l in range(c["n_layers"])}}
    return d


def _oracle_cache(n_heads, data, heads):
    from oracle import ws_oracle as orc
    c = dict(CFG)
    c["n_heads"] = n_heads
    cache = orc.UnitCache(orc.Config(**c))
    for u in UNITS:
        k, v = data["cond"][u]
        assert cache.append(u, orc.SEG_COND, k[:, :, heads], v[:, :, heads]) == orc.OK
        if u in data["commit"]:
            k, v = data["commit"][u]
            assert cache.append(u, orc.SEG_LATENT, k[:, :, heads], v[:, :, heads]) == orc.OK
    return cache


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    from kv_cache_serving_ws_b200.ulysses import UlyssesAttention
    from oracle import ws_oracle as orc
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        c = CFG
        data = _data()
        plan = UlyssesPlan(c["n_video"], c["n_audio"], c["n_heads"], c["head_dim"], world, rank)
        h0, h1 = head_bounds(c["n_heads"], world, rank)
        cache = _oracle_cache(h1 - h0, data, list(range(h0, h1)))     # this rank's pre-sharded history

        def attention_fn(layer, unit, qh, kh, vh):
            to_bits = lambda t: t.numpy().astype(np.uint16)
            st, out = cache.unit_attention(layer, unit, to_bits(qh), to_bits(kh), to_bits(vh))
            assert st == orc.OK
            return torch.from_numpy(out)

        ua = UlyssesAttention(plan, attention_fn)
        v0, v1 = video_bounds(c["n_video"], world, rank)
        rows = list(range(v0, v1)) + list(range(c["n_video"], c["n_video"] + c["n_audio"]))
        outs = []
        for layer in range(c["n_layers"]):
            qf, kf, vf = data["q"][layer]
            # the rank's sequence shard, as bf16 bit patterns carried in int64 tensors
            loc = [torch.from_numpy(t[rows].astype(np.int64)) for t in (qf, kf, vf)]
            out = ua(layer, UNITS[-1], *loc)
            assert out.shape == (len(rows), c["n_heads"], c["head_dim"])
            outs.append(out.numpy())
        q.put((rank, rows, outs))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_equals_single_rank_attention(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs)
    c = CFG
    data = _data()
    full = _oracle_cache(c["n_heads"], data, list(range(c["n_heads"])))
    want = []
    for layer in range(c["n_layers"]):
        st, o = full.unit_attention(layer, UNITS[-1], *data["q"][layer])
        assert st == 0
        want.append(o)
    covered = set()
    for rank, rows, outs in res:
        for layer in range(c["n_layers"]):
            assert np.array_equal(outs[layer], want[layer][rows]), (rank, layer)
        covered |= set(rows[: len(rows) - c["n_audio"]])
    assert covered == set(range(c["n_video"]))


def test_shard_bounds():
    assert [video_bounds(11, 4, r) for r in range(4)] == [(0, 3), (3, 6), (6, 9), (9, 11)]
    assert [video_bounds(3, 4, r) for r in range(4)] == [(0, 1), (1, 2), (2, 3), (3, 3)]
    assert head_bounds(40, 8, 7) == (35, 40)
    with pytest.raises(ValueError):
        head_bounds(40, 3, 0)
    with pytest.raises(ValueError):
        UlyssesPlan(920, 4, 40, 128, 3, 0)
    x = np.arange(2 * 3 * 4 * 2).reshape(2, 3, 4, 2)
    assert np.array_equal(head_slice(x, 4, 2, 1), x[:, :, 2:4, :])
