"""The Ulysses plumbing on a GPU with the library's attention: a one-rank NCCL
group (the exchanges are copies to self) must reproduce direct ws_unit_attention
calls bit for bit, with bf16 tensors, uneven video runs and audio rows, and match
the fp64 oracle over the same history.  More ranks need more GPUs; their exchange
logic is covered by the gloo tests."""
import os
import socket

import numpy as np
import pytest
import torch

from gpu_util import ATOL_MAX, ATOL_MEAN, dev_f64, from_dev, require_gpu, to_dev
from kv_cache_serving_ws_b200 import native as ws
from kv_cache_serving_ws_b200 import synth
from kv_cache_serving_ws_b200.ulysses import UlyssesAttention, UlyssesPlan, head_slice, library_attention_fn
from oracle import ws_oracle as orc


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.gpu
def test_one_rank_nccl_equals_direct_calls():
    require_gpu()
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        L, H, D, Nv, Na, Nc, U = 2, 4, 128, 131, 3, 5, 3
        Nq = Nv + Na
        cfg = ws.make_config(L, H, D, Nv, Na, Nc, U)
        _, h_direct = ws.ws_cache_create(cfg)
        _, h_rank = ws.ws_cache_create(cfg)
        oracle = orc.UnitCache(orc.Config(L, H, D, Nv, Na, Nc, U))
        key = lambda kind, u, layer=0: synth.stream_key(71, kind, u, layer)
        for u in range(5):
            cs, ls = (L, Nc, H, D), (L, Nq, H, D)
            ck, cv = synth.normal_tensor(key(synth.KIND_COND_K, u), cs), synth.normal_tensor(key(synth.KIND_COND_V, u), cs)
            for h in (h_direct, h_rank):
                ws.ws_cache_append(h, u, ws.WS_SEG_COND, to_dev(ck), to_dev(cv))
            assert oracle.append(u, orc.SEG_COND, ck, cv) == orc.OK
            if u < 4:
                lk = synth.normal_tensor(key(synth.KIND_COMMIT_K, u), ls)
                lv = synth.normal_tensor(key(synth.KIND_COMMIT_V, u), ls)
                ws.ws_cache_append(h_direct, u, ws.WS_SEG_LATENT, to_dev(lk), to_dev(lv))
                ws.ws_cache_append(h_rank, u, ws.WS_SEG_LATENT, to_dev(head_slice(lk, H, 1, 0)),
                                   to_dev(head_slice(lv, H, 1, 0)))
                assert oracle.append(u, orc.SEG_LATENT, lk, lv) == orc.OK
        ua = UlyssesAttention(UlyssesPlan(Nv, Na, H, D, 1, 0), library_attention_fn(h_rank))
        for layer in range(L):
            qs = (Nq, H, D)
            qb, knb, vnb = (synth.normal_tensor(key(k, 4, layer), qs)
                            for k in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
            q, kn, vn = to_dev(qb), to_dev(knb), to_dev(vnb)
            want = torch.empty_like(q)
            ws.ws_unit_attention(h_direct, layer, 4, q, kn, vn, want)
            got = ua(layer, 4, q, kn, vn)
            torch.cuda.synchronize()
            assert got.dtype == torch.bfloat16 and got.shape == want.shape
            assert np.array_equal(from_dev(got), from_dev(want)), layer
            st, ref = oracle.unit_attention(layer, 4, qb, knb, vnb)
            assert st == orc.OK
            d = np.abs(dev_f64(got) - ref)
            assert np.all(np.isfinite(dev_f64(got)))
            assert d.max() <= ATOL_MAX and d.mean() <= ATOL_MEAN, (layer, float(d.max()), float(d.mean()))
        assert ws.ws_sync(h_rank, check=False) == ws.WS_OK
        ws.ws_cache_destroy(h_direct)
        ws.ws_cache_destroy(h_rank)
    finally:
        dist.destroy_process_group()
