"""Cases run through whichever library WS_LIBRARY selects (libws.so, or libws_debug.so with
device index checks): the tiny workload, ragged key runs with a gap and an uncommitted
unit at both head sizes, a cache readback, a two-unit prefill and a two-session call.
Writes every output and status to the .npz file named on the command line."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gpu_util import from_dev, to_dev  # noqa: E402
from kv_cache_serving_ws_b200 import native as ws  # noqa: E402
from kv_cache_serving_ws_b200 import synth  # noqa: E402
from kv_cache_serving_ws_b200.workloads import TINY, GpuSession  # noqa: E402

res = {}


def bits(seed, kind, shape, u=0, layer=0):
    return synth.normal_tensor(synth.stream_key(seed, kind, u, layer), shape)


def ragged(D, splits):
    L, H, Nv, Na, Nc, U = 2, 3, 130, 3, 5, 4
    Nq = Nv + Na
    _, h = ws.ws_cache_create(ws.make_config(L, H, D, Nv, Na, Nc, U))
    ws.ws_cache_set_splits(h, splits)
    for u in (0, 1, 2, 4, 5, 6):
        ws.ws_cache_append(h, u, ws.WS_SEG_COND, to_dev(bits(D, synth.KIND_COND_K, (L, Nc, H, D), u)),
                           to_dev(bits(D, synth.KIND_COND_V, (L, Nc, H, D), u)))
        if u not in (5, 6):
            ws.ws_cache_append(h, u, ws.WS_SEG_LATENT, to_dev(bits(D, synth.KIND_COMMIT_K, (L, Nq, H, D), u)),
                               to_dev(bits(D, synth.KIND_COMMIT_V, (L, Nq, H, D), u)))
    s = (Nq, H, D)
    out = torch.empty(s, dtype=torch.bfloat16, device="cuda")
    ws.ws_unit_attention(h, 1, 6, to_dev(bits(D, synth.KIND_Q, s, 6, 1)), to_dev(bits(D, synth.KIND_K_NEW, s, 6, 1)),
                         to_dev(bits(D, synth.KIND_V_NEW, s, 6, 1)), out)
    kb = torch.empty((Nc, H, D), dtype=torch.bfloat16, device="cuda")
    vb = torch.empty_like(kb)
    ws.ws_cache_read(h, 0, 4, ws.WS_SEG_COND, kb, vb)
    res[f"ragged_{D}_{splits}_status"] = np.array(ws.ws_sync(h, check=False))
    res[f"ragged_{D}_{splits}_out"] = from_dev(out)
    res[f"ragged_{D}_{splits}_read"] = from_dev(kb)
    ws.ws_cache_destroy(h)


def prefill_and_sessions(D):
    L, H, Nv, Na, Nc, U = 1, 2, 120, 4, 16, 3
    Nq = Nv + Na
    _, h = ws.ws_pool_create(ws.make_config(L, H, D, Nv, Na, Nc, U), 2)
    for s_ in range(2):
        for u in range(2):
            ws.ws_session_append(h, s_, u, ws.WS_SEG_COND, to_dev(bits(7 + s_, synth.KIND_COND_K, (L, Nc, H, D), u)),
                                 to_dev(bits(7 + s_, synth.KIND_COND_V, (L, Nc, H, D), u)))
    shape = (2, Nq, H, D)
    q, kn, vn = (to_dev(bits(9, k, shape)) for k in (synth.KIND_Q, synth.KIND_K_NEW, synth.KIND_V_NEW))
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    ws.ws_session_attention(h, 0, [0, 1], [1, 1], q, kn, vn, out)
    out2 = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    ws.ws_session_attention(h, 0, [0, 0], [0, 1], q, kn, vn, out2)     # a prefill stretch of session 0
    res[f"pool_{D}_status"] = np.array(ws.ws_sync(h, check=False))
    res[f"pool_{D}_out"] = from_dev(out)
    res[f"pool_{D}_prefill"] = from_dev(out2)
    ws.ws_cache_destroy(h)


g = GpuSession(TINY)
g.prefill()
q, kn, vn = g.step_inputs(0)
o = g.attention(0, q, kn, vn)
res["tiny_status"] = np.array(ws.ws_sync(g.h, check=False))
res["tiny_out"] = from_dev(o)
g.close()
for D in (64, 128):
    for splits in (0, 3):
        ragged(D, splits)
    prefill_and_sessions(D)
np.savez(sys.argv[1], **res)
print("library", ws.LIB_PATH, "cases", len(res))
