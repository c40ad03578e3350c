"""Seeded synthetic workloads of the unit step (shapes and input streams), shared by the
GPU tests, smoke() and bench.py.  No attention, cache or Euler arithmetic.

Shapes (per unit): the pages' 640x368 stream at 25 FPS in 160 ms units; the latent
grid is the frame size divided by 16 (one latent frame per unit), plus a few audio
latent tokens and the thinker's conditioning tokens.  Every tensor element is drawn
by kv_cache_serving_ws_b200.synth from (seed, tensor kind, unit, layer, step).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_heads: int
    head_dim: int
    n_video: int
    n_audio: int
    n_cond: int
    history_units: int
    seed: int
    unit: int            # the unit being generated (earlier units fill the history)
    steps: int = 1       # Euler steps per unit
    dt: float = 0.25

    @property
    def n_query(self):
        return self.n_video + self.n_audio

    @property
    def tokens_per_unit(self):
        return self.n_cond + self.n_query

    @property
    def n_keys(self):
        """Keys a query sees in steady state: U + 1 full units."""
        return (self.history_units + 1) * self.tokens_per_unit

    def flops_per_call(self):
        return 4.0 * self.n_query * self.n_keys * self.n_heads * self.head_dim

    def history(self):
        return list(range(self.unit - self.history_units, self.unit))


# 192x336 frame -> 12x21 latent grid = 252 video tokens; 368x640 -> 23x40 = 920.
TINY = Workload("tiny-192x336-5units-8x64", 1, 8, 64, 252, 8, 64, 4, seed=1, unit=4)
V01 = Workload("v01-192x336-hist16-40x128", 1, 40, 128, 252, 4, 32, 16, seed=2, unit=16)
V02 = Workload("v02-640x368-hist32-40x128", 1, 40, 128, 920, 4, 32, 32, seed=3, unit=32)
RING = Workload("v02-640x368-ring128-u1000-40x128", 1, 40, 128, 920, 4, 32, 128, seed=4, unit=1000)
FULL = Workload("v02-640x368-unit-40L-4steps-hist64-40x128", 40, 40, 128, 920, 4, 32, 64, seed=5, unit=64,
                steps=4)
# the same unit with a 32-unit history: the window one B200 can run inside the 160 ms unit
FULL32 = Workload("v02-640x368-unit-40L-4steps-hist32-40x128", 40, 40, 128, 920, 4, 32, 32, seed=7, unit=32,
                  steps=4)
ALL = {w.name: w for w in (TINY, V01, V02, RING, FULL, FULL32)}


def key(w: Workload, kind: int, unit: int = 0, layer: int = 0, step: int = 0) -> int:
    return synth.stream_key(w.seed, kind, unit, layer, step)


def gen_heads(k: int, shape, heads, layer=None) -> np.ndarray:
    """Elements of one logical tensor restricted to some heads (and one layer).

    shape is (L, n, H, D) with ``layer`` given, or (n, H, D).  Returns uint16
    bf16 patterns [n, len(heads), D] without generating the other heads.
    """
    if len(shape) == 4:
        L, n, H, D = shape
        base = layer * n * H * D
    else:
        n, H, D = shape
        base = 0
    heads = np.asarray(heads, dtype=np.int64)
    t = np.arange(n, dtype=np.int64)[:, None, None]
    idx = base + (t * H + heads[None, :, None]) * D + np.arange(D, dtype=np.int64)[None, None, :]
    return synth.normal_bf16(k, idx.reshape(-1).astype(np.uint64)).reshape(n, len(heads), D)


class GpuSession:
    """Drives the library through its C ABI for one workload (device inputs from the
    device generator, bit-identical to the numpy one)."""

    def __init__(self, w: Workload, device="cuda:0"):
        import torch

        from . import native as ws
        self.ws, self.torch, self.w = ws, torch, w
        self.dev = torch.device(device)
        self.cfg = ws.make_config(w.n_layers, w.n_heads, w.head_dim, w.n_video, w.n_audio, w.n_cond,
                                  w.history_units)
        _, self.h = ws.ws_cache_create(self.cfg)
        e = torch.empty
        self.cond_k = e((w.n_layers, w.n_cond, w.n_heads, w.head_dim), dtype=torch.bfloat16, device=self.dev)
        self.cond_v = torch.empty_like(self.cond_k)
        self._commit = None

    def fill(self, t, k: int):
        self.ws.synth_fill(t, k)
        return t

    def commit_buffers(self):
        if self._commit is None:
            w, torch = self.w, self.torch
            shape = (w.n_layers, w.n_query, w.n_heads, w.head_dim)
            self._commit = (torch.empty(shape, dtype=torch.bfloat16, device=self.dev),
                            torch.empty(shape, dtype=torch.bfloat16, device=self.dev))
        return self._commit

    def append_cond(self, u):
        s = synth
        self.fill(self.cond_k, key(self.w, s.KIND_COND_K, u))
        self.fill(self.cond_v, key(self.w, s.KIND_COND_V, u))
        return self.ws.ws_cache_append(self.h, u, self.ws.WS_SEG_COND, self.cond_k, self.cond_v)

    def commit(self, u):
        s = synth
        ck, cv = self.commit_buffers()
        self.fill(ck, key(self.w, s.KIND_COMMIT_K, u))
        self.fill(cv, key(self.w, s.KIND_COMMIT_V, u))
        return self.ws.ws_cache_append(self.h, u, self.ws.WS_SEG_LATENT, ck, cv)

    def prefill(self):
        for u in self.w.history():
            self.append_cond(u)
            self.commit(u)
        self.append_cond(self.w.unit)

    def step_inputs(self, layer, step=0):
        s, torch, w = synth, self.torch, self.w
        shape = (w.n_query, w.n_heads, w.head_dim)
        q = torch.empty(shape, dtype=torch.bfloat16, device=self.dev)
        kn, vn = torch.empty_like(q), torch.empty_like(q)
        self.fill(q, key(w, s.KIND_Q, w.unit, layer, step))
        self.fill(kn, key(w, s.KIND_K_NEW, w.unit, layer, step))
        self.fill(vn, key(w, s.KIND_V_NEW, w.unit, layer, step))
        return q, kn, vn

    def attention(self, layer, q, kn, vn, out=None):
        if out is None:
            out = self.torch.empty_like(q)
        self.ws.ws_unit_attention(self.h, layer, self.w.unit, q, kn, vn, out)
        return out

    def close(self):
        if self.h is not None:
            self.ws.ws_cache_destroy(self.h)
            self.h = None


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def errors(got, want):
    d = np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))
    return float(d.max()), float(d.mean())
