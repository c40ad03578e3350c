"""Ulysses head-sharded performer step over R ranks (one process per GPU).

The pages' performer group spreads the long high-resolution video latent over
several GPUs with Ulysses-style context parallelism, keeps the short audio
latent unsharded, and pre-shards the thinker's K/V slices so that each GPU
only ever holds its own part of the history ("Wan-Streamer v0.2：更高分辨率，
相同延迟", paper.rainbus.top, section 前置知识, entries Ulysses上下文并行 and
K/V缓存预分片; "Technical Summary: Wan-Streamer v0.2", gist.science, section
Methodology, item 2; remio.ai, section 思考者与执行者的分工掩盖了更高分辨率的成本).

Layouts, for H heads split into R equal groups and Nv video rows split into R
near-equal runs (rank r: video rows [v0(r), v1(r)), heads [h0(r), h1(r))):

* sequence shard of rank r (what the model around attention holds): its video
  rows plus every audio row, ``[v1(r)-v0(r) + Na][H][D]``, video first;
* head shard of rank r (what attention works on): every latent row for its
  heads, ``[Nv + Na][H/R][D]``, the row order of one cache slot's latent
  segment;
* the K/V cache of rank r holds heads [h0(r), h1(r)) only: its conditioning and
  commit slices are the head slices of the full ones (``head_slice``).

One attention call: an all-to-all moves the video rows of q, k_new and v_new to
the ranks that own their heads (audio rows are already everywhere: each rank
takes its heads' columns locally), every rank runs block-causal attention for
its heads over the whole unit (``attention_fn``: the library on a GPU), and a
second all-to-all returns each rank's video rows for all heads; an all-gather
gives every rank the audio output of all heads.  Heads are independent in the
attention, so the result is the single-GPU result, head for head.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable


def video_bounds(n_video: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [v0, v1) of the video latent owned by `rank` (sizes differ by at most one)."""
    base, extra = divmod(n_video, world)
    v0 = rank * base + min(rank, extra)
    return v0, v0 + base + (1 if rank < extra else 0)


def head_bounds(n_heads: int, world: int, rank: int) -> tuple[int, int]:
    if n_heads % world:
        raise ValueError(f"{n_heads} heads do not split over {world} ranks")
    g = n_heads // world
    return rank * g, (rank + 1) * g


def head_slice(t, n_heads: int, world: int, rank: int):
    """The rank's heads of a [..., H, D] tensor (a conditioning or commit slice)."""
    h0, h1 = head_bounds(n_heads, world, rank)
    part = t[..., h0:h1, :]
    return part.contiguous() if hasattr(part, "contiguous") else part.copy()


@dataclass
class UlyssesPlan:
    n_video: int
    n_audio: int
    n_heads: int
    head_dim: int
    world: int
    rank: int

    def __post_init__(self):
        head_bounds(self.n_heads, self.world, 0)          # validates the split
        self.hg = self.n_heads // self.world
        self.v = [video_bounds(self.n_video, self.world, r) for r in range(self.world)]

    @property
    def local_rows(self) -> int:
        v0, v1 = self.v[self.rank]
        return v1 - v0 + self.n_audio


class UlyssesAttention:
    """Head-sharded attention of one rank.  ``attention_fn(layer, unit, q, k_new,
    v_new)`` takes and returns head-shard tensors ``[Nq][H/R][D]``; ``group`` is a
    torch.distributed process group (NCCL on GPUs, gloo on CPU)."""

    def __init__(self, plan: UlyssesPlan, attention_fn: Callable, group=None):
        self.plan = plan
        self.attention_fn = attention_fn
        self.group = group

    # -- sequence shard -> head shard --------------------------------------
    def to_heads(self, *xs):
        """Sequence-shard tensors [nv_r + Na][H][D] -> head-shard [Nv + Na][H/R][D],
        all in one all-to-all."""
        import torch
        import torch.distributed as dist
        p = self.plan
        R, hg, D = p.world, p.hg, p.head_dim
        v0, v1 = p.v[p.rank]
        nv = v1 - v0
        k = len(xs)
        # send buffer: for destination s, the video rows x heads of s of every tensor
        send = torch.stack([x[:nv] for x in xs])                       # [k][nv][H][D]
        send = send.view(k, nv, R, hg, D).permute(2, 0, 1, 3, 4).contiguous()   # [R][k][nv][hg][D]
        recv_rows = [p.v[s][1] - p.v[s][0] for s in range(R)]
        recv = torch.empty(k * sum(recv_rows) * hg * D, dtype=send.dtype, device=send.device)
        dist.all_to_all_single(recv, send.view(-1),
                               output_split_sizes=[k * n * hg * D for n in recv_rows],
                               input_split_sizes=[k * nv * hg * D] * R, group=self.group)
        h0, h1 = p.rank * hg, (p.rank + 1) * hg
        outs = []
        chunks = recv.split([k * n * hg * D for n in recv_rows])
        parts = [c.view(k, n, hg, D) for c, n in zip(chunks, recv_rows)]
        for i, x in enumerate(xs):
            video = torch.cat([pt[i] for pt in parts], dim=0)           # [Nv][hg][D], rank order = row order
            audio = x[nv:, h0:h1]                                        # [Na][hg][D], already here
            outs.append(torch.cat([video, audio], dim=0).contiguous())
        return outs

    # -- head shard -> sequence shard --------------------------------------
    def to_sequence(self, out_heads):
        """Head-shard output [Nv + Na][H/R][D] -> sequence shard [nv_r + Na][H][D]."""
        import torch
        import torch.distributed as dist
        p = self.plan
        R, hg, D = p.world, p.hg, p.head_dim
        v0, v1 = p.v[p.rank]
        nv = v1 - v0
        rows = [p.v[s][1] - p.v[s][0] for s in range(R)]
        send = out_heads[:p.n_video].contiguous()                       # rows in rank order
        recv = torch.empty(R * nv * hg * D, dtype=send.dtype, device=send.device)
        dist.all_to_all_single(recv, send.view(-1), output_split_sizes=[nv * hg * D] * R,
                               input_split_sizes=[n * hg * D for n in rows], group=self.group)
        video = recv.view(R, nv, hg, D).permute(1, 0, 2, 3).reshape(nv, R * hg, D)
        audio_parts = [torch.empty(p.n_audio, hg, D, dtype=send.dtype, device=send.device) for _ in range(R)]
        dist.all_gather(audio_parts, out_heads[p.n_video:].contiguous(), group=self.group)
        audio = torch.cat(audio_parts, dim=1)                            # [Na][H][D], heads in rank order
        return torch.cat([video, audio], dim=0).contiguous()

    def __call__(self, layer: int, unit: int, q, k_new, v_new):
        """One attention call on sequence-shard inputs; returns the sequence-shard output."""
        qh, kh, vh = self.to_heads(q, k_new, v_new)
        out_h = self.attention_fn(layer, unit, qh, kh, vh)
        return self.to_sequence(out_h)


def library_attention_fn(h, stream=None):
    """``attention_fn`` for a GPU rank: block-causal attention of the head-shard
    tensors (bf16, ``[Nv + Na][H/R][D]``) on this rank's head-shard cache ``h``
    (created with ``n_heads = H/R``, appended with ``head_slice`` data)."""
    import torch

    from . import native as ws

    def fn(layer, unit, q, k_new, v_new):
        out = torch.empty_like(q)
        ws.ws_unit_attention(h, layer, unit, q, k_new, v_new, out, stream=stream)
        return out
    return fn
