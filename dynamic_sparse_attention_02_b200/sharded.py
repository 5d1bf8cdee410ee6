"""Head-sharded prefill across GPUs: one process per GPU, each holding a
contiguous range of KV heads and the query heads that read them.

Every (query head, query block) of a layer is independent and needs only its
own KV head, so a layer splits across ranks by KV-head group with no exchange
during the computation: each rank runs the whole hot path (index estimation
and sparse attention, one mi_prefill_layer call) on its own heads.  The one
collective is afterwards, and only for callers that want every head's output
on every rank: an all-gather of `out` (NCCL over NVLink / NVSwitch on GPUs).
In a tensor-parallel model the ranks would keep their own heads and the
output projection's reduction would follow instead; that belongs to the model,
not to this layer.  The project's v0.1.5.post1 release added multi-GPU support
(hysenlabs project review, "Licence, maintenance cadence").

The split keeps whole GQA groups together (query head h reads KV head
floor(h * Hkv / Hq)), so a rank's local tensors are a valid layer of their own
with the same group ratio, and its local pattern table is the global table's
slice.  Shards differ by at most one KV head when world does not divide Hkv.
"""
from __future__ import annotations

from typing import Callable, Optional

import numpy as np
import torch


def kv_range(Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """[g0, g1): the KV heads of `rank`; the first Hkv % world ranks take one extra."""
    if not (0 <= rank < world) or world < 1:
        raise ValueError(f"rank {rank} outside world {world}")
    base, extra = divmod(Hkv, world)
    g0 = rank * base + min(rank, extra)
    return g0, g0 + base + (1 if rank < extra else 0)


def head_range(Hq: int, Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """[h0, h1): the query heads that read the KV heads of kv_range()."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    gq = Hq // Hkv
    g0, g1 = kv_range(Hkv, world, rank)
    return g0 * gq, g1 * gq


def shard_inputs(q, k, v, pattern, world: int, rank: int):
    """This rank's contiguous views of the layer's q [Hq,N,d], k, v [Hkv,N,d]
    and host pattern table [Hq] (views share storage; no copy)."""
    Hq, Hkv = q.shape[0], k.shape[0]
    g0, g1 = kv_range(Hkv, world, rank)
    h0, h1 = head_range(Hq, Hkv, world, rank)
    return q[h0:h1], k[g0:g1], v[g0:g1], np.asarray(pattern)[h0:h1]


class ShardedPrefill:
    """Run one layer over this rank's heads, then (optionally) all-gather the
    output so that every rank holds out [Hq, N, d].

    layer_fn(q, k, v, pattern, params, out) computes this rank's heads into
    `out`; by default the library's mi_prefill_layer.  dist / group are the
    torch.distributed module and process group (NCCL on GPUs).
    """

    def __init__(self, dist, group=None, layer_fn: Optional[Callable] = None):
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if layer_fn is None:
            from . import binding

            def layer_fn(q, k, v, pattern, params, out):
                binding.mi_prefill_layer(q, k, v, pattern, params, out=out)
        self.layer_fn = layer_fn

    def local(self, q_loc, k_loc, v_loc, pattern_loc, params, out_loc=None):
        """This rank's heads only: out_loc [Hq_rank, N, d] (no collective)."""
        if out_loc is None:
            out_loc = torch.empty_like(q_loc)
        if q_loc.shape[0]:
            self.layer_fn(q_loc, k_loc, v_loc, pattern_loc, params, out_loc)
        return out_loc

    def gather(self, out_loc, Hq: int, Hkv: int, out: Optional[torch.Tensor] = None):
        """All-gather every rank's out_loc into out [Hq, N, d] on every rank.
        Equal shards gather straight into `out`; unequal ones go through a
        padded buffer of world x the largest shard."""
        N, d = out_loc.shape[1], out_loc.shape[2]
        if out is None:
            out = torch.empty((Hq, N, d), dtype=out_loc.dtype, device=out_loc.device)
        sizes = [head_range(Hq, Hkv, self.world, r) for r in range(self.world)]
        hmax = max(h1 - h0 for h0, h1 in sizes)
        if all(h1 - h0 == hmax for h0, h1 in sizes):
            self.dist.all_gather_into_tensor(out, out_loc.contiguous(), group=self.group)
            return out
        pad = torch.zeros((hmax, N, d), dtype=out_loc.dtype, device=out_loc.device)
        pad[:out_loc.shape[0]] = out_loc
        full = torch.empty((self.world * hmax, N, d), dtype=out_loc.dtype,
                           device=out_loc.device)
        self.dist.all_gather_into_tensor(full, pad, group=self.group)
        for r, (h0, h1) in enumerate(sizes):
            out[h0:h1] = full[r * hmax:r * hmax + (h1 - h0)]
        return out

    def __call__(self, q_loc, k_loc, v_loc, pattern_loc, params, Hq: int, Hkv: int,
                 out: Optional[torch.Tensor] = None):
        """local() then gather(): out [Hq, N, d] on every rank."""
        out_loc = self.local(q_loc, k_loc, v_loc, pattern_loc, params)
        return self.gather(out_loc, Hq, Hkv, out)
