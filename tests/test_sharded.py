"""Head-sharded layer (sharded.py) on CPU: the KV-head partition, the local
GQA mapping, and the all-gather that reassembles out [Hq, N, d], with two
ranks over gloo.  The per-rank layer is a stand-in (the library needs a GPU):
it writes out[h] = q[h] + k[g(h)] with the rank's own local GQA mapping, so a
wrong slice, group mapping or reassembly order shows up as a mismatch."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from dynamic_sparse_attention_02_b200 import sharded  # noqa: E402


def test_kv_ranges_partition_the_heads():
    for Hkv in (1, 2, 3, 7, 8):
        for world in (1, 2, 3, 4, 8):
            rs = [sharded.kv_range(Hkv, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == Hkv
            for (a0, a1), (b0, b1) in zip(rs, rs[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1
            assert sizes == sorted(sizes, reverse=True)
    # whole GQA groups: query head h of a rank reads a KV head of the same rank
    Hq, Hkv = 32, 8
    for world in (1, 2, 3, 8):
        for r in range(world):
            h0, h1 = sharded.head_range(Hq, Hkv, world, r)
            g0, g1 = sharded.kv_range(Hkv, world, r)
            for h in range(h0, h1):
                assert g0 <= h * Hkv // Hq < g1
    with pytest.raises(ValueError):
        sharded.kv_range(8, 2, 2)


def _stand_in_layer(q, k, v, pattern, params, out):
    Hq, Hkv = q.shape[0], k.shape[0]
    for h in range(Hq):
        out[h] = q[h] + k[h * Hkv // Hq] + float(pattern[h])


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, Hq, Hkv, res):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    from dynamic_sparse_attention_02_b200 import sharded as S
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        N, d = 128, 8
        g = torch.Generator().manual_seed(5)  # every rank draws the same full layer
        q = torch.randn(Hq, N, d, generator=g)
        k = torch.randn(Hkv, N, d, generator=g)
        v = torch.randn(Hkv, N, d, generator=g)
        pattern = np.arange(Hq, dtype=np.int8) % 3
        ql, kl, vl, pl = S.shard_inputs(q, k, v, pattern, world, rank)
        runner = S.ShardedPrefill(dist, layer_fn=_stand_in_layer)
        out = runner(ql, kl, vl, pl, None, Hq, Hkv)
        want = torch.empty_like(q)
        _stand_in_layer(q, k, v, pattern, None, want)
        res.put((rank, bool(torch.equal(out, want)), int(ql.shape[0])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (12, 3), (4, 1)])
def test_two_ranks_reassemble_the_layer(Hq, Hkv):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, Hq, Hkv, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok, _ in res)
    # the ranks' shards cover the query heads (one rank may hold none: Hkv = 1)
    assert sum(n for _, _, n in res) == Hq
