"""The multi-rank bench path on CPU: two gloo ranks, as `bench.py --gpus 2`
launches them (one process each, torchrun environment), must own disjoint
layer stacks with distinct inputs, meet at the barrier, and agree on the
slowest rank's time (the max over ranks that the bench reports)."""

import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, layers_per_rank, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist

    import bench
    import oracle
    from prefill_eviction_scoring_b200 import workloads as wl

    D = bench.Dist(backend="gloo")
    D.init()
    layers = wl.split_layers(layers_per_rank, world, rank)
    sums = []
    for li in layers:
        lay = wl.make_layer("tiny", layer=li, lens=(96,))
        s = oracle.score(wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K),
                         lay.cu_seqlens.numpy(), 1.0, 16)
        sums.append(float(np.sum(s[:, :40])))
    D.barrier()
    gathered = [None] * world
    dist.all_gather_object(gathered, (rank, layers, sums))
    slowest = D.max(0.25 * (rank + 1))
    D.close()
    q.put((rank, gathered, slowest))


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks_shard_layers_and_reduce_max(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, 2, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, gathered, slowest in results:
        assert slowest == pytest.approx(0.25 * world)
        owned = [set(layers) for _, layers, _ in gathered]
        assert set.union(*owned) == set(range(2 * world))          # every layer once
        assert sum(len(o) for o in owned) == 2 * world
        sums = [x for _, _, s in gathered for x in s]
        assert len(set(round(x, 9) for x in sums)) == len(sums)     # distinct inputs


def _heads_rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist

    import bench
    import oracle
    from prefill_eviction_scoring_b200 import workloads as wl

    D = bench.Dist(backend="gloo")
    D.init()
    lay = wl.make_layer("llama1b", lens=(160, 90), heads=(8, 4), head_dim=16)
    g0, g1 = bench.head_shard(rank, world, 4)
    G = 2
    s = oracle.score(wl.to_numpy64(lay.Q[:, g0 * G:g1 * G]), wl.to_numpy64(lay.K[:, g0:g1]),
                     lay.cu_seqlens.numpy(), 1.0, 16)
    gathered = [None] * world
    dist.all_gather_object(gathered, (g0, g1, s))
    full = oracle.score(wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K), lay.cu_seqlens.numpy(),
                        1.0, 16)
    D.close()
    q.put((rank, gathered, full))


def test_two_gloo_ranks_split_kv_heads():
    """Tensor-parallel split: each rank scores its own KV heads of the same
    layer (with their query heads); the shards, put back in head order, are
    the whole layer's scores bit for bit (the heads are independent)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_heads_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import numpy as np
    for rank, gathered, full in results:
        spans = sorted((g0, g1) for g0, g1, _ in gathered)
        assert spans == [(0, 2), (2, 4)]
        cat = np.concatenate([s for _, _, s in sorted(gathered, key=lambda x: x[0])])
        np.testing.assert_array_equal(cat, full)


@pytest.mark.parametrize("world,Hkv", [(1, 8), (2, 8), (3, 8), (8, 8), (16, 8), (4, 4)])
def test_head_shards_partition_the_heads(world, Hkv):
    sys.path.insert(0, ROOT)
    import bench
    spans = [bench.head_shard(r, world, Hkv) for r in range(world)]
    owned = [g for g0, g1 in spans for g in range(g0, g1)]
    assert owned == list(range(Hkv))
