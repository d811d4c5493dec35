"""Multi-rank host logic on CPU (gloo, world size 2): sharding covers every
unit exactly once, a rank's share of an LZ4 stream decodes to its share of
the tensor, and the timing reductions give the slowest rank and the total."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from weight_dequantization_b200.shard import shard_blocks, shard_range


@pytest.mark.parametrize("n,world", [(0, 1), (1, 2), (7, 2), (448, 3), (6528, 8), (5, 8)])
def test_shard_range_partitions_units(n, world):
    seen = []
    for r in range(world):
        a, b = shard_range(n, r, world)
        assert 0 <= a <= b <= n
        seen.extend(range(a, b))
        assert b - a in (n // world, n // world + 1)
    assert seen == list(range(n))


def test_shard_range_rejects_bad_ranks():
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, result_q):
    import torch.distributed as dist

    import oracle
    from weight_dequantization_b200.shard import reduce_max, reduce_sum
    from weight_dequantization_b200.synth import int4_gauss_groups_packed, lz4_compress_blocks

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # every rank holds the same compressed stream; each decodes its share
        packed = int4_gauss_groups_packed(3, 7 * 2 * 16384)
        comp, offs = lz4_compress_blocks(packed, 16384)
        b0, nb, rebased, base = shard_blocks(offs, rank, world)
        end = base + rebased[-1]
        raw, st = oracle.lz4_decode_blocks(comp[base:end], np.array(rebased, np.uint64), 16384, nb * 16384)
        ok = st == 0 and np.array_equal(raw, packed[b0 * 16384:(b0 + nb) * 16384])
        mx = reduce_max(1.5 + rank)
        sm = reduce_sum(float(nb))
        result_q.put((rank, ok, nb, mx, sm))
    finally:
        dist.destroy_process_group()


def test_two_ranks_decode_disjoint_shares_and_reduce_timings():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    assert all(ok for _, ok, _, _, _ in results)
    assert sum(nb for _, _, nb, _, _ in results) == 7  # every block decoded by exactly one rank
    assert all(mx == 2.5 for _, _, _, mx, _ in results)  # the slowest rank's time
    assert all(sm == 7.0 for _, _, _, _, sm in results)
