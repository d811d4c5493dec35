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


def _worker_next_rows(rank, world, port, result_q):
    import torch.distributed as dist

    import oracle
    from tests._pins import hct2_build, libxxhash
    from weight_dequantization_b200.shard import reduce_sum, shard_range

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(5)  # the same stream on every rank
        # value dictionary: each rank decodes a whole-byte range of the indices
        n, bits = 8 * 1000 + 6, 2
        packed = rng.integers(0, 256, (n * bits + 7) // 8, dtype=np.uint8)
        d = rng.integers(0, 1 << 16, 1 << bits).astype(np.uint16)
        full, _ = oracle.value_dict_decode(packed, bits, d, n)
        per_byte = 8 // bits
        b0, b1 = shard_range(len(packed), rank, world)
        k0, k1 = b0 * per_byte, min(n, b1 * per_byte)
        part, st = oracle.value_dict_decode(packed[b0:b1], bits, d, k1 - k0)
        ok_dict = st == 0 and np.array_equal(part, full[k0:k1])
        covered = reduce_sum(float(k1 - k0))
        # container blocks: each rank checks its block range, one block is bad
        bad_blocks = -1.0
        if libxxhash() is not None:
            secret = rng.integers(0, 256, 192, dtype=np.uint8).tobytes()
            blocks = [rng.integers(0, 256, m, dtype=np.uint8).tobytes() for m in (300, 17, 4100, 2, 999, 64)]
            c = bytearray(hct2_build(blocks, 8192, 1, 8, 0, 0, b"", b"", secret, compression=1))
            _, _, sec = oracle.hct2_meta(bytes(c))
            c[sec["payload"] + 300 + 17 + 5] ^= 1  # a byte of block 2
            offs = np.frombuffer(bytes(c[sec["offsets"]:sec["offsets"] + 8 * 7]), np.uint64)
            stored = np.frombuffer(bytes(c[sec["hashes"]:sec["hashes"] + 8 * 6]), np.uint64)
            payload = bytes(c[sec["payload"]:])
            lo, hi = shard_range(6, rank, world)
            mine = sum(oracle.xxh3_64(payload[offs[b]:offs[b + 1]], secret) != int(stored[b]) for b in range(lo, hi))
            bad_blocks = reduce_sum(float(mine))
        result_q.put((rank, ok_dict, covered, bad_blocks))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_the_value_dictionary_and_container_checks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_next_rows, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok, _, _ in results)
    assert all(cov == 8 * 1000 + 6 for _, _, cov, _ in results)  # every element decoded exactly once
    assert all(bad in (1.0, -1.0) for _, _, _, bad in results)  # the one bad block found once
