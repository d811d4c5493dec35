"""Oracle decodes of block ranges of LZ4 + INT4 matrices, spread over host
threads (the oracle's C code runs outside the interpreter lock). Used by the
full-size parity tests, which compare the GPU's output with the oracle's
element by element on the workload's own matrices."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle


def lz4_int4_block_range(m: dict, b0: int, b1: int):
    """Oracle decode of blocks [b0, b1) of matrix ``m`` (a workload dict with
    comp, offsets, scales, zeros, rows, cols, group_size, block_bytes):
    (binary16 bits of codes [2*b0*block_bytes, ...), status)."""
    bb, G = m["block_bytes"], m["group_size"]
    n = m["rows"] * m["cols"]
    c0 = 2 * b0 * bb
    c1 = min(n, 2 * b1 * bb)
    assert c0 % G == 0, "block ranges must start on a group boundary"
    offs = m["offsets"]
    s0, s1 = int(offs[b0]), int(offs[b1])
    sub_offs = (np.asarray(offs[b0:b1 + 1], dtype=np.uint64) - np.uint64(s0)).astype(np.uint64)
    g0, g1 = c0 // G, (c1 + G - 1) // G
    z = None if m.get("zeros") is None else m["zeros"][g0:g1]
    return oracle.lz4_int4_decode(m["comp"][s0:s1], sub_offs, bb, m["scales"][g0:g1], z, 1, c1 - c0, G)


def pieces(n_blocks: int, per: int):
    return [(a, min(n_blocks, a + per)) for a in range(0, n_blocks, per)]


def pool(threads: int | None = None) -> ThreadPoolExecutor:
    return ThreadPoolExecutor(max_workers=threads or os.cpu_count() or 1)
