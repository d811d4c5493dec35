"""Random valid LZ4 blocks built sequence by sequence (not by a compressor).

Each block mixes every match regime a decoder must get right: offset 1
(byte runs), short periodic offsets 2..15, overlapping offsets >= 16,
non-overlapping copies and far offsets, with literal runs of every length
class (0, < 15, 15, >= 270 needing two extension bytes). The expected output
is produced alongside by direct simulation of the format (append literals;
append out[-d] M times), independently of the oracle and of the GPU
decoder. The end-of-block rules of the reference encoder (last 5 bytes are
literals, no match starting within the last 12 bytes) are kept so that the
system LZ4 library accepts the blocks too.
"""
from __future__ import annotations

import numpy as np


def _len_bytes(n: int) -> bytes:
    out = bytearray()
    while n >= 255:
        out.append(255)
        n -= 255
    out.append(n)
    return bytes(out)


def _sequence(lits: bytes, d: int, m: int) -> bytes:
    L = len(lits)
    tok = (min(L, 15) << 4) | (min(m - 4, 15) if m else 0)
    b = bytearray([tok])
    if L >= 15:
        b += _len_bytes(L - 15)
    b += lits
    if m:
        b += d.to_bytes(2, "little")
        if m - 4 >= 15:
            b += _len_bytes(m - 4 - 15)
    return bytes(b)


def random_block(rng: np.random.Generator, size: int) -> tuple[bytes, bytes]:
    """(compressed block, decompressed bytes of length `size`)."""
    out = bytearray()
    comp = bytearray()
    while True:
        remaining = size - len(out)
        # room for one more (literals + match) sequence before the last 12
        if remaining < 12 + 8 + 5:
            break
        regime = rng.integers(0, 6)
        lit_cls = rng.integers(0, 5)
        L = [0, int(rng.integers(1, 15)), 15, int(rng.integers(16, 270)), int(rng.integers(270, 700))][lit_cls]
        L = min(L, remaining - 12 - 5 - 4)
        if len(out) + L == 0:
            L = max(L, 1)
        lits = rng.integers(0, 256, L, dtype=np.uint8).tobytes()
        op = len(out) + L
        if regime == 0:
            d = 1
        elif regime == 1:
            d = int(rng.integers(2, 16))
        elif regime == 2:
            d = int(rng.integers(16, 64))
        elif regime == 3:
            d = int(rng.integers(64, 4096))
        elif regime == 4:
            d = int(rng.integers(4096, 65536))
        else:
            d = int(rng.integers(1, 65536))
        d = max(1, min(d, op, 65535))
        m_cls = rng.integers(0, 4)
        m = [int(rng.integers(4, 19)), 19, int(rng.integers(20, 300)), int(rng.integers(300, 1200))][m_cls]
        # match must end at least 5 bytes early and start 12+ before the end
        m = max(4, min(m, size - op - 5 - 7))
        if op + m > size - 5 or op > size - 12:
            break
        comp += _sequence(lits, d, m)
        out += lits
        for _ in range(m):
            out.append(out[-d])
    tail = rng.integers(0, 256, size - len(out), dtype=np.uint8).tobytes()
    comp += _sequence(tail, 0, 0)
    out += tail
    assert len(out) == size
    return bytes(comp), bytes(out)


def random_blocks(seed: int, n_blocks: int, block_bytes: int, last: int | None = None):
    """n_blocks independent blocks -> (comp uint8, offsets uint64, raw uint8)."""
    rng = np.random.default_rng(seed)
    comps, raws = [], []
    for b in range(n_blocks):
        size = block_bytes if (last is None or b < n_blocks - 1) else last
        c, r = random_block(rng, size)
        comps.append(c)
        raws.append(r)
    offs = np.concatenate([[0], np.cumsum([len(c) for c in comps])]).astype(np.uint64)
    return (np.frombuffer(b"".join(comps), np.uint8).copy(), offs,
            np.frombuffer(b"".join(raws), np.uint8).copy())
