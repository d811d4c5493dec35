"""Independent reference helpers for pinning the oracle (no oracle code here).

* ``nearest_f16_bits``: round an exact rational to binary16 by searching the
  whole grid of binary16 values (exact Fractions), nearest first, ties to the
  encoding with an even last bit, magnitudes at or past 65520 to infinity.
* ``liblz4``: the system LZ4 library (ctypes), used as an outside decoder and
  encoder of the raw LZ4 block format.
* ``libxxhash``: the system xxHash library (ctypes), an outside XXH3-64.
* ``hct2_build``: an HCT v2 container laid out byte by byte with ``struct``,
  its hashes from the system xxHash library.
"""
from __future__ import annotations

import bisect
import ctypes
import ctypes.util
from fractions import Fraction
from functools import lru_cache

import numpy as np


@lru_cache(maxsize=1)
def _grid():
    # non-negative finite encodings 0x0000..0x7BFF increase with their value;
    # 0x7C00 (infinity) stands in for 2^16 so that values past the last
    # midpoint round "up" to it exactly as ties-to-even prescribes.
    bits = np.arange(0x7C00, dtype=np.uint16)
    vals = [Fraction(float(v)) for v in bits.view(np.float16).astype(np.float64)]
    vals.append(Fraction(65536))
    return vals


def nearest_f16_bits(t: Fraction) -> int:
    t = Fraction(t)
    sign = 0x8000 if t < 0 else 0
    a = abs(t)
    grid = _grid()
    i = bisect.bisect_left(grid, a)
    if i < len(grid) and grid[i] == a:
        return sign | i
    if i >= len(grid):
        return sign | 0x7C00
    lo, hi = i - 1, i
    dlo, dhi = a - grid[lo], grid[hi] - a
    if dlo < dhi:
        pick = lo
    elif dhi < dlo:
        pick = hi
    else:
        pick = lo if lo % 2 == 0 else hi
    return sign | pick


@lru_cache(maxsize=1)
def liblz4():
    name = ctypes.util.find_library("lz4") or "liblz4.so.1"
    try:
        lib = ctypes.CDLL(name)
    except OSError:
        return None
    lib.LZ4_decompress_safe.argtypes = [ctypes.c_char_p, ctypes.c_char_p, ctypes.c_int, ctypes.c_int]
    lib.LZ4_decompress_safe.restype = ctypes.c_int
    lib.LZ4_compress_default.argtypes = [ctypes.c_char_p, ctypes.c_char_p, ctypes.c_int, ctypes.c_int]
    lib.LZ4_compress_default.restype = ctypes.c_int
    lib.LZ4_compressBound.argtypes = [ctypes.c_int]
    lib.LZ4_compressBound.restype = ctypes.c_int
    return lib


def lz4_lib_decompress(comp: bytes, out_len: int) -> bytes | None:
    lib = liblz4()
    dst = ctypes.create_string_buffer(max(out_len, 1))
    r = lib.LZ4_decompress_safe(bytes(comp), dst, len(comp), out_len)
    return None if r < 0 else dst.raw[:r]


def lz4_lib_compress(data: bytes) -> bytes:
    lib = liblz4()
    cap = lib.LZ4_compressBound(len(data))
    dst = ctypes.create_string_buffer(cap)
    r = lib.LZ4_compress_default(bytes(data), dst, len(data), cap)
    assert r > 0
    return dst.raw[:r]


def hexbytes(s: str) -> bytes:
    return bytes.fromhex(s.replace(" ", ""))


@lru_cache(maxsize=1)
def libxxhash():
    name = ctypes.util.find_library("xxhash") or "libxxhash.so.0"
    try:
        lib = ctypes.CDLL(name)
    except OSError:
        return None
    lib.XXH3_64bits_withSecret.argtypes = [ctypes.c_char_p, ctypes.c_size_t, ctypes.c_char_p, ctypes.c_size_t]
    lib.XXH3_64bits_withSecret.restype = ctypes.c_uint64
    return lib


def xxh3_lib(data: bytes, secret: bytes) -> int:
    return int(libxxhash().XXH3_64bits_withSecret(bytes(data), len(data), bytes(secret), len(secret)))


def _pad16(b: bytearray) -> None:
    b.extend(b"\0" * (-len(b) % 16))


def hct2_build(blocks, block_size: int, rows: int, cols: int, group_size: int, quantization: int,
               scales: bytes = b"", zeros: bytes = b"", secret: bytes = b"", compression: int = 1) -> bytes:
    """An HCT v2 container: 64-byte header, secret, offsets, block hashes,
    scales, zero points and payload, each section from a 16-byte boundary."""
    import struct

    payload = b"".join(bytes(x) for x in blocks)
    offs = [0]
    for x in blocks:
        offs.append(offs[-1] + len(x))
    head = bytearray(struct.pack("<4sHHBBBBIQQIIQQQ", b"HCT2", 2, 0, compression, quantization, 1, 0, block_size,
                                 rows, cols, group_size, len(secret), len(blocks), len(payload), 0))
    assert len(head) == 64
    head += secret
    _pad16(head)
    head += struct.pack(f"<{len(offs)}Q", *offs)
    _pad16(head)
    head += struct.pack(f"<{len(blocks)}Q", *[xxh3_lib(bytes(x), secret) for x in blocks])
    _pad16(head)
    head += scales
    _pad16(head)
    head += zeros
    _pad16(head)
    head[56:64] = struct.pack("<Q", xxh3_lib(bytes(head), secret))
    return bytes(head) + payload
