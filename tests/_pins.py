"""Independent reference helpers for pinning the oracle (no oracle code here).

* ``nearest_f16_bits``: round an exact rational to binary16 by searching the
  whole grid of binary16 values (exact Fractions), nearest first, ties to the
  encoding with an even last bit, magnitudes at or past 65520 to infinity.
* ``liblz4``: the system LZ4 library (ctypes), used as an outside decoder and
  encoder of the raw LZ4 block format.
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
