"""CPU oracle for the compressed-tensor decoders -- TEST INFRASTRUCTURE ONLY.

Plain, slow, element-by-element statement of what the on-device decoders
compute (``lt_oracle.c``, plain C, built in-tree as ``liblt_oracle.so``).
Only the test suite, the smoke check and the benchmark's CPU-baseline leg
may use it; the product path never does, and it shares no code with the CUDA
library. Every function here is a ctypes marshalling shim over one C
function; the arithmetic lives in the C file, which cites its sources.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "lt_oracle.c")
LIB = os.path.join(_HERE, "liblt_oracle.so")

OK, INVALID, CORRUPT, SIZE_MISMATCH = 0, 1, 4, 5

_lib = None


def build(force: bool = False) -> str:
    """Compile ``lt_oracle.c`` (gcc, -O2, no fast-math)."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp"
    subprocess.run(["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-fvisibility=hidden",
                    "-fno-fast-math", SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        P, I64, U64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_f16_from_f64.argtypes = [ctypes.c_double]
        lib.oracle_f16_from_f64.restype = ctypes.c_uint16
        lib.oracle_f16_from_f64_array.argtypes = [P, I64, P]
        lib.oracle_f16_to_f64_array.argtypes = [P, I64, P]
        lib.oracle_dequant_int4.argtypes = [P, P, P, I64, I64, I64, P]
        lib.oracle_dequant_int8.argtypes = [P, P, P, I32, I64, I64, P]
        lib.oracle_zrle_decode.argtypes = [P, U64, P, I64, I64, P]
        lib.oracle_lz4_block_decode.argtypes = [P, U64, P, U64]
        lib.oracle_lz4_decode_blocks.argtypes = [P, U64, P, I64, P, U64]
        lib.oracle_lz4_int4_decode.argtypes = [P, U64, P, I64, P, P, I64, I64, I64, P]
        lib.oracle_value_dict_decode.argtypes = [P, I32, P, I64, P]
        lib.oracle_xxh3_64_secret.argtypes = [P, U64, P, U64]
        lib.oracle_xxh3_64_secret.restype = U64
        lib.oracle_hct2_validate.argtypes = [P, U64, P]
        lib.oracle_hct2_validate.restype = I32
        lib.oracle_hct2_meta.argtypes = [P, U64, P, P]
        lib.oracle_hct2_meta.restype = I32
        lib.oracle_int4_matmul.argtypes = [P, I64, P, P, P, I64, I64, I64, P, P]
        lib.oracle_int4_matmul.restype = I32
        for f in ("oracle_dequant_int4", "oracle_dequant_int8", "oracle_zrle_decode", "oracle_value_dict_decode",
                  "oracle_lz4_block_decode", "oracle_lz4_decode_blocks", "oracle_lz4_int4_decode"):
            getattr(lib, f).restype = I32
        _lib = lib
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data


def f16_from_f64(x) -> np.ndarray:
    """Round doubles to fp16 bit patterns (RNE), own implementation."""
    x = _c(np.atleast_1d(x), np.float64)
    out = np.zeros(x.size, dtype=np.uint16)
    _load().oracle_f16_from_f64_array(_p(x), x.size, _p(out))
    return out


def f16_to_f64(h) -> np.ndarray:
    h = _c(np.atleast_1d(h), np.uint16)
    out = np.zeros(h.size, dtype=np.float64)
    _load().oracle_f16_to_f64_array(_p(h), h.size, _p(out))
    return out


def dequant_int4(packed, scales, zeros, rows: int, cols: int, group_size: int):
    """Returns (fp16 bits as uint16 [rows*cols], status)."""
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint16)
    zeros = None if zeros is None else _c(zeros, np.uint8)
    out = np.zeros(rows * cols, dtype=np.uint16)
    st = _load().oracle_dequant_int4(_p(packed), _p(scales), _p(zeros), rows, cols, group_size, _p(out))
    return out, st


def dequant_int8(q, scales, zeros, per_row: bool, rows: int, cols: int):
    q = _c(q, np.int8)
    scales = _c(scales, np.uint16)
    zeros = None if zeros is None else _c(zeros, np.int8)
    out = np.zeros(rows * cols, dtype=np.uint16)
    st = _load().oracle_dequant_int8(_p(q), _p(scales), _p(zeros), int(per_row), rows, cols, _p(out))
    return out, st


def zrle_decode(enc, offsets, n: int, chunk_elems: int):
    enc = _c(enc, np.uint8)
    offsets = _c(offsets, np.uint64)
    out = np.zeros(n, dtype=np.uint16)
    st = _load().oracle_zrle_decode(_p(enc), enc.size, _p(offsets), n, chunk_elems, _p(out))
    return out, st


def lz4_block_decode(src, dst_len: int):
    src = _c(np.frombuffer(bytes(src), np.uint8) if not isinstance(src, np.ndarray) else src, np.uint8)
    out = np.zeros(max(dst_len, 1), dtype=np.uint8)
    st = _load().oracle_lz4_block_decode(_p(src), src.size, _p(out), dst_len)
    return out[:dst_len], st


def lz4_decode_blocks(comp, offsets, block_bytes: int, dst_len: int):
    comp = _c(comp, np.uint8)
    offsets = _c(offsets, np.uint64)
    out = np.zeros(max(dst_len, 1), dtype=np.uint8)
    st = _load().oracle_lz4_decode_blocks(_p(comp), comp.size, _p(offsets), block_bytes, _p(out), dst_len)
    return out[:dst_len], st


def lz4_int4_decode(comp, offsets, block_bytes: int, scales, zeros, rows: int, cols: int, group_size: int):
    comp = _c(comp, np.uint8)
    offsets = _c(offsets, np.uint64)
    scales = _c(scales, np.uint16)
    zeros = None if zeros is None else _c(zeros, np.uint8)
    out = np.zeros(rows * cols, dtype=np.uint16)
    st = _load().oracle_lz4_int4_decode(_p(comp), comp.size, _p(offsets), block_bytes, _p(scales), _p(zeros),
                                        rows, cols, group_size, _p(out))
    return out, st


def value_dict_decode(packed, bits: int, dictionary, n: int):
    """Returns (fp16 bits as uint16 [n], status): out[k] = dictionary[index k],
    index k the ``bits``-wide field at bit k * bits, least-significant first."""
    packed = _c(packed, np.uint8)
    dictionary = _c(dictionary, np.uint16)
    if bits in (1, 2, 4, 8):
        if dictionary.size != 1 << bits:
            raise ValueError("the dictionary holds 2**bits entries")
        if n > 0 and packed.size * 8 < n * bits:
            raise ValueError("packed holds fewer than n indices")
    out = np.zeros(max(n, 0), dtype=np.uint16)
    st = _load().oracle_value_dict_decode(_p(packed), bits, _p(dictionary), n, _p(out))
    return out, st


XXH3_SECRET_MIN = 136


def xxh3_64(data, secret) -> int:
    """XXH3 64-bit hash of ``data`` with ``secret`` (>= 136 bytes), seed 0."""
    d = _c(np.frombuffer(bytes(data), np.uint8) if not isinstance(data, np.ndarray) else data, np.uint8)
    sec = _c(np.frombuffer(bytes(secret), np.uint8) if not isinstance(secret, np.ndarray) else secret, np.uint8)
    if sec.size < XXH3_SECRET_MIN:
        raise ValueError("the XXH3 secret holds at least 136 bytes")
    buf = d if d.size else np.zeros(1, np.uint8)
    return int(_load().oracle_xxh3_64_secret(_p(buf), d.size, _p(sec), sec.size))


HCT_OK, HCT_BAD_HEADER, HCT_TRUNCATED, HCT_META_MISMATCH, HCT_BLOCK_MISMATCH = 0, 1, 2, 3, 4
HCT_META_FIELDS = ("version", "compression", "quantization", "checksum", "block_size", "rows", "cols",
                   "group_size", "secret_len", "n_blocks", "payload_bytes", "n_groups")
HCT_SECTIONS = ("offsets", "hashes", "scales", "zeros", "payload", "end")


def _buf(container) -> np.ndarray:
    b = container if isinstance(container, np.ndarray) else np.frombuffer(bytes(container), np.uint8)
    b = _c(b, np.uint8)
    return b if b.size else np.zeros(1, np.uint8)


def hct2_validate(container):
    """(status, first mismatching block or None) of an HCT v2 container."""
    b = _buf(container)
    n = len(container)
    bad = np.zeros(1, np.uint64)
    st = _load().oracle_hct2_validate(_p(b), n, _p(bad))
    return st, (int(bad[0]) if st == HCT_BLOCK_MISMATCH else None)


def hct2_meta(container):
    """(status, header fields as a dict, section byte offsets as a dict)."""
    b = _buf(container)
    meta = np.zeros(12, np.uint64)
    sec = np.zeros(6, np.uint64)
    st = _load().oracle_hct2_meta(_p(b), len(container), _p(meta), _p(sec))
    return st, dict(zip(HCT_META_FIELDS, map(int, meta))), dict(zip(HCT_SECTIONS, map(int, sec)))


def int4_matmul(x, M: int, packed, scales, zeros, K: int, N: int, group_size: int):
    """(out, absum, status): out = x @ W in double, W the INT4 dequant of a
    [K, N] matrix (groups along each row), x binary16 bits [M, K]; absum is
    the sum of |x[m, k] * W[k, n]|."""
    x = _c(x, np.uint16)
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint16)
    zeros = None if zeros is None else _c(zeros, np.uint8)
    out = np.zeros((M, N), np.float64)
    absum = np.zeros((M, N), np.float64)
    st = _load().oracle_int4_matmul(_p(x), M, _p(packed), _p(scales), _p(zeros), K, N, group_size, _p(out),
                                    _p(absum))
    return out, absum, st
