"""Seeded synthetic inputs for the decode path (numpy arrays on the host).

This module builds the *inputs* of the decoders -- codes, scales, zero
points, INT4 packing, LZ4-compressed blocks and zero-run streams -- from the
value laws of the workloads. It holds no decoding arithmetic and imports
neither the CUDA library nor the CPU oracle; both consume its output.

The heavy lifting is in ``lt_synth.c`` (xoshiro256** substreams, Box-Muller
normals, an LZ4 block-format compressor, a zero-run encoder), built in-tree
as ``liblt_synth.so``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblt_synth.so")
_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from .._build import build_synth

        build_synth()
    lib = ctypes.CDLL(_LIB_PATH)
    P, I64, U64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int32, ctypes.c_double
    lib.synth_set_threads.argtypes = [ctypes.c_int]
    lib.synth_int4_uniform.argtypes = [U64, U64, I64, P]
    lib.synth_int4_gauss_groups.argtypes = [U64, U64, I64, I32, D, D, D, P]
    lib.synth_fp16_uniform.argtypes = [U64, U64, I64, D, D, P]
    lib.synth_u8_uniform.argtypes = [U64, U64, I64, I32, I32, P]
    lib.synth_int8_normal.argtypes = [U64, U64, I64, D, P]
    lib.synth_relu_runs.argtypes = [U64, U64, I64, D, D, D, I64, P]
    lib.synth_lz4_bound.argtypes = [I64]
    lib.synth_lz4_bound.restype = I64
    lib.synth_lz4_compress_block.argtypes = [P, I64, P, ctypes.c_int]
    lib.synth_lz4_compress_block.restype = I64
    lib.synth_lz4_compress_blocks.argtypes = [P, I64, I32, P, P, ctypes.c_int]
    lib.synth_lz4_compress_blocks.restype = I64
    lib.synth_zrle_plan.argtypes = [P, I64, I32, I32, P]
    lib.synth_zrle_plan.restype = I64
    lib.synth_zrle_write.argtypes = [P, I64, I32, P, P]
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def set_threads(n: int) -> None:
    """Threads used by the generator (0 = all online cores). Output does not
    depend on it."""
    _load().synth_set_threads(int(n))


# --------------------------------------------------------------------------
# value laws
# --------------------------------------------------------------------------

def int4_uniform_packed(seed: int, n: int, stream: int = 0) -> np.ndarray:
    """n codes uniform on {0..15}, packed two per byte, even code in the low
    nibble (ceil(n/2) bytes)."""
    out = np.zeros((n + 1) // 2, dtype=np.uint8)
    if n:
        _load().synth_int4_uniform(seed, stream, n, _ptr(out))
    return out


def int4_gauss_groups_packed(seed: int, n: int, group: int = 128, p_const: float = 0.3,
                             mu: float = 8.0, sigma: float = 2.0, stream: int = 0) -> np.ndarray:
    """n codes ~ clip(round(N(mu, sigma)), 0, 15); each aligned run of
    ``group`` codes is constant (one draw repeated) with probability
    ``p_const``. Packed as in :func:`int4_uniform_packed`."""
    if 131072 % group:
        raise ValueError("group must divide 131072")
    out = np.zeros((n + 1) // 2, dtype=np.uint8)
    if n:
        _load().synth_int4_gauss_groups(seed, stream, n, group, p_const, mu, sigma, _ptr(out))
    return out


def fp16_uniform(seed: int, n: int, lo: float, hi: float, stream: int = 0) -> np.ndarray:
    """n fp16 bit patterns (uint16) of fp16_rn(U[lo, hi])."""
    out = np.zeros(n, dtype=np.uint16)
    if n:
        _load().synth_fp16_uniform(seed, stream, n, lo, hi, _ptr(out))
    return out


def u8_uniform(seed: int, n: int, lo: int, hi: int, stream: int = 0) -> np.ndarray:
    """n bytes uniform on the integers {lo..hi}."""
    out = np.zeros(n, dtype=np.uint8)
    if n:
        _load().synth_u8_uniform(seed, stream, n, lo, hi, _ptr(out))
    return out


def int8_normal(seed: int, n: int, sigma: float, stream: int = 0) -> np.ndarray:
    """n int8 values clip(round(N(0, sigma)), -128, 127)."""
    out = np.zeros(n, dtype=np.int8)
    if n:
        _load().synth_int8_normal(seed, stream, n, sigma, _ptr(out))
    return out


def relu_runs(seed: int, n: int, mean_zero_run: float = 20.0, p_nz: float = 9.0 / 20.0,
              p_first_zero: float = 0.9, restart: int = 1 << 20, stream: int = 0) -> np.ndarray:
    """ReLU-like fp16 activations (uint16 bit patterns): alternating zero runs
    (Geometric, mean ``mean_zero_run``) and non-zero runs (Geometric(p_nz)),
    non-zeros fp16_rn(|N(0,1)|) never rounding to +0. The run process restarts
    every ``restart`` elements (for parallel generation)."""
    out = np.zeros(n, dtype=np.uint16)
    if n:
        _load().synth_relu_runs(seed, stream, n, mean_zero_run, p_nz, p_first_zero, restart, _ptr(out))
    return out


# --------------------------------------------------------------------------
# encoders
# --------------------------------------------------------------------------

def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Pack codes in {0..15} two per byte, even code in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8).ravel()
    if c.size and c.max() > 15:
        raise ValueError("codes must be in [0, 15]")
    n = c.size
    out = np.zeros((n + 1) // 2, dtype=np.uint8)
    out[:] = c[0::2]
    out[: n // 2] |= c[1::2] << 4
    return out


def lz4_bound(n: int) -> int:
    return int(_load().synth_lz4_bound(n))


def lz4_compress_block(data: np.ndarray | bytes, force_literals: bool = False) -> np.ndarray:
    """One LZ4 block (raw block format, no frame) for ``data``."""
    src = np.frombuffer(bytes(data), dtype=np.uint8) if not isinstance(data, np.ndarray) else data
    src = np.ascontiguousarray(src, dtype=np.uint8)
    dst = np.zeros(lz4_bound(src.size), dtype=np.uint8)
    m = _load().synth_lz4_compress_block(_ptr(src), src.size, _ptr(dst), int(force_literals))
    return dst[:m].copy()


def lz4_compress_blocks(src: np.ndarray, block_bytes: int = 65536, force_literals: bool = False):
    """Compress ``src`` in independent LZ4 blocks of ``block_bytes``
    (decompressed size; the last block holds the remainder).

    Returns ``(comp, offsets)``: the concatenated blocks (uint8) and
    ``n_blocks + 1`` uint64 byte offsets."""
    src = np.ascontiguousarray(src, dtype=np.uint8).ravel()
    n_blocks = (src.size + block_bytes - 1) // block_bytes
    offsets = np.zeros(n_blocks + 1, dtype=np.uint64)
    dst = np.empty(max(1, n_blocks * lz4_bound(block_bytes)), dtype=np.uint8)
    total = _load().synth_lz4_compress_blocks(_ptr(src), src.size, block_bytes, _ptr(dst),
                                              _ptr(offsets), int(force_literals))
    comp = dst[:total].copy()
    del dst
    return comp, offsets


def zrle_encode(x: np.ndarray, chunk_elems: int = 4096, pad: int = 16):
    """Zero-run encode fp16 bit patterns ``x`` (uint16) per chunk.

    Returns ``(enc, offsets)``: the concatenated chunk streams (uint8) and
    ``n_chunks + 1`` uint64 byte offsets. Each chunk is padded with zero bytes
    to a multiple of ``pad``."""
    x = np.ascontiguousarray(x, dtype=np.uint16).ravel()
    n_chunks = (x.size + chunk_elems - 1) // chunk_elems
    offsets = np.zeros(n_chunks + 1, dtype=np.uint64)
    lib = _load()
    total = lib.synth_zrle_plan(_ptr(x), x.size, chunk_elems, pad, _ptr(offsets))
    enc = np.zeros(max(total, 1), dtype=np.uint8)
    lib.synth_zrle_write(_ptr(x), x.size, chunk_elems, _ptr(offsets), _ptr(enc))
    return enc[:total], offsets
