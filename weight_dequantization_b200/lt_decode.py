"""Python binding of liblt_decode.so (ctypes; argument marshalling only).

Every function has the name and the arguments of the C entry point declared
in ``include/lt_decode.h``. Tensor arguments are CUDA tensors (their device
pointers are passed) or raw integer device addresses; ``None`` is NULL. The
stream defaults to PyTorch's current stream on the output's device. A non-OK
status raises :class:`LtError`. There is no CPU path: CPU tensors are
rejected, and a missing or unloadable library raises at import of this
module's first call.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblt_decode.so")

LT_OK = 0
LT_ERR_INVALID_ARG = 1
LT_ERR_MISALIGNED = 2
LT_ERR_UNSUPPORTED = 3
LT_ERR_CORRUPT_STREAM = 4
LT_ERR_SIZE_MISMATCH = 5
LT_ERR_CUDA = 6
LT_ERR_TIMEOUT = 7
LT_ERR_CHECKSUM = 8
LT_SCALE_PER_TENSOR = 0
LT_SCALE_PER_ROW = 1
LT_LZ4_BATCH_MAX = 64

EXPORTED = (
    "lt_dequant_int4", "lt_dequant_int8", "lt_value_dict_decode", "lt_zrle_decode", "lt_lz4_int4_decode",
    "lt_lz4_int4_decode_batch", "lt_lz4_index_batch", "lt_lz4_int4_expand_batch", "lt_lz4_decode",
    "lt_lz4_workspace_bytes", "lt_lz4_int4_decode_noalloc", "lt_lz4_int4_decode_checked", "lt_xxh3_blocks",
    "lt_int4_gemm",
    "lt_int4_gemm_workspace_bytes",
    "lt_hct2_layout", "lt_hct2_read_header", "lt_hct2_write_header",
    "lt_status_string", "lt_abi_version",
)
LT_NOALLOC_MAX_BLOCKS = 512


class LtError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class LtLz4Int4Desc(ctypes.Structure):
    _fields_ = [
        ("comp", ctypes.c_void_p), ("comp_bytes", ctypes.c_uint64), ("block_offsets", ctypes.c_void_p),
        ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("group_size", ctypes.c_int32),
        ("block_bytes", ctypes.c_int32),
    ]


class LtHct2Header(ctypes.Structure):
    """lt_hct2_header: the stored header fields, then the derived ones."""
    _fields_ = [
        ("version", ctypes.c_uint16), ("compression", ctypes.c_uint8), ("quantization", ctypes.c_uint8),
        ("checksum", ctypes.c_uint8), ("block_size", ctypes.c_uint32), ("rows", ctypes.c_uint64),
        ("cols", ctypes.c_uint64), ("group_size", ctypes.c_uint32), ("secret_len", ctypes.c_uint32),
        ("n_blocks", ctypes.c_uint64), ("payload_bytes", ctypes.c_uint64), ("meta_hash", ctypes.c_uint64),
        ("n_groups", ctypes.c_uint64), ("offsets_at", ctypes.c_uint64), ("hashes_at", ctypes.c_uint64),
        ("scales_at", ctypes.c_uint64), ("zeros_at", ctypes.c_uint64), ("payload_at", ctypes.c_uint64),
        ("total_bytes", ctypes.c_uint64),
    ]


LT_HCT2_VERSION = 2
LT_HCT2_HEADER_BYTES = 64
LT_HCT2_SECRET_MIN = 136

_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load liblt_decode.so (no compute; works without a GPU)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is not built: run __graft_entry__.build() (the decoders have no CPU fallback)")
    lib = ctypes.CDLL(p)
    P, U64, I64, I32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32
    lib.lt_dequant_int4.argtypes = [P, P, P, I64, I64, I32, P, P]
    lib.lt_dequant_int8.argtypes = [P, P, P, I32, I64, I64, P, P]
    lib.lt_value_dict_decode.argtypes = [P, I32, P, I64, P, P]
    lib.lt_zrle_decode.argtypes = [P, U64, P, I64, I32, P, P, P]
    lib.lt_lz4_int4_decode.argtypes = [P, U64, P, I32, P, P, I64, I64, I32, P, P, U64, P, P]
    lib.lt_lz4_int4_decode_batch.argtypes = [ctypes.POINTER(LtLz4Int4Desc), I32, P, U64, P, P]
    lib.lt_lz4_index_batch.argtypes = [ctypes.POINTER(LtLz4Int4Desc), I32, P, U64, P]
    lib.lt_lz4_int4_expand_batch.argtypes = [ctypes.POINTER(LtLz4Int4Desc), I32, P, U64, I64, I64, P, P]
    lib.lt_lz4_decode.argtypes = [P, U64, P, I32, P, U64, P, U64, P, P]
    lib.lt_lz4_int4_decode_noalloc.argtypes = [P, U64, P, I32, P, P, I64, I64, I32, P, P, P]
    lib.lt_lz4_int4_decode_checked.argtypes = [P, U64, P, I32, P, P, I64, I64, I32, P, P, U64, P, I32, P, P, P, P]
    lib.lt_lz4_int4_decode_checked.restype = ctypes.c_int
    lib.lt_lz4_int4_decode_noalloc.restype = ctypes.c_int
    lib.lt_xxh3_blocks.argtypes = [P, U64, P, I64, P, I32, P, P, P, P, P]
    lib.lt_xxh3_blocks.restype = ctypes.c_int
    lib.lt_hct2_layout.argtypes = [ctypes.POINTER(LtHct2Header)]
    lib.lt_hct2_read_header.argtypes = [ctypes.c_char_p, U64, ctypes.POINTER(LtHct2Header)]
    lib.lt_hct2_write_header.argtypes = [ctypes.POINTER(LtHct2Header), ctypes.c_char_p]
    for f in ("lt_hct2_layout", "lt_hct2_read_header", "lt_hct2_write_header"):
        getattr(lib, f).restype = ctypes.c_int
    lib.lt_int4_gemm.argtypes = [P, I64, I64, P, P, P, I64, I32, P, P, U64, P, P]
    lib.lt_int4_gemm.restype = ctypes.c_int
    lib.lt_int4_gemm_workspace_bytes.argtypes = [I64, I64, I64]
    lib.lt_int4_gemm_workspace_bytes.restype = U64
    lib.lt_lz4_workspace_bytes.argtypes = [I64]
    lib.lt_lz4_workspace_bytes.restype = U64
    for f in ("lt_dequant_int4", "lt_dequant_int8", "lt_value_dict_decode", "lt_zrle_decode", "lt_lz4_int4_decode",
              "lt_lz4_int4_decode_batch", "lt_lz4_index_batch", "lt_lz4_int4_expand_batch", "lt_lz4_decode"):
        getattr(lib, f).restype = ctypes.c_int
    lib.lt_status_string.argtypes = [ctypes.c_int]
    lib.lt_status_string.restype = ctypes.c_char_p
    lib.lt_abi_version.argtypes = []
    lib.lt_abi_version.restype = I32
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().lt_status_string(int(status)).decode()


def abi_version() -> int:
    return int(load_library().lt_abi_version())


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    dev = getattr(x, "device", None)
    if dev is None or dev.type != "cuda":
        raise TypeError("liblt_decode takes CUDA tensors or device addresses (there is no CPU path)")
    if not x.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return x.data_ptr()


def _stream(stream, like) -> int | None:
    if stream is None:
        import torch

        dev = getattr(like, "device", None)
        s = torch.cuda.current_stream(dev if dev is not None and dev.type == "cuda" else None)
        return s.cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != LT_OK:
        raise LtError(status, where)


def lt_dequant_int4(packed, scales, zeros, rows: int, cols: int, group_size: int, out, stream=None) -> None:
    _check(load_library().lt_dequant_int4(_ptr(packed), _ptr(scales), _ptr(zeros), rows, cols, group_size,
                                          _ptr(out), _stream(stream, out)), "lt_dequant_int4")


def lt_dequant_int8(q, scales, zeros, scale_mode: int, rows: int, cols: int, out, stream=None) -> None:
    _check(load_library().lt_dequant_int8(_ptr(q), _ptr(scales), _ptr(zeros), scale_mode, rows, cols, _ptr(out),
                                          _stream(stream, out)), "lt_dequant_int8")


def lt_value_dict_decode(packed, bits: int, dictionary, n: int, out, stream=None) -> None:
    _check(load_library().lt_value_dict_decode(_ptr(packed), bits, _ptr(dictionary), n, _ptr(out),
                                               _stream(stream, out)), "lt_value_dict_decode")


def lt_zrle_decode(enc, enc_bytes: int, chunk_offsets, n_elements: int, chunk_elems: int, out, d_status=None,
                   stream=None) -> None:
    _check(load_library().lt_zrle_decode(_ptr(enc), enc_bytes, _ptr(chunk_offsets), n_elements, chunk_elems,
                                         _ptr(out), _ptr(d_status), _stream(stream, out)), "lt_zrle_decode")


def lt_xxh3_blocks(data, data_bytes: int, offsets, n_blocks: int, secret, secret_len: int, hashes=None,
                   expected=None, d_status=None, d_first_bad=None, stream=None) -> None:
    like = hashes if hashes is not None else expected
    _check(load_library().lt_xxh3_blocks(_ptr(data), data_bytes, _ptr(offsets), n_blocks, _ptr(secret), secret_len,
                                         _ptr(hashes), _ptr(expected), _ptr(d_status), _ptr(d_first_bad),
                                         _stream(stream, like)), "lt_xxh3_blocks")


def lt_lz4_workspace_bytes(n_blocks: int) -> int:
    return int(load_library().lt_lz4_workspace_bytes(int(n_blocks)))


def _ws(workspace):
    if workspace is None:
        return None, 0
    if isinstance(workspace, tuple):
        return workspace
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def lt_lz4_int4_decode(comp, comp_bytes: int, block_offsets, block_bytes: int, scales, zeros, rows: int, cols: int,
                       group_size: int, out, workspace=None, d_status=None, stream=None) -> None:
    """``workspace``: a CUDA tensor (its bytes), an (address, bytes) pair, or
    None (correct but slow decode)."""
    wp, wb = _ws(workspace)
    _check(load_library().lt_lz4_int4_decode(_ptr(comp), comp_bytes, _ptr(block_offsets), block_bytes,
                                             _ptr(scales), _ptr(zeros), rows, cols, group_size, _ptr(out), wp, wb,
                                             _ptr(d_status), _stream(stream, out)), "lt_lz4_int4_decode")


def lt_lz4_int4_decode_checked(comp, comp_bytes: int, block_offsets, block_bytes: int, scales, zeros, rows: int,
                               cols: int, group_size: int, out, secret, secret_len: int, expected_hashes,
                               workspace=None, d_status=None, d_first_bad=None, stream=None) -> None:
    """lt_lz4_int4_decode with every compressed block's XXH3-64 checked
    against ``expected_hashes`` first (LT_ERR_CHECKSUM and the first bad
    block in ``d_first_bad``)."""
    wp, wb = _ws(workspace)
    _check(load_library().lt_lz4_int4_decode_checked(
        _ptr(comp), comp_bytes, _ptr(block_offsets), block_bytes, _ptr(scales), _ptr(zeros), rows, cols, group_size,
        _ptr(out), wp, wb, _ptr(secret), secret_len, _ptr(expected_hashes), _ptr(d_status), _ptr(d_first_bad),
        _stream(stream, out)), "lt_lz4_int4_decode_checked")


def lt_lz4_int4_decode_batch(descs: Sequence[dict], workspace=None, d_status=None, stream=None) -> None:
    """``descs``: dicts with the keys of lt_lz4_int4_desc (tensors or addresses)."""
    arr = _desc_array(descs)
    like = descs[0]["out"] if descs else None
    wp, wb = _ws(workspace)
    _check(load_library().lt_lz4_int4_decode_batch(arr, len(descs), wp, wb, _ptr(d_status), _stream(stream, like)),
           "lt_lz4_int4_decode_batch")


def _desc_array(descs: Sequence[dict]):
    arr = (LtLz4Int4Desc * max(len(descs), 1))()
    for i, d in enumerate(descs):
        arr[i] = LtLz4Int4Desc(_ptr(d["comp"]), d["comp_bytes"], _ptr(d["block_offsets"]), _ptr(d["scales"]),
                               _ptr(d.get("zeros")), _ptr(d["out"]), d["rows"], d["cols"], d["group_size"],
                               d["block_bytes"])
    return arr


def desc_blocks(d: dict) -> int:
    """LZ4 blocks of one lt_lz4_int4_desc (as a dict): its numbering width in an index."""
    packed = (d["rows"] * d["cols"] + 1) // 2
    return (packed + d["block_bytes"] - 1) // d["block_bytes"]


def lt_lz4_index_batch(descs: Sequence[dict], index, stream=None) -> None:
    """Sequence index of every block of ``descs`` into ``index`` (a device
    tensor of at least lt_lz4_workspace_bytes(total blocks) bytes)."""
    arr = _desc_array(descs)
    ip, ib = _ws(index)
    like = descs[0]["out"] if descs else None
    _check(load_library().lt_lz4_index_batch(arr, len(descs), ip, ib, _stream(stream, like)), "lt_lz4_index_batch")


def lt_lz4_int4_expand_batch(descs: Sequence[dict], index, index_blocks: int, first_block: int, d_status=None,
                             stream=None) -> None:
    """Decode ``descs`` from an index built by lt_lz4_index_batch over a
    descriptor list of ``index_blocks`` blocks in which these start at block
    ``first_block``."""
    arr = _desc_array(descs)
    ip, ib = _ws(index)
    like = descs[0]["out"] if descs else None
    _check(load_library().lt_lz4_int4_expand_batch(arr, len(descs), ip, ib, index_blocks, first_block,
                                                    _ptr(d_status), _stream(stream, like)),
           "lt_lz4_int4_expand_batch")


def lt_lz4_decode(comp, comp_bytes: int, block_offsets, block_bytes: int, out, out_bytes: int, workspace=None,
                  d_status=None, stream=None) -> None:
    wp, wb = _ws(workspace)
    _check(load_library().lt_lz4_decode(_ptr(comp), comp_bytes, _ptr(block_offsets), block_bytes, _ptr(out),
                                        out_bytes, wp, wb, _ptr(d_status), _stream(stream, out)), "lt_lz4_decode")


def lt_lz4_int4_decode_noalloc(comp, comp_bytes: int, block_offsets, block_bytes: int, scales, zeros, rows: int,
                               cols: int, group_size: int, out, d_status=None, stream=None) -> None:
    """lt_lz4_int4_decode without a workspace argument, for callers that may
    not allocate device memory: the sequence index lives in a scratch array
    built into the library (at most LT_NOALLOC_MAX_BLOCKS blocks per call;
    calls that overlap on the GPU race on it)."""
    _check(load_library().lt_lz4_int4_decode_noalloc(_ptr(comp), comp_bytes, _ptr(block_offsets), block_bytes,
                                                     _ptr(scales), _ptr(zeros), rows, cols, group_size, _ptr(out),
                                                     _ptr(d_status), _stream(stream, out)),
           "lt_lz4_int4_decode_noalloc")


def lt_int4_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(load_library().lt_int4_gemm_workspace_bytes(int(M), int(N), int(K)))


def lt_int4_gemm(x, M: int, K: int, packed, scales, zeros, N: int, group_size: int, out, workspace=None,
                 d_status=None, stream=None) -> None:
    """out[M, N] = x[M, K] @ W[K, N], W the INT4 dequant of ``packed`` /
    ``scales`` / ``zeros`` (lt_dequant_int4's layout with rows = K, cols =
    N), decoded tile by tile into shared memory and multiplied on the tensor
    cores. ``workspace``: optional CUDA tensor (or (address, bytes)) of at
    least lt_int4_gemm_workspace_bytes(M, N, K) bytes for splitting K."""
    wp, wb = _ws(workspace)
    _check(load_library().lt_int4_gemm(_ptr(x), M, K, _ptr(packed), _ptr(scales), _ptr(zeros), N, group_size,
                                       _ptr(out), wp, wb, _ptr(d_status), _stream(stream, out)), "lt_int4_gemm")


# HCT v2 container header: host functions (host memory, no device)
def lt_hct2_layout(h: LtHct2Header) -> LtHct2Header:
    _check(load_library().lt_hct2_layout(ctypes.byref(h)), "lt_hct2_layout")
    return h


def lt_hct2_read_header(buf) -> LtHct2Header:
    b = bytes(buf)
    h = LtHct2Header()
    _check(load_library().lt_hct2_read_header(b, len(b), ctypes.byref(h)), "lt_hct2_read_header")
    return h


def lt_hct2_write_header(h: LtHct2Header) -> bytes:
    out = ctypes.create_string_buffer(LT_HCT2_HEADER_BYTES)
    _check(load_library().lt_hct2_write_header(ctypes.byref(h), out), "lt_hct2_write_header")
    return out.raw
