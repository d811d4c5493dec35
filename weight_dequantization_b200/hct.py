"""HCT v2 containers: a compressed tensor with per-block XXH3-64 checksums
("GPU Compression Pipeline - TDD Roadmap", Phase 6.1 HCT Format V2: a v2
header with compression and quantization metadata and the block size, XXH3
checksums, a flipped byte reported as a checksum mismatch).

Layout (little-endian; the page lists the header as a task and leaves it
undesigned, so this layout is this library's):

  0  "HCT2"   4 version u16 = 2   6 reserved u16
  8  compression u8 (0 none, 1 LZ4 raw blocks)   9 quantization u8 (0 none,
     1 INT4, 2 INT8)   10 checksum u8 (1 XXH3-64)   11 reserved u8
  12 block_size u32   16 rows u64   24 cols u64   32 group_size u32
  36 secret_len u32   40 n_blocks u64   48 payload_bytes u64   56 meta_hash u64
  64 the XXH3 secret (secret_len >= 136 bytes), then from 16-byte boundaries:
     block offsets u64[n_blocks + 1] (relative to the payload), block hashes
     u64[n_blocks], scales fp16[n_groups], zero points u8[n_groups] (INT4
     only), and the payload (the compressed blocks), which ends the file.

meta_hash is XXH3-64 of every byte before the payload with the meta_hash
field read as zero; block hash b covers the payload bytes of block b. The
header is laid out, parsed and written by the library's host functions
(``lt_hct2_layout``, ``lt_hct2_read_header``, ``lt_hct2_write_header``) and
all hashing runs on the device through ``lt_xxh3_blocks``; this module only
moves bytes.
"""
from __future__ import annotations

import struct

import numpy as np

from . import lt_decode as L

SECRET_MIN = L.LT_HCT2_SECRET_MIN
HEADER_BYTES = L.LT_HCT2_HEADER_BYTES
COMPRESSION_NONE, COMPRESSION_LZ4 = 0, 1
QUANT_NONE, QUANT_INT4, QUANT_INT8 = 0, 1, 2
CHECKSUM_XXH3 = 1


class HctError(ValueError):
    pass


def make_header(compression: int, quantization: int, block_size: int, rows: int, cols: int, group_size: int,
                secret_len: int, n_blocks: int, payload_bytes: int, meta_hash: int = 0) -> L.LtHct2Header:
    """A header with its sections laid out (lt_hct2_layout)."""
    h = L.LtHct2Header(version=L.LT_HCT2_VERSION, compression=compression, quantization=quantization,
                       checksum=CHECKSUM_XXH3, block_size=block_size, rows=rows, cols=cols, group_size=group_size,
                       secret_len=secret_len, n_blocks=n_blocks, payload_bytes=payload_bytes, meta_hash=meta_hash)
    try:
        return L.lt_hct2_layout(h)
    except L.LtError as e:
        raise HctError(str(e)) from e


def read_header(buf) -> L.LtHct2Header:
    """Parse and check the header of a whole container (no checksum is
    checked here)."""
    try:
        return L.lt_hct2_read_header(buf)
    except L.LtError as e:
        raise HctError(str(e)) from e


def sections(h: L.LtHct2Header) -> dict:
    """Byte offsets of the sections, and the end of the container."""
    return {"offsets": h.offsets_at, "hashes": h.hashes_at, "scales": h.scales_at, "zeros": h.zeros_at,
            "payload": h.payload_at, "end": h.total_bytes}


def _device_hashes(data_dev, data_bytes: int, offsets, secret_dev, secret_len: int):
    import torch

    n = len(offsets) - 1
    offs = torch.from_numpy(np.asarray(offsets, np.uint64).view(np.int64).copy()).cuda()
    hashes = torch.empty(max(n, 1), dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lt_xxh3_blocks(data_dev, data_bytes, offs, n, secret_dev, secret_len, hashes, None, status, None)
    if int(status.item()) != 0:
        raise HctError(f"hashing failed: {L.status_string(int(status.item()))}")
    return [int(x) for x in hashes.cpu().numpy().view(np.uint64)[:n]]


def write(blocks, block_size: int, rows: int, cols: int, quantization: int, group_size: int = 0, scales=None,
          zeros=None, secret: bytes = b"", compression: int = COMPRESSION_LZ4) -> bytes:
    """Lay out a container around already-compressed ``blocks`` (a list of
    byte strings, in order), hashing on the device."""
    import torch

    if len(secret) < SECRET_MIN:
        raise HctError(f"the XXH3 secret holds at least {SECRET_MIN} bytes")
    payload = b"".join(bytes(x) for x in blocks)
    offs = np.zeros(len(blocks) + 1, np.uint64)
    offs[1:] = np.cumsum([len(x) for x in blocks], dtype=np.uint64)
    hdr = make_header(compression, quantization, block_size, rows, cols, group_size, len(secret), len(blocks),
                      len(payload))
    sec = sections(hdr)
    sc = b"" if scales is None else np.ascontiguousarray(scales, np.uint16).tobytes()
    ze = b"" if zeros is None else np.ascontiguousarray(zeros, np.uint8).tobytes()
    if len(sc) != 2 * hdr.n_groups or len(ze) != (hdr.n_groups if quantization == QUANT_INT4 else 0):
        raise HctError("scales / zero points do not match the shape and quantization")
    meta = bytearray(sec["payload"])
    meta[:HEADER_BYTES] = L.lt_hct2_write_header(hdr)
    meta[HEADER_BYTES:HEADER_BYTES + len(secret)] = secret
    meta[sec["offsets"]:sec["offsets"] + offs.nbytes] = offs.tobytes()
    meta[sec["scales"]:sec["scales"] + len(sc)] = sc
    meta[sec["zeros"]:sec["zeros"] + len(ze)] = ze

    secret_dev = torch.frombuffer(bytearray(secret), dtype=torch.uint8).cuda()
    pay_dev = torch.frombuffer(bytearray(payload), dtype=torch.uint8).cuda() if payload else None
    hashes = _device_hashes(pay_dev, len(payload), offs, secret_dev, len(secret))
    meta[sec["hashes"]:sec["hashes"] + 8 * len(hashes)] = struct.pack(f"<{len(hashes)}Q", *hashes)
    meta_dev = torch.frombuffer(bytearray(meta), dtype=torch.uint8).cuda()
    (mh,) = _device_hashes(meta_dev, len(meta), [0, len(meta)], secret_dev, len(secret))
    meta[56:64] = struct.pack("<Q", mh)
    return bytes(meta) + payload


def _meta_ok(buf, h, sec, dev):
    """The metadata hash (every byte before the payload, meta_hash read as
    zero) checked on the device, and the block offsets' consistency."""
    import torch

    secret_dev = dev[HEADER_BYTES:HEADER_BYTES + h.secret_len]
    meta = bytearray(bytes(buf[:sec["payload"]]))
    meta[56:64] = bytes(8)
    meta_dev = torch.frombuffer(meta, dtype=torch.uint8).cuda()
    (mh,) = _device_hashes(meta_dev, len(meta), [0, len(meta)], secret_dev, h.secret_len)
    offs = np.frombuffer(bytes(buf[sec["offsets"]:sec["offsets"] + 8 * (h.n_blocks + 1)]), np.uint64)
    return (mh == h.meta_hash and offs[0] == 0 and offs[-1] == h.payload_bytes
            and not np.any(np.diff(offs.astype(np.int64)) < 0))


def verify(buf):
    """Check a container's checksums on the device (PyTorch's current
    stream). Returns (ok, first bad block or None, meta_ok)."""
    import torch

    h = read_header(buf)
    sec = sections(h)
    dev = torch.frombuffer(bytearray(bytes(buf)), dtype=torch.uint8).cuda()
    if not _meta_ok(buf, h, sec, dev):
        return False, None, False
    if h.n_blocks == 0:
        return True, None, True
    secret_dev = dev[HEADER_BYTES:HEADER_BYTES + h.secret_len]
    payload = dev[sec["payload"]:]
    stored = dev[sec["hashes"]:sec["hashes"] + 8 * h.n_blocks].view(torch.int64)
    offs_dev = dev[sec["offsets"]:sec["offsets"] + 8 * (h.n_blocks + 1)].view(torch.int64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int64, device="cuda")  # all ones: no block yet
    L.lt_xxh3_blocks(payload if h.payload_bytes else None, h.payload_bytes, offs_dev, h.n_blocks, secret_dev,
                     h.secret_len, None, stored, status, first)
    st = int(status.item())
    if st == 0:
        return True, None, True
    if st != L.LT_ERR_CHECKSUM:
        raise HctError(L.status_string(st))
    return False, int(first.item()), True


def decode(buf, check: bool = True):
    """Decode a container on the device into a new fp16 [rows, cols] tensor,
    after checking its checksums (``check``). LZ4 + INT4 takes the fused
    decode, INT4 and INT8 the dequant kernels, LZ4 of raw fp16 the LZ4
    decoder. Raises HctError on a checksum mismatch, a corrupt stream or a
    combination no kernel implements (LZ4 + INT8)."""
    import torch

    h = read_header(buf)
    if h.compression == COMPRESSION_LZ4 and h.quantization == QUANT_INT8:
        raise HctError("LZ4-compressed INT8 has no decoder")
    sec = sections(h)
    # LZ4 + INT4: the payload blocks are checked inside the decode itself
    # (lt_lz4_int4_decode_checked: each block's hash while it is read for
    # decoding); every other kind is verified first
    fused_check = check and h.compression == COMPRESSION_LZ4 and h.quantization == QUANT_INT4
    if check and not fused_check:
        ok, bad, meta_ok = verify(buf)
        if not ok:
            raise HctError("metadata checksum mismatch" if not meta_ok else f"checksum mismatch in block {bad}")
    n = h.rows * h.cols
    # bytes the decoded stream must hold: packed INT4, INT8 or raw fp16
    need = {QUANT_INT4: (n + 1) // 2, QUANT_INT8: n, QUANT_NONE: 2 * n}[h.quantization]
    if h.compression == COMPRESSION_LZ4:
        if h.n_blocks != (need + h.block_size - 1) // h.block_size:
            raise HctError(f"{h.n_blocks} blocks of {h.block_size} bytes cannot hold {need} bytes")
    elif h.payload_bytes < need:
        raise HctError(f"the payload holds {h.payload_bytes} bytes, the shape needs {need}")
    dev = torch.frombuffer(bytearray(bytes(buf)), dtype=torch.uint8).cuda()
    if fused_check and not _meta_ok(buf, h, sec, dev):
        raise HctError("metadata checksum mismatch")
    out = torch.empty((h.rows, h.cols), dtype=torch.float16, device="cuda")
    if n == 0:
        return out
    payload = dev[sec["payload"]:]
    offs = dev[sec["offsets"]:sec["offsets"] + 8 * (h.n_blocks + 1)].view(torch.int64)
    scales = dev[sec["scales"]:sec["scales"] + 2 * h.n_groups].view(torch.float16)
    zeros = dev[sec["zeros"]:sec["zeros"] + h.n_groups] if h.quantization == QUANT_INT4 else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = None
    if h.compression == COMPRESSION_LZ4 and h.quantization == QUANT_INT4:
        ws = torch.empty(max(L.lt_lz4_workspace_bytes(h.n_blocks), 16), dtype=torch.uint8, device="cuda")
        if fused_check:
            stored = dev[sec["hashes"]:sec["hashes"] + 8 * h.n_blocks].view(torch.int64)
            first = torch.full((1,), -1, dtype=torch.int64, device="cuda")  # all ones: no block yet
            L.lt_lz4_int4_decode_checked(payload, h.payload_bytes, offs, h.block_size, scales, zeros, h.rows, h.cols,
                                         h.group_size, out, dev[HEADER_BYTES:HEADER_BYTES + h.secret_len],
                                         h.secret_len, stored, ws, status, first)
        else:
            L.lt_lz4_int4_decode(payload, h.payload_bytes, offs, h.block_size, scales, zeros, h.rows, h.cols,
                                 h.group_size, out, ws, status)
    elif h.compression == COMPRESSION_LZ4 and h.quantization == QUANT_NONE:
        ws = torch.empty(max(L.lt_lz4_workspace_bytes(h.n_blocks), 16), dtype=torch.uint8, device="cuda")
        L.lt_lz4_decode(payload, h.payload_bytes, offs, h.block_size, out.view(torch.uint8).view(-1), 2 * n, ws,
                        status)
    elif h.compression == COMPRESSION_NONE and h.quantization == QUANT_INT4:
        L.lt_dequant_int4(payload, scales, zeros, h.rows, h.cols, h.group_size, out)
    elif h.compression == COMPRESSION_NONE and h.quantization == QUANT_INT8:
        L.lt_dequant_int8(payload, scales, None, L.LT_SCALE_PER_ROW, h.rows, h.cols, out)
    else:  # neither compressed nor quantized: the payload is the fp16 tensor
        out.view(torch.uint8).view(-1).copy_(payload[:2 * n])
    st = int(status.item())
    if st == L.LT_ERR_CHECKSUM and first is not None:
        raise HctError(f"checksum mismatch in block {int(first.item())}")
    if st != 0:
        raise HctError(L.status_string(st))
    return out
