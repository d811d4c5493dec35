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
field read as zero; block hash b covers the payload bytes of block b. All
hashing runs on the device through ``lt_xxh3_blocks``; this module only
lays out and parses bytes on the host.
"""
from __future__ import annotations

import struct
from dataclasses import dataclass

import numpy as np

from . import lt_decode as L

MAGIC = b"HCT2"
VERSION = 2
HEADER_BYTES = 64
SECRET_MIN = 136
COMPRESSION_NONE, COMPRESSION_LZ4 = 0, 1
QUANT_NONE, QUANT_INT4, QUANT_INT8 = 0, 1, 2
CHECKSUM_XXH3 = 1
_HEADER = struct.Struct("<4sHHBBBBIQQIIQQQ")


def _r16(x: int) -> int:
    return (x + 15) & ~15


@dataclass(frozen=True)
class Header:
    compression: int
    quantization: int
    block_size: int
    rows: int
    cols: int
    group_size: int
    secret_len: int
    n_blocks: int
    payload_bytes: int
    meta_hash: int = 0
    version: int = VERSION
    checksum: int = CHECKSUM_XXH3

    @property
    def n_groups(self) -> int:
        if self.quantization == QUANT_INT4:
            return self.rows * self.cols // self.group_size
        if self.quantization == QUANT_INT8:
            return self.rows
        return 0

    def sections(self) -> dict:
        """Byte offsets of the sections (and the end of the container)."""
        at = _r16(HEADER_BYTES + self.secret_len)
        out = {"offsets": at}
        at = _r16(at + 8 * (self.n_blocks + 1))
        out["hashes"] = at
        at = _r16(at + 8 * self.n_blocks)
        out["scales"] = at
        at = _r16(at + 2 * self.n_groups)
        out["zeros"] = at
        at = _r16(at + (self.n_groups if self.quantization == QUANT_INT4 else 0))
        out["payload"] = at
        out["end"] = at + self.payload_bytes
        return out

    def pack(self) -> bytes:
        return _HEADER.pack(MAGIC, self.version, 0, self.compression, self.quantization, self.checksum, 0,
                            self.block_size, self.rows, self.cols, self.group_size, self.secret_len, self.n_blocks,
                            self.payload_bytes, self.meta_hash)


class HctError(ValueError):
    pass


def read_header(buf) -> Header:
    """Parse and sanity-check the header (no checksum is checked here)."""
    b = bytes(buf[:HEADER_BYTES])
    if len(b) < HEADER_BYTES:
        raise HctError("shorter than the 64-byte header")
    (magic, version, _, compression, quantization, checksum, _, block_size, rows, cols, group_size, secret_len,
     n_blocks, payload_bytes, meta_hash) = _HEADER.unpack(b)
    if magic != MAGIC or version != VERSION:
        raise HctError("not an HCT v2 container")
    if compression > 1 or quantization > 2 or checksum != CHECKSUM_XXH3 or secret_len < SECRET_MIN:
        raise HctError("unsupported header fields")
    if block_size == 0 or n_blocks > (1 << 40) or (cols and rows > (1 << 50) // cols):
        raise HctError("sizes out of range")
    if quantization == QUANT_INT4 and (group_size == 0 or cols % group_size):
        raise HctError("group_size must divide cols")
    h = Header(compression, quantization, block_size, rows, cols, group_size, secret_len, n_blocks, payload_bytes,
               meta_hash, version, checksum)
    if h.sections()["end"] != len(buf):
        raise HctError(f"container is {len(buf)} bytes, its header says {h.sections()['end']}")
    return h


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
    hdr = Header(compression, quantization, block_size, rows, cols, group_size, len(secret), len(blocks),
                 len(payload))
    sec = hdr.sections()
    sc = b"" if scales is None else np.ascontiguousarray(scales, np.uint16).tobytes()
    ze = b"" if zeros is None else np.ascontiguousarray(zeros, np.uint8).tobytes()
    if len(sc) != 2 * hdr.n_groups or len(ze) != (hdr.n_groups if quantization == QUANT_INT4 else 0):
        raise HctError("scales / zero points do not match the shape and quantization")
    meta = bytearray(sec["payload"])
    meta[:HEADER_BYTES] = hdr.pack()
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


def verify(buf):
    """Check a container's checksums on the device (PyTorch's current
    stream). Returns (ok, first bad block or None, meta_ok)."""
    import torch

    h = read_header(buf)
    sec = h.sections()
    dev = torch.frombuffer(bytearray(bytes(buf)), dtype=torch.uint8).cuda()
    secret_dev = dev[HEADER_BYTES:HEADER_BYTES + h.secret_len]
    meta = bytearray(bytes(buf[:sec["payload"]]))
    meta[56:64] = bytes(8)
    meta_dev = torch.frombuffer(meta, dtype=torch.uint8).cuda()
    (mh,) = _device_hashes(meta_dev, len(meta), [0, len(meta)], secret_dev, h.secret_len)
    meta_ok = mh == h.meta_hash
    offs = np.frombuffer(bytes(buf[sec["offsets"]:sec["offsets"] + 8 * (h.n_blocks + 1)]), np.uint64)
    if not meta_ok or offs[0] != 0 or offs[-1] != h.payload_bytes or np.any(np.diff(offs.astype(np.int64)) < 0):
        return False, None, False
    if h.n_blocks == 0:
        return True, None, True
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
