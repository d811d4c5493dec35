"""The five decode workloads, as seeded synthetic host arrays.

Each builder returns a dict of numpy arrays plus the shape parameters the
decoders take. ``scale`` shrinks the workload for parity tests (the value
laws and the layout stay the same; only the element count changes).

  C1  INT4 group dequant: 1,048,576 codes uniform on {0..15} as a
      [1024, 1024] tensor, group 256, fp16 scales fp16_rn(U[0.001, 0.1]),
      uint8 zero points uniform on {0..15}.                       seed 1
  C2  INT8 per-row dequant: [8192, 8192] int8 clip(round(N(0, 32))),
      one fp16 scale per row fp16_rn(U[0.001, 0.02]), zero point 0. seed 2
  C3  Zero-run decode: 8 x 2048 x 11008 fp16 ReLU-like activations, ~90 %
      zeros in runs of mean length 20, non-zeros |N(0, 1)|; chunks of 4096
      elements.                                                    seed 3
  C4  Fused LZ4 + INT4: [4096, 14336] codes clip(round(N(8, 2)), 0, 15),
      30 % of the 128-code groups constant; group 128 with C1's scale and
      zero-point laws; packed, then LZ4-compressed in independent 64 KB
      blocks.                                                      seed 4
  C5  Llama-2-70B-shaped sweep: 8 layers x {q, o: 8192 x 8192; k, v:
      8192 x 1024; gate, up: 8192 x 28672; down: 28672 x 8192}, C4's law and
      layout; one stream id per (layer, matrix).                   seed 5
  V   Value-dictionary decode: [4096, 14336] (C4's shape), 4-bit indices
      with C4's code law (clip(round(N(8, 2)), 0, 15), 30 % of the
      128-index runs constant), one dictionary of 16 fp16 entries
      fp16_rn(U[-0.1, 0.1]). Other widths (1, 2, 8 bits) take uniform
      random index bytes.                                          seed 6
"""
from __future__ import annotations

import numpy as np

from . import (fp16_uniform, int4_gauss_groups_packed, int4_uniform_packed, int8_normal, lz4_compress_blocks,
               relu_runs, u8_uniform, zrle_encode)

LZ4_BLOCK = 65536
ZRLE_CHUNK = 4096

LLAMA70B_MATRICES = (
    ("q", 8192, 8192),
    ("o", 8192, 8192),
    ("k", 8192, 1024),
    ("v", 8192, 1024),
    ("gate", 8192, 28672),
    ("up", 8192, 28672),
    ("down", 28672, 8192),
)
LLAMA70B_LAYERS = 8


def c1_int4(scale: float = 1.0, seed: int = 1):
    rows = max(1, int(round(1024 * scale)))
    cols, G = 1024, 256
    n = rows * cols
    return dict(
        kind="int4", rows=rows, cols=cols, group_size=G,
        packed=int4_uniform_packed(seed, n, stream=0),
        scales=fp16_uniform(seed, n // G, 0.001, 0.1, stream=1),
        zeros=u8_uniform(seed, n // G, 0, 15, stream=2),
    )


def worked_example_int4():
    """The roadmap's INT4 worked example: packed [0x10, 0x32, 0x54, 0x76]
    (codes 0..7), one group, scale fp16(0.5), zero point 0."""
    return dict(kind="int4", rows=1, cols=8, group_size=8,
                packed=np.array([0x10, 0x32, 0x54, 0x76], dtype=np.uint8),
                scales=np.array([0x3800], dtype=np.uint16),
                zeros=np.array([0], dtype=np.uint8))


def c2_int8(scale: float = 1.0, seed: int = 2):
    rows = max(1, int(round(8192 * scale)))
    cols = 8192
    return dict(
        kind="int8", rows=rows, cols=cols, per_row=True,
        q=int8_normal(seed, rows * cols, 32.0, stream=0),
        scales=fp16_uniform(seed, rows, 0.001, 0.02, stream=1),
        zeros=None,
    )


def c3_zrle(scale: float = 1.0, seed: int = 3):
    n_full = 8 * 2048 * 11008
    n = max(1, int(round(n_full * scale)))
    x = relu_runs(seed, n, mean_zero_run=20.0, p_nz=9.0 / 20.0, p_first_zero=0.9, stream=0)
    enc, offsets = zrle_encode(x, ZRLE_CHUNK, pad=16)
    return dict(kind="zrle", n=n, chunk_elems=ZRLE_CHUNK, enc=enc, offsets=offsets, x=x)


def _lz4_int4_matrix(seed: int, stream: int, rows: int, cols: int, G: int = 128):
    n = rows * cols
    packed = int4_gauss_groups_packed(seed, n, group=G, p_const=0.3, mu=8.0, sigma=2.0, stream=3 * stream)
    comp, offsets = lz4_compress_blocks(packed, LZ4_BLOCK)
    return dict(
        kind="lz4_int4", rows=rows, cols=cols, group_size=G, block_bytes=LZ4_BLOCK,
        comp=comp, offsets=offsets, packed_bytes=packed.size,
        scales=fp16_uniform(seed, n // G, 0.001, 0.1, stream=3 * stream + 1),
        zeros=u8_uniform(seed, n // G, 0, 15, stream=3 * stream + 2),
    ), packed


def c4_lz4_int4(scale: float = 1.0, seed: int = 4, keep_packed: bool = False):
    rows = max(1, int(round(4096 * scale)))
    d, packed = _lz4_int4_matrix(seed, 0, rows, 14336)
    if keep_packed:
        d["packed"] = packed
    return d


def c5_layers(layers: int = LLAMA70B_LAYERS, scale: float = 1.0, seed: int = 5, keep_packed: bool = False):
    """List (per layer) of lists (per matrix) of C4-style matrix dicts."""
    out = []
    for layer in range(layers):
        mats = []
        for mi, (name, r, c) in enumerate(LLAMA70B_MATRICES):
            rr = max(1, int(round(r * scale)))
            d, packed = _lz4_int4_matrix(seed, layer * len(LLAMA70B_MATRICES) + mi, rr, c)
            d["name"] = name
            if keep_packed:
                d["packed"] = packed
            mats.append(d)
        out.append(mats)
    return out


def v_value_dict(scale: float = 1.0, seed: int = 6, bits: int = 4):
    if bits not in (1, 2, 4, 8):
        raise ValueError("bits is 1, 2, 4 or 8")
    rows = max(1, int(round(4096 * scale)))
    cols = 14336
    n = rows * cols
    if bits == 4:
        packed = int4_gauss_groups_packed(seed, n, group=128, p_const=0.3, mu=8.0, sigma=2.0, stream=0)
    else:
        packed = u8_uniform(seed, (n * bits + 7) // 8, 0, 255, stream=0)
    return dict(kind="value_dict", rows=rows, cols=cols, n=n, bits=bits, packed=packed,
                dictionary=fp16_uniform(seed, 1 << bits, -0.1, 0.1, stream=1))
