"""Streaming decode of LZ4 + INT4 layers from pinned host memory
("GPU Compression Pipeline - TDD Roadmap", Phase 5.1 Async Decompression
with CUDA Streams: overlap the host-to-device transfer of layer N with the
decompression of layer N-1; the result must equal sequential loading).

Each layer's compressed inputs (for every matrix: LZ4 blocks, block offsets,
scales, zero points) are packed once into one pinned host buffer. Two device
staging slots alternate: while layer i decodes from slot i % 2 into the one
reused fp16 output buffer on the compute stream, layer i + 1 is copied into
the other slot on a copy stream. Events order the three hazards: a decode
waits for its layer's copy; a copy into a slot waits for the decode that last
read the slot; the next decode overwrites the output only after the
consumer's work for the previous layer, which runs on the compute stream.
"""
from __future__ import annotations

import numpy as np

from . import lt_decode as L

_ALIGN = 256


def _r(x: int) -> int:
    return (x + _ALIGN - 1) // _ALIGN * _ALIGN


class LayerStreamer:
    """``layers``: one list per layer of matrix dicts with the host (numpy)
    arrays ``comp`` (uint8), ``offsets`` (uint64, n_blocks + 1), ``scales``
    (fp16 bits as uint16), ``zeros`` (uint8 or None) and the ints ``rows``,
    ``cols``, ``group_size``, ``block_bytes``; at most LT_LZ4_BATCH_MAX
    matrices per layer."""

    def __init__(self, layers):
        import torch

        if not layers:
            raise ValueError("no layers")
        self.torch = torch
        self.layers = []  # per layer: (pinned host buffer, nbytes, [per-matrix dict of offsets and shape])
        max_bytes, max_elems, max_blocks = 0, 0, 0
        for mats in layers:
            if not 1 <= len(mats) <= L.LT_LZ4_BATCH_MAX:
                raise ValueError(f"a layer holds 1 to {L.LT_LZ4_BATCH_MAX} matrices")
            at, placed, parts = 0, [], []
            elems = blocks = 0
            for m in mats:
                entry = {k: m[k] for k in ("rows", "cols", "group_size", "block_bytes")}
                entry["comp_bytes"] = int(m["comp"].size)
                for key in ("comp", "offsets", "scales", "zeros"):
                    a = m.get(key)
                    if a is None:
                        entry[key] = None
                        continue
                    b = np.ascontiguousarray(a).view(np.uint8).ravel()
                    entry[key] = at
                    parts.append((at, b))
                    at = _r(at + b.size)
                entry["out_at"] = elems
                elems += m["rows"] * m["cols"]
                blocks += len(m["offsets"]) - 1
                placed.append(entry)
            host = torch.empty(max(at, 1), dtype=torch.uint8).pin_memory()
            hv = host.numpy()
            for off, b in parts:
                hv[off:off + b.size] = b
            self.layers.append((host, at, placed))
            max_bytes, max_elems, max_blocks = max(max_bytes, at), max(max_elems, elems), max(max_blocks, blocks)
        self.slots = [torch.empty(max(max_bytes, 1), dtype=torch.uint8, device="cuda") for _ in range(2)]
        self.out = torch.empty(max_elems, dtype=torch.float16, device="cuda")
        self.ws = torch.empty(max(L.lt_lz4_workspace_bytes(max_blocks), 16), dtype=torch.uint8, device="cuda")
        self.d_status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.copy_stream = torch.cuda.Stream()

    def _descs(self, i: int, slot):
        base = slot.data_ptr()
        descs, views = [], []
        for e in self.layers[i][2]:
            n = e["rows"] * e["cols"]
            out = self.out[e["out_at"]:e["out_at"] + n]
            descs.append(dict(comp=base + e["comp"], comp_bytes=e["comp_bytes"], block_offsets=base + e["offsets"],
                              scales=base + e["scales"], zeros=None if e["zeros"] is None else base + e["zeros"],
                              out=out, rows=e["rows"], cols=e["cols"], group_size=e["group_size"],
                              block_bytes=e["block_bytes"]))
            views.append(out.view(e["rows"], e["cols"]))
        return descs, views

    def _copy(self, i: int, freed):
        torch = self.torch
        host, nbytes, _ = self.layers[i]
        slot = self.slots[i % 2]
        self.copy_stream.wait_event(freed[i % 2])
        with torch.cuda.stream(self.copy_stream):
            if nbytes:
                slot[:nbytes].copy_(host[:nbytes], non_blocking=True)
        done = torch.cuda.Event()
        done.record(self.copy_stream)
        return done

    def run(self, consume=None, stream=None):
        """Enqueue the whole sweep. ``consume(i, views)`` is called once per
        layer with fp16 [rows, cols] views of its matrices in the reused
        buffer, under the compute stream, so that the work it enqueues runs
        before the next layer overwrites them. Returns without synchronizing;
        ``status()`` reads the decoders' device status afterwards."""
        torch = self.torch
        s = stream if stream is not None else torch.cuda.current_stream()
        n = len(self.layers)
        # freed[k]: the last decode that read slot k (first: all earlier work on s)
        freed = [torch.cuda.Event(), torch.cuda.Event()]
        for e in freed:
            e.record(s)
        copied = [None] * n
        copied[0] = self._copy(0, freed)
        for i in range(n):
            if i + 1 < n:  # into the slot decode i - 1 read; overlaps decode i
                copied[i + 1] = self._copy(i + 1, freed)
            s.wait_event(copied[i])
            descs, views = self._descs(i, self.slots[i % 2])
            L.lt_lz4_int4_decode_batch(descs, self.ws, self.d_status, s)
            freed[i % 2].record(s)
            if consume is not None:
                with torch.cuda.stream(s):
                    consume(i, views)

    def run_sequential(self, consume=None, stream=None):
        """Sequential loading, the baseline the roadmap's streaming test
        compares against: each layer is copied into slot 0 and then decoded,
        both on the compute stream, so no copy overlaps a decode. Same
        results as ``run``."""
        torch = self.torch
        s = stream if stream is not None else torch.cuda.current_stream()
        slot = self.slots[0]
        for i, (host, nbytes, _) in enumerate(self.layers):
            with torch.cuda.stream(s):
                if nbytes:
                    slot[:nbytes].copy_(host[:nbytes], non_blocking=True)
            descs, views = self._descs(i, slot)
            L.lt_lz4_int4_decode_batch(descs, self.ws, self.d_status, s)
            if consume is not None:
                with torch.cuda.stream(s):
                    consume(i, views)

    def status(self) -> int:
        """The first error status of the decodes so far (0: none); waits for
        the device."""
        self.torch.cuda.synchronize()
        return int(self.d_status.item())
