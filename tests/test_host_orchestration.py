"""Host logic of the container and streaming modules, without a GPU.

hct.py (write / verify / decode) and stream.py (LayerStreamer) only lay out
bytes, slice buffers and order calls; the arithmetic is in the library's
kernels. Here every device call is replaced, for the duration of one test,
by a fake that keeps the C ABI's contract (argument checks, alignment,
status words) and computes with the oracle, and CUDA tensors, streams and
events by their CPU counterparts. The scenarios are those of the GPU tests
(tests/test_gpu_xxh3.py, tests/test_gpu_stream.py), which run the real
kernels; this file checks the offsets, views and call order around them.
"""
from __future__ import annotations

import contextlib
import ctypes
import functools

import numpy as np
import pytest

import oracle
from tests._pins import libxxhash

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.skipif(libxxhash() is None, reason="system libxxhash not present")


def _u8(t):
    return t.numpy().view(np.uint8).ravel()


def _u16(t):
    return t.numpy().view(np.uint16).ravel()


def _mem(addr, n, dt=np.uint8):
    if n == 0:
        return np.zeros(0, dt)
    return np.ctypeslib.as_array((ctypes.c_uint8 * n).from_address(addr)).view(dt)


def _put_out(out, bits):
    o = out.reshape(-1).numpy().view(np.uint16)
    assert o.size == bits.size
    o[:] = bits


def _fake_xxh3(data, data_bytes, offsets, n, secret, secret_len, hashes=None, expected=None, d_status=None,
               d_first_bad=None, stream=None):
    assert secret_len >= 136 and n >= 0 and (hashes is not None or expected is not None)
    if n == 0:
        return
    for t in (offsets, hashes, expected, d_first_bad):
        assert t is None or t.data_ptr() % 8 == 0
    d = _u8(data)[:data_bytes] if data is not None else np.zeros(0, np.uint8)
    offs = offsets.numpy().view(np.uint64)[:n + 1]
    sec = _u8(secret)[:secret_len]
    for b in range(n):
        s0, s1 = int(offs[b]), int(offs[b + 1])
        if s1 < s0 or s1 > data_bytes:
            if d_status is not None and d_status[0] == 0:
                d_status[0] = 4
            continue
        h = oracle.xxh3_64(d[s0:s1], sec)
        if hashes is not None:
            hashes.numpy().view(np.uint64)[b] = h
        if expected is not None and int(expected.numpy().view(np.uint64)[b]) != h:
            if d_status is not None and d_status[0] == 0:
                d_status[0] = 8
            if d_first_bad is not None:
                fb = d_first_bad.numpy().view(np.uint64)
                fb[0] = min(int(fb[0]), b)


def _fake_lz4_int4(comp, comp_bytes, offs, bs, scales, zeros, rows, cols, G, out, ws=None, st=None, stream=None):
    nb = ((rows * cols + 1) // 2 + bs - 1) // bs
    w, s = oracle.lz4_int4_decode(_u8(comp)[:comp_bytes], offs.numpy().view(np.uint64)[:nb + 1], bs,
                                  _u16(scales)[: rows * cols // G],
                                  None if zeros is None else _u8(zeros)[: rows * cols // G], rows, cols, G)
    _put_out(out, w)
    if s and st is not None:
        st[0] = s


def _fake_lz4_checked(comp, comp_bytes, offs, bs, scales, zeros, rows, cols, G, out, secret, secret_len, expected,
                      ws=None, st=None, first=None, stream=None):
    assert secret_len >= 136 and expected is not None and expected.data_ptr() % 8 == 0
    nb = ((rows * cols + 1) // 2 + bs - 1) // bs
    d = _u8(comp)[:comp_bytes]
    o = offs.numpy().view(np.uint64)[:nb + 1]
    sec = _u8(secret)[:secret_len]
    bad = [b for b in range(nb) if oracle.xxh3_64(d[int(o[b]):int(o[b + 1])], sec) !=
           int(expected.numpy().view(np.uint64)[b])]
    if bad:
        if st is not None and st[0] == 0:
            st[0] = 8
        if first is not None:
            fb = first.numpy().view(np.uint64)
            fb[0] = min(int(fb[0]), bad[0])
        return
    _fake_lz4_int4(comp, comp_bytes, offs, bs, scales, zeros, rows, cols, G, out, ws, st, stream)


def _fake_lz4(comp, comp_bytes, offs, bs, out, out_bytes, ws=None, st=None, stream=None):
    nb = (out_bytes + bs - 1) // bs
    w, s = oracle.lz4_decode_blocks(_u8(comp)[:comp_bytes], offs.numpy().view(np.uint64)[:nb + 1], bs, out_bytes)
    o = out.numpy().view(np.uint8).ravel()
    assert o.size == out_bytes
    o[:] = w
    if s and st is not None:
        st[0] = s


def _fake_int4(packed, scales, zeros, rows, cols, G, out, stream=None):
    n = rows * cols
    assert _u8(packed).size >= (n + 1) // 2
    w, _ = oracle.dequant_int4(_u8(packed)[:(n + 1) // 2], _u16(scales)[: n // G],
                               None if zeros is None else _u8(zeros)[: n // G], rows, cols, G)
    _put_out(out, w)


def _fake_int8(q, scales, zeros, mode, rows, cols, out, stream=None):
    n = rows * cols
    assert _u8(q).size >= n
    w, _ = oracle.dequant_int8(_u8(q)[:n].view(np.int8), _u16(scales)[: rows if mode else 1], None, bool(mode),
                               rows, cols)
    _put_out(out, w)


def _fake_batch(descs, ws=None, st=None, stream=None):
    for d in descs:
        n = d["rows"] * d["cols"]
        nb = ((n + 1) // 2 + d["block_bytes"] - 1) // d["block_bytes"]
        G = d["group_size"]
        comp = _mem(d["comp"], d["comp_bytes"])
        offs = _mem(d["block_offsets"], 8 * (nb + 1), np.uint64)
        scales = _mem(d["scales"], 2 * (n // G), np.uint16)
        zeros = None if d["zeros"] is None else _mem(d["zeros"], n // G)
        w, s = oracle.lz4_int4_decode(comp, offs, d["block_bytes"], scales, zeros, d["rows"], d["cols"], G)
        _put_out(d["out"], w)
        if s and st is not None:
            st[0] = s


class _Event:
    def record(self, stream=None):
        pass


class _Stream:
    def wait_event(self, event):
        pass


@pytest.fixture
def cpu_device(monkeypatch):
    from weight_dequantization_b200 import lt_decode as L

    monkeypatch.setattr(torch.Tensor, "cuda", lambda self, *a, **k: self)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self, *a, **k: self)
    for name in ("empty", "zeros", "full"):
        f = getattr(torch, name)

        def wrap(f):
            @functools.wraps(f)
            def g(*a, **k):
                k.pop("device", None)
                return f(*a, **k)
            return g
        monkeypatch.setattr(torch, name, wrap(f))
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: _Event())
    monkeypatch.setattr(torch.cuda, "Stream", lambda *a, **k: _Stream())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _Stream())
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    for name, fake in (("lt_xxh3_blocks", _fake_xxh3), ("lt_lz4_int4_decode", _fake_lz4_int4),
                       ("lt_lz4_int4_decode_checked", _fake_lz4_checked),
                       ("lt_lz4_decode", _fake_lz4), ("lt_dequant_int4", _fake_int4),
                       ("lt_dequant_int8", _fake_int8), ("lt_lz4_int4_decode_batch", _fake_batch)):
        monkeypatch.setattr(L, name, fake)


def test_container_write_verify_decode(cpu_device):
    import tests.test_gpu_xxh3 as T
    T.test_container_written_on_the_device_is_the_reference_layout()
    T.test_container_verified_on_the_device()
    T.test_container_decodes_like_the_oracle()
    T.test_uncompressed_and_raw_containers_decode_like_the_oracle()


def test_layer_streamer_slots_and_views(cpu_device):
    import tests.test_gpu_stream as T
    T.test_streamed_layers_decode_like_the_oracle()
