"""GPU parity: zero-run decoding vs the CPU oracle (bit-exact, and the same
device status)."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
from tests._gpu import dev, f16_out, host_bits, need_gpu, status_buf, torch
from tests._pins import hexbytes
from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import relu_runs, zrle_encode
from weight_dequantization_b200.synth import workloads as W

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(12)


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def run_zrle(enc, offsets, n, chunk, out_offset=0, enc_shift=0):
    """enc_shift > 0 places the stream that many bytes into the device buffer
    (and moves the offsets with it) to exercise unaligned chunk starts."""
    if enc_shift:
        enc = np.concatenate([np.zeros(enc_shift, np.uint8), enc])
        offsets = offsets + np.uint64(enc_shift)
    out = f16_out(n, out_offset)
    stat = status_buf()
    L.lt_zrle_decode(dev(enc) if enc.size else None, int(enc.size), dev(offsets), n, chunk, out, stat)
    torch.cuda.synchronize()
    return host_bits(out), int(stat.item())


def test_zrle_handmade(golden_dir):
    cases = json.load(open(os.path.join(golden_dir, "zrle_handmade.json")))["cases"]
    for c in cases:
        enc = np.frombuffer(hexbytes(c["enc"]), np.uint8)
        offs = np.array(c["offsets"], np.uint64)
        want, st_o = oracle.zrle_decode(enc, offs, c["n"], c["chunk"])
        got, st_g = run_zrle(enc, offs, c["n"], c["chunk"])
        assert st_g == st_o == c["status"], c["name"]
        if c["status"] == 0:
            assert list(got) == c["out"], c["name"]


def test_zrle_c3_full_size():
    d = W.c3_zrle()
    want, st = oracle.zrle_decode(d["enc"], d["offsets"], d["n"], d["chunk_elems"])
    assert st == 0
    got, st_g = run_zrle(d["enc"], d["offsets"], d["n"], d["chunk_elems"])
    assert st_g == 0
    assert np.array_equal(got, want)
    assert np.array_equal(got, d["x"])


@pytest.mark.parametrize("n,chunk,pad,out_offset,enc_shift", [
    (1, 1, 1, 0, 0), (4096, 4096, 16, 0, 0), (100_003, 4096, 16, 0, 0),   # ragged tail chunk
    (50_000, 7, 1, 0, 0), (50_000, 64, 2, 0, 0), (70_000, 8192, 16, 0, 0),
    (70_000, 8193, 16, 0, 0), (200_000, 65535, 16, 0, 0),                  # direct (untiled) path
    (30_000, 4096, 16, 3, 0), (30_000, 4096, 16, 0, 1), (30_000, 4096, 2, 0, 6),  # unaligned out / stream
    (30_000, 1000, 16, 0, 0),                                               # chunk not a multiple of 8
])
def test_zrle_shapes(n, chunk, pad, out_offset, enc_shift):
    x = relu_runs(n + chunk, n)
    enc, offs = zrle_encode(x, chunk, pad=pad)
    got, st = run_zrle(enc, offs, n, chunk, out_offset, enc_shift)
    assert st == 0
    assert np.array_equal(got, x)


def test_zrle_dense_and_all_zero_inputs():
    for x in (np.zeros(10_000, np.uint16), RNG.integers(1, 0x7C00, 10_000).astype(np.uint16),
              np.full(10_000, 0x8000, np.uint16)):
        enc, offs = zrle_encode(x, 4096)
        got, st = run_zrle(enc, offs, x.size, 4096)
        assert st == 0 and np.array_equal(got, x)


def test_zrle_corrupt_streams_match_oracle_status():
    x = relu_runs(21, 4096)
    enc, offs = zrle_encode(x, 4096, pad=16)
    seen = set()
    for trial in range(60):
        e = enc.copy()
        o = offs.copy()
        kind = trial % 3
        if kind == 0:    # flip a bit in a header or literal
            e[int(RNG.integers(0, e.size))] ^= np.uint8(1 << int(RNG.integers(0, 8)))
        elif kind == 1:  # truncate the chunk
            o[1] = np.uint64(int(RNG.integers(0, int(o[1]))) & ~1)
        else:            # offsets past the stream
            o[1] = np.uint64(e.size + 2 + int(RNG.integers(0, 100)))
        want, st_o = oracle.zrle_decode(e, o, x.size, 4096)
        got, st_g = run_zrle(e, o, x.size, 4096)
        assert st_g == st_o, trial
        seen.add(st_o)
        if st_o == 0:
            assert np.array_equal(got, want)
    assert {4, 5} <= seen
