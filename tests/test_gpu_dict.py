"""GPU parity: value-dictionary decoding vs the CPU oracle (bit for bit)."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
from tests._gpu import dev, f16_out, host_bits, need_gpu, torch
from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import fp16_uniform, u8_uniform
from weight_dequantization_b200.synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def run(packed, bits, dictionary, n, out_offset=0, packed_offset=0):
    """Decode on the device; offsets shift the output / index buffers off
    their natural alignment (the scalar and narrow-store paths)."""
    out = f16_out(n, out_offset)
    p = dev(np.concatenate([np.zeros(packed_offset, np.uint8), np.asarray(packed, np.uint8)]))
    p = p[packed_offset:] if packed_offset else p
    L.lt_value_dict_decode(p, bits, dev(dictionary), n, out)
    torch.cuda.synchronize()
    return host_bits(out)


def check(packed, bits, dictionary, n, **kw):
    want, st = oracle.value_dict_decode(packed, bits, dictionary, n)
    assert st == 0
    got = run(packed, bits, dictionary, n, **kw)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"bits {bits} n {n} {kw}: {bad.size} differ, first at {bad[0]}"


def test_worked_example_order(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "int4_worked_example.json")))
    d = np.array(g["expected_f16_bits"] + [0x7E00] * 8, np.uint16)
    assert list(run(np.array(g["packed"], np.uint8), 4, d, 8)) == g["expected_f16_bits"]


def test_full_size_workload():
    d = W.v_value_dict()
    check(d["packed"], d["bits"], d["dictionary"], d["n"])


@pytest.mark.parametrize("bits", [1, 2, 8])
def test_other_widths_full_size(bits):
    # 4096 x 14336 elements: more words than one resident wave of CTAs covers
    d = W.v_value_dict(bits=bits)
    check(d["packed"], d["bits"], d["dictionary"], d["n"])


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_ragged_sizes_span_tiles(bits):
    per_word = 4 * (8 // bits)
    tile = 256 * 4 * per_word  # elements one CTA covers per pass
    dictionary = fp16_uniform(21, 1 << bits, -4.0, 4.0)
    for n in (1, per_word - 1, per_word, per_word + 1, 3 * tile + 17, 5 * tile + per_word * 3 + 1):
        packed = u8_uniform(22 + n % 7, (n * bits + 7) // 8, 0, 255)
        check(packed, bits, dictionary, n)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_unaligned_buffers(bits):
    n = 3 * 4096 + 5
    packed = u8_uniform(31, (n * bits + 7) // 8, 0, 255)
    dictionary = fp16_uniform(32, 1 << bits, -1.0, 1.0)
    check(packed, bits, dictionary, n, out_offset=1)        # out 2-byte aligned only
    check(packed, bits, dictionary, n, packed_offset=1)     # indices 1-byte aligned
    check(packed, bits, dictionary, n, out_offset=4)        # out 8-byte aligned


def test_bit_patterns_copied_exactly():
    specials = [0x8000, 0x0000, 0x7C00, 0xFC00, 0x7E01, 0xFD55, 0x0001, 0x83FF,
                0x7BFF, 0xFBFF, 0x3C00, 0xBC00, 0x7FFF, 0x0400, 0x8400, 0x3555]
    d = np.array(specials, np.uint16)
    packed = np.arange(256, dtype=np.uint8)
    check(np.tile(packed, 64), 4, d, 256 * 64 * 2)


def test_empty_is_a_no_op():
    out = f16_out(4)
    before = host_bits(out).copy()
    L.lt_value_dict_decode(dev(np.zeros(4, np.uint8)), 4, dev(np.zeros(16, np.uint16)), 0, out)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), before)


def test_writes_stay_inside_the_output():
    n = 4096 + 3
    buf = torch.full((n + 64,), float("nan"), dtype=torch.float16, device="cuda")
    guard = host_bits(buf)[n:].copy()
    packed = u8_uniform(41, (n * 4 + 7) // 8, 0, 255)
    L.lt_value_dict_decode(dev(packed), 4, dev(fp16_uniform(42, 16, 0.0, 1.0)), n, buf[:n])
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(buf)[n:], guard)
