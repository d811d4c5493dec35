"""GPU parity: INT4 group and INT8 dequantization vs the CPU oracle."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
from tests._gpu import assert_f16_parity, dev, f16_out, host_bits, need_gpu, torch
from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import fp16_uniform, int4_uniform_packed, int8_normal, u8_uniform
from weight_dequantization_b200.synth import workloads as W

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(11)


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def run_int4(packed, scales, zeros, rows, cols, G, offset=0):
    out = f16_out(rows * cols, offset)
    L.lt_dequant_int4(dev(packed), dev(scales), dev(zeros), rows, cols, G, out)
    torch.cuda.synchronize()
    return host_bits(out)


def run_int8(q, scales, zeros, per_row, rows, cols, offset=0):
    out = f16_out(rows * cols, offset)
    L.lt_dequant_int8(dev(q), dev(scales), dev(zeros), L.LT_SCALE_PER_ROW if per_row else L.LT_SCALE_PER_TENSOR,
                      rows, cols, out)
    torch.cuda.synchronize()
    return host_bits(out)


# --------------------------------------------------------------------------- INT4

def test_int4_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "int4_worked_example.json")))
    got = run_int4(np.array(g["packed"], np.uint8), np.array([g["scale_f16_bits"]], np.uint16),
                   np.array([g["zero_point"]], np.uint8), 1, 8, 8)
    assert list(got) == g["expected_f16_bits"]


def test_int4_c1_full_size():
    d = W.c1_int4()
    want, st = oracle.dequant_int4(d["packed"], d["scales"], d["zeros"], d["rows"], d["cols"], d["group_size"])
    assert st == 0
    got = run_int4(d["packed"], d["scales"], d["zeros"], d["rows"], d["cols"], d["group_size"])
    assert_f16_parity(got, want, what="C1")


def test_int4_every_code_zero_point_and_scale():
    # all 16 x 16 (q, z) pairs with all 65536 binary16 scales, including
    # subnormal, infinite and NaN scales
    n_s = 1 << 16
    q = np.tile(np.arange(16, dtype=np.uint8), 16 * n_s)
    z = np.tile(np.arange(16, dtype=np.uint8), n_s)
    s = np.repeat(np.arange(n_s, dtype=np.uint32).astype(np.uint16), 16)
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)
    want, _ = oracle.dequant_int4(packed, s, z, n_s, 256, 16)
    got = run_int4(packed, s, z, n_s, 256, 16)
    assert_f16_parity(got, want, what="brute force")


def test_int4_zero_points_above_15():
    # uint8 zero points up to 255 (|q - z| up to 255)
    rows, cols, G = 64, 256, 32
    n = rows * cols
    packed = int4_uniform_packed(5, n)
    s = fp16_uniform(5, n // G, -2.0, 2.0, stream=1)
    z = u8_uniform(5, n // G, 0, 255, stream=2)
    want, _ = oracle.dequant_int4(packed, s, z, rows, cols, G)
    assert_f16_parity(run_int4(packed, s, z, rows, cols, G), want)


@pytest.mark.parametrize("rows,cols,G,offset,with_z", [
    (1, 8, 8, 0, True), (3, 40, 8, 0, True), (7, 96, 32, 0, False), (5, 384, 128, 0, True),
    (2, 512, 256, 0, False), (9, 24, 24, 0, True),            # vector path, pow2 and non-pow2 groups
    (3, 5, 5, 0, True), (1, 1, 1, 0, True), (4, 36, 12, 0, True), (33, 6, 2, 0, False),  # scalar path
    (2, 64, 32, 3, True),                                         # output not 16-byte aligned
    (13, 72, 8, 0, True),                                         # n % 8 == 0, ragged wave
    (17, 1000, 8, 0, True),                                       # many waves
])
def test_int4_shapes(rows, cols, G, offset, with_z):
    n = rows * cols
    packed = int4_uniform_packed(rows * 1000 + cols, n)
    s = fp16_uniform(7, n // G, 0.001, 0.1, stream=1)
    z = u8_uniform(7, n // G, 0, 15, stream=2) if with_z else None
    want, st = oracle.dequant_int4(packed, s, z, rows, cols, G)
    assert st == 0
    assert_f16_parity(run_int4(packed, s, z, rows, cols, G, offset), want, what=f"{rows}x{cols}/G{G}")


def test_int4_unaligned_packed_pointer():
    rows, cols, G = 4, 256, 64
    n = rows * cols
    packed = int4_uniform_packed(3, n)
    s = fp16_uniform(3, n // G, 0.001, 0.1, stream=1)
    z = u8_uniform(3, n // G, 0, 15, stream=2)
    buf = dev(np.concatenate([np.zeros(1, np.uint8), packed]))
    out = f16_out(n)
    L.lt_dequant_int4(buf[1:], dev(s), dev(z), rows, cols, G, out)
    torch.cuda.synchronize()
    want, _ = oracle.dequant_int4(packed, s, z, rows, cols, G)
    assert_f16_parity(host_bits(out), want)


def test_int4_empty_is_a_no_op():
    out = f16_out(4)
    before = host_bits(out).copy()
    L.lt_dequant_int4(dev(np.zeros(2, np.uint8)), dev(np.zeros(1, np.uint16)), None, 0, 8, 8, out)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), before)


# --------------------------------------------------------------------------- INT8

def test_int8_page_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "int8_example.json")))
    vals = np.array(g["values"], np.int8)
    s = np.array([0x211F], np.uint16)
    want, _ = oracle.dequant_int8(vals, s, None, False, 1, 8)
    assert_f16_parity(run_int8(vals, s, None, False, 1, 8), want)


def test_int8_c2_full_size():
    d = W.c2_int8()
    want, st = oracle.dequant_int8(d["q"], d["scales"], d["zeros"], True, d["rows"], d["cols"])
    assert st == 0
    got = run_int8(d["q"], d["scales"], d["zeros"], True, d["rows"], d["cols"])
    assert_f16_parity(got, want, what="C2")


def test_int8_every_code_and_zero_point_with_many_scales():
    q = np.tile(np.arange(-128, 128, dtype=np.int16).astype(np.int8), 256)
    rows, cols = 256 * 64, 256
    qq = np.tile(q[:256], rows)
    z = np.repeat(np.arange(-128, 128, dtype=np.int16).astype(np.int8), 64)  # one zero point per row
    s = RNG.integers(0, 1 << 16, rows, dtype=np.uint32).astype(np.uint16)    # arbitrary bit patterns
    want, _ = oracle.dequant_int8(qq, s, z, True, rows, cols)
    assert_f16_parity(run_int8(qq, s, z, True, rows, cols), want, what="int8 brute force")


@pytest.mark.parametrize("rows,cols,per_row,with_z,offset", [
    (1, 8, False, False, 0), (5, 64, True, True, 0), (3, 1000, False, True, 0), (64, 4096, True, False, 0),
    (7, 13, True, True, 0), (5, 7, False, False, 0), (1, 1, True, False, 0),   # scalar path
    (4, 64, True, True, 5),                                                     # unaligned output
    (129, 24, True, True, 0),
])
def test_int8_shapes(rows, cols, per_row, with_z, offset):
    n = rows * cols
    q = int8_normal(rows + cols, n, 32.0)
    ns = rows if per_row else 1
    s = fp16_uniform(9, ns, 0.001, 0.02, stream=1)
    z = (RNG.integers(-128, 128, ns).astype(np.int8)) if with_z else None
    want, st = oracle.dequant_int8(q, s, z, per_row, rows, cols)
    assert st == 0
    assert_f16_parity(run_int8(q, s, z, per_row, rows, cols, offset), want, what=f"{rows}x{cols}")
