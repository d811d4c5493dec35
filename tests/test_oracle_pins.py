"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here is checked against the oracle itself: expected values come from
the pages' worked examples (tests/golden), from numpy's own binary16
conversion and bit unpacking, from an exact-rational brute-force search of the binary16 grid,
from closed forms and invariants, and from the system LZ4 and xxHash
libraries.
"""
from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests._pins import (hct2_build, hexbytes, liblz4, libxxhash, lz4_lib_compress, lz4_lib_decompress,
                         nearest_f16_bits, xxh3_lib)

RNG = np.random.default_rng(20261202)


# ---------------------------------------------------------------------------
# binary16 conversion (IEEE 754-2008)
# ---------------------------------------------------------------------------

def _np_f16_bits(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore", invalid="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def test_f16_to_f64_exhaustive_matches_numpy():
    h = np.arange(1 << 16, dtype=np.uint16)
    got = oracle.f16_to_f64(h)
    ref = h.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


def test_f16_from_f64_on_every_grid_point_and_midpoint():
    # every finite binary16 value, each midpoint to its successor (an exact
    # tie), and the doubles just either side of each midpoint
    h = np.arange(0x7C00, dtype=np.uint16)
    v = h.view(np.float16).astype(np.float64)
    nxt = np.append(v[1:], 65536.0)
    mid = (v + nxt) / 2  # exact in double
    cases = np.concatenate([v, mid, np.nextafter(mid, -np.inf), np.nextafter(mid, np.inf)])
    cases = np.concatenate([cases, -cases])
    got = oracle.f16_from_f64(cases)
    ref = _np_f16_bits(cases)
    assert np.array_equal(got, ref)


def test_f16_from_f64_ties_go_to_even():
    # 1 + 2^-11 lies halfway between 1 (0x3C00, even) and 1 + 2^-10 (0x3C01)
    assert oracle.f16_from_f64(1 + 2.0 ** -11)[0] == 0x3C00
    # 1 + 3 * 2^-11 lies halfway between 0x3C01 (odd) and 0x3C02 (even)
    assert oracle.f16_from_f64(1 + 3 * 2.0 ** -11)[0] == 0x3C02
    # smallest subnormal is 2^-24; half of it ties to 0 (even)
    assert oracle.f16_from_f64(2.0 ** -25)[0] == 0x0000
    assert oracle.f16_from_f64(3 * 2.0 ** -25)[0] == 0x0002
    # 65520 is the midpoint between 65504 and 2^16 and rounds to infinity
    assert oracle.f16_from_f64(65519.99)[0] == 0x7BFF
    assert oracle.f16_from_f64(65520.0)[0] == 0x7C00
    assert oracle.f16_from_f64(-65520.0)[0] == 0xFC00


def test_f16_from_f64_special_values():
    got = oracle.f16_from_f64(np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e300, -1e-300]))
    assert list(got[:4]) == [0x0000, 0x8000, 0x7C00, 0xFC00]
    assert (got[4] & 0x7C00) == 0x7C00 and (got[4] & 0x03FF) != 0
    assert got[5] == 0x7C00 and got[6] == 0x8000


def test_f16_from_f64_random_doubles_match_numpy():
    # log-uniform magnitudes over the whole binary16 range and beyond
    e = RNG.uniform(-30, 17, size=400_000)
    x = np.exp2(e) * RNG.choice([-1.0, 1.0], size=e.size)
    assert np.array_equal(oracle.f16_from_f64(x), _np_f16_bits(x))


def test_f16_from_f64_random_float32_match_numpy():
    # random fp32 bit patterns in the finite range (fp32 -> fp16 is the
    # conversion the dequantization needs)
    b = RNG.integers(0, 0x7F800000, size=1_000_000, dtype=np.uint32)
    x = b.view(np.float32).astype(np.float64) * RNG.choice([-1.0, 1.0], size=b.size)
    assert np.array_equal(oracle.f16_from_f64(x), _np_f16_bits(x))


def test_f16_from_f64_brute_force_grid_search():
    # exact rationals, rounded by searching the binary16 grid
    for _ in range(300):
        t = Fraction(int(RNG.integers(-(1 << 40), 1 << 40)), 1 << int(RNG.integers(20, 60)))
        assert oracle.f16_from_f64(float(t))[0] == nearest_f16_bits(t), t


# ---------------------------------------------------------------------------
# INT4 group dequantization (roadmap Phase 1.1)
# ---------------------------------------------------------------------------

def test_int4_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "int4_worked_example.json")))
    out, st = oracle.dequant_int4(np.array(g["packed"], np.uint8), np.array([g["scale_f16_bits"]], np.uint16),
                                  np.array([g["zero_point"]], np.uint8), 1, 8, 8)
    assert st == 0
    assert list(out) == g["expected_f16_bits"]
    assert list(out.view(np.float16).astype(np.float64)) == g["expected_values"]


def test_int4_zero_point_none_equals_zero():
    packed = RNG.integers(0, 256, 64, dtype=np.uint8)
    s = np.full(4, 0x3800, np.uint16)
    a, _ = oracle.dequant_int4(packed, s, None, 4, 32, 32)
    b, _ = oracle.dequant_int4(packed, s, np.zeros(4, np.uint8), 4, 32, 32)
    assert np.array_equal(a, b)


def test_int4_all_codes_zero_points_and_scales_brute_force():
    # every (q, z) pair with every binary16 scale; expected through numpy's
    # binary16 rounding of the exact product (q - z) * s
    n_s = 1 << 16
    q = np.tile(np.arange(16, dtype=np.uint8), 16 * n_s)          # code varies fastest
    z = np.tile(np.repeat(np.arange(16, dtype=np.uint8), 1), n_s)  # one zero point per group of 16
    s = np.repeat(np.arange(n_s, dtype=np.uint32).astype(np.uint16), 16)  # 16 groups per scale
    rows, cols, G = n_s, 256, 16
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)
    out, st = oracle.dequant_int4(packed, s, z, rows, cols, G)
    assert st == 0
    sv = s.view(np.float16).astype(np.float64)
    with np.errstate(invalid="ignore"):
        expect = ((q.reshape(-1, 16).astype(np.float64) - z[:, None]) * sv[:, None]).ravel()
    ref = _np_f16_bits(expect)
    nan = np.isnan(expect)
    assert np.array_equal(out[~nan], ref[~nan])
    assert np.all((out[nan] & 0x7C00) == 0x7C00) and np.all((out[nan] & 0x3FF) != 0)


def test_int4_group_layout_rows_and_nibbles():
    # distinct scale per group, groups of G along each row of [rows, cols]
    rows, cols, G = 6, 48, 8
    codes = RNG.integers(0, 16, rows * cols).astype(np.uint8)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    n_g = rows * cols // G
    scales = (np.arange(n_g) + 1).astype(np.float16).view(np.uint16)  # 1, 2, 3, ... exact
    zeros = RNG.integers(0, 16, n_g).astype(np.uint8)
    out, st = oracle.dequant_int4(packed, scales, zeros, rows, cols, G)
    assert st == 0
    c3 = codes.reshape(rows, cols // G, G).astype(np.int64)
    z3 = zeros.reshape(rows, cols // G, 1).astype(np.int64)
    s3 = (np.arange(n_g) + 1).reshape(rows, cols // G, 1)
    expect = ((c3 - z3) * s3).ravel().astype(np.float64)  # small integers: exact in fp16
    assert np.array_equal(out.view(np.float16).astype(np.float64), expect)


def test_int4_equal_code_and_zero_point_gives_signed_zero():
    packed = np.array([0x77], np.uint8)
    pos, _ = oracle.dequant_int4(packed, np.array([0x3C00], np.uint16), np.array([7], np.uint8), 1, 2, 2)
    neg, _ = oracle.dequant_int4(packed, np.array([0xBC00], np.uint16), np.array([7], np.uint8), 1, 2, 2)
    assert list(pos) == [0x0000, 0x0000]
    assert list(neg) == [0x8000, 0x8000]  # (+0) * negative scale = -0 under IEEE


def test_int4_odd_element_count_ignores_last_high_nibble():
    packed = np.array([0x21, 0xF3], np.uint8)  # codes 1, 2, 3 (+ ignored 0xF)
    out, st = oracle.dequant_int4(packed, np.array([0x3C00], np.uint16), None, 1, 3, 3)
    assert st == 0 and list(out.view(np.float16)) == [1.0, 2.0, 3.0]


# ---------------------------------------------------------------------------
# INT8 dequantization (roadmap Phase 1.2)
# ---------------------------------------------------------------------------

def test_int8_example_values_times_scale(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "int8_example.json")))
    s_bits = int(np.float32(g["scale_f32"]).astype(np.float16).view(np.uint16))
    assert s_bits == 0x211F
    s_exact = Fraction(float(np.uint16(s_bits).view(np.float16)))
    vals = np.array(g["values"], np.int8)
    out, st = oracle.dequant_int8(vals, np.array([s_bits], np.uint16), None, False, 1, 8)
    assert st == 0
    expect = [nearest_f16_bits(int(v) * s_exact) for v in g["values"]]
    assert list(out) == expect
    # 96 * s lands exactly halfway between two binary16 values and must go to
    # the even encoding (0.9599609375, not 0.96044921875)
    assert float(out.view(np.float16)[5]) == 0.9599609375


def test_int8_per_channel_uses_row_scale_and_zero_point():
    rows, cols = 5, 7
    q = RNG.integers(-128, 128, rows * cols).astype(np.int8)
    s = np.array([1, 2, 4, 0.5, -1], np.float16)
    z = np.array([0, 3, -5, 127, -128], np.int8)
    out, st = oracle.dequant_int8(q, s.view(np.uint16), z, True, rows, cols)
    assert st == 0
    expect = (q.reshape(rows, cols).astype(np.float64) - z[:, None]) * s.astype(np.float64)[:, None]
    assert np.array_equal(out, _np_f16_bits(expect.ravel()))


def test_int8_per_tensor_equals_per_row_with_repeated_scale():
    rows, cols = 9, 33
    q = RNG.integers(-128, 128, rows * cols).astype(np.int8)
    s = np.array([0x2A3B], np.uint16)
    a, _ = oracle.dequant_int8(q, s, None, False, rows, cols)
    b, _ = oracle.dequant_int8(q, np.repeat(s, rows), None, True, rows, cols)
    assert np.array_equal(a, b)


def test_int8_symmetric_quantizer_round_trip_within_half_step():
    # the per-tensor symmetric quantizer of the KV-compression benchmark page
    # (scale = max|x| / 127, q = clip(round(x / scale), -128, 127)); with the
    # scale stored in binary16 the reconstruction stays within half a step
    # plus the scale's own rounding and the output's binary16 rounding
    x = RNG.standard_normal(4096) * 3.0
    scale = np.max(np.abs(x)) / 127
    q = np.clip(np.round(x / scale), -128, 127).astype(np.int8)
    s16 = np.float16(scale)
    out, st = oracle.dequant_int8(q, np.array([s16]).view(np.uint16), None, False, 1, x.size)
    assert st == 0
    xhat = out.view(np.float16).astype(np.float64)
    bound = scale / 2 + np.abs(q) * abs(float(s16) - scale) + np.abs(xhat) * 2.0 ** -11
    assert np.all(np.abs(xhat - x) <= bound * (1 + 1e-12))


# ---------------------------------------------------------------------------
# value-dictionary decoding (LoreToken page and sidecar page, strategy lists)
# ---------------------------------------------------------------------------

def _unpack_indices(packed: np.ndarray, bits: int, n: int) -> np.ndarray:
    # numpy's little-endian bit unpacking: bit j of byte b is stream bit 8b + j
    stream = np.unpackbits(np.asarray(packed, np.uint8), bitorder="little")[: n * bits]
    fields = stream.reshape(n, bits).astype(np.int64)
    return (fields << np.arange(bits)).sum(axis=1)


def test_value_dict_int4_worked_example_order(golden_dir):
    # the INT4 worked example's bytes hold codes 0..7, low nibble first; a
    # dictionary whose entry i is the page's expected value for code i must
    # reproduce the page's output (entries 8..15 are never used)
    g = json.load(open(os.path.join(golden_dir, "int4_worked_example.json")))
    d = np.array(g["expected_f16_bits"] + [0x7E00] * 8, np.uint16)
    out, st = oracle.value_dict_decode(np.array(g["packed"], np.uint8), 4, d, 8)
    assert st == 0
    assert list(out) == g["expected_f16_bits"]


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_value_dict_every_byte_value(bits):
    packed = np.arange(256, dtype=np.uint8)
    n = 256 * 8 // bits
    d = RNG.permutation(np.arange(1 << 16, dtype=np.uint32))[: 1 << bits].astype(np.uint16)
    out, st = oracle.value_dict_decode(packed, bits, d, n)
    assert st == 0
    assert np.array_equal(out, d[_unpack_indices(packed, bits, n)])


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_value_dict_ragged_tail_ignores_unused_bits(bits):
    per_byte = 8 // bits
    for n in range(0, 3 * per_byte + 1):
        packed = RNG.integers(0, 256, 3, dtype=np.uint8)
        packed[-1] = 0xFF  # unused high fields of the last byte point at the last entry
        d = np.arange(1 << bits, dtype=np.uint16) + 0x1000
        out, st = oracle.value_dict_decode(packed, bits, d, n)
        assert st == 0 and out.size == n
        assert np.array_equal(out, d[_unpack_indices(packed, bits, n)])


def test_value_dict_copies_bit_patterns():
    specials = [0x8000, 0x0000, 0x7C00, 0xFC00, 0x7E01, 0xFD55, 0x0001, 0x83FF,
                0x7BFF, 0xFBFF, 0x3C00, 0xBC00, 0x7FFF, 0x0400, 0x8400, 0x3555]
    d = np.array(specials, np.uint16)
    codes = np.arange(32) % 16
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    out, st = oracle.value_dict_decode(packed, 4, d, 32)
    assert st == 0 and list(out) == specials * 2


def test_value_dict_affine_dictionary_equals_int4_dequant():
    # with dictionary entry q = fp16_rn((q - z) * s) (numpy's rounding of the
    # exact product), decoding 4-bit indices is INT4 dequant with one group
    for s_bits, z in ((0x3800, 0), (0x2E66, 7), (0xB1EC, 15), (0x0003, 3)):
        s = float(np.array([s_bits], np.uint16).view(np.float16)[0])
        d = _np_f16_bits((np.arange(16, dtype=np.float64) - z) * s)
        packed = RNG.integers(0, 256, 512, dtype=np.uint8)
        got, st = oracle.value_dict_decode(packed, 4, d, 1024)
        ref, st2 = oracle.dequant_int4(packed, np.array([s_bits], np.uint16), np.array([z], np.uint8),
                                       1, 1024, 1024)
        assert st == 0 and st2 == 0
        assert np.array_equal(got, ref)


@pytest.mark.parametrize("bits", [0, 3, 5, 16, -1])
def test_value_dict_rejects_other_widths(bits):
    _, st = oracle.value_dict_decode(np.zeros(4, np.uint8), bits, np.zeros(2, np.uint16), 4)
    assert st == oracle.INVALID


# ---------------------------------------------------------------------------
# zero-run decoding (LoreToken page, compression strategies)
# ---------------------------------------------------------------------------

def _zrle_cases(golden_dir):
    return json.load(open(os.path.join(golden_dir, "zrle_handmade.json")))["cases"]


@pytest.mark.parametrize("idx", range(12))
def test_zrle_handmade(golden_dir, idx):
    cases = _zrle_cases(golden_dir)
    assert len(cases) == 12
    c = cases[idx]
    enc = np.frombuffer(hexbytes(c["enc"]), np.uint8)
    out, st = oracle.zrle_decode(enc, np.array(c["offsets"], np.uint64), c["n"], c["chunk"])
    assert st == c["status"], c["name"]
    if c["status"] == 0:
        assert list(out) == c["out"], c["name"]


def test_zrle_round_trip_generated_relu():
    from weight_dequantization_b200.synth import relu_runs, zrle_encode
    x = relu_runs(7, 100_003)
    enc, off = zrle_encode(x, 4096)
    out, st = oracle.zrle_decode(enc, off, x.size, 4096)
    assert st == 0 and np.array_equal(out, x)
    # the law: about 90 % zeros
    assert 0.85 < np.mean(x == 0) < 0.95


def test_zrle_decoder_independent_of_chunk_partition():
    # the same tensor encoded with different chunk sizes decodes identically
    x = RNG.integers(1, 0x7C00, 5000).astype(np.uint16)
    x[RNG.random(5000) < 0.8] = 0
    from weight_dequantization_b200.synth import zrle_encode
    for chunk in (1, 7, 64, 4096, 5000, 65535):
        enc, off = zrle_encode(x, chunk, pad=1)
        out, st = oracle.zrle_decode(enc, off, x.size, chunk)
        assert st == 0 and np.array_equal(out, x), chunk


# ---------------------------------------------------------------------------
# LZ4 block decoding
# ---------------------------------------------------------------------------

def _lz4_cases(golden_dir):
    return json.load(open(os.path.join(golden_dir, "lz4_handmade.json")))["cases"]


def _expected_out(c) -> bytes:
    if "out" in c:
        return hexbytes(c["out"])
    r = c["out_repeat"]
    return hexbytes(r["unit"]) * r["count"] + hexbytes(r["extra"]) + hexbytes(r["tail"])


@pytest.mark.parametrize("idx", range(16))
def test_lz4_handmade(golden_dir, idx):
    cases = _lz4_cases(golden_dir)
    assert len(cases) == 16
    c = cases[idx]
    comp = hexbytes(c["comp"])
    if c["status"] == 0:
        want = _expected_out(c)
        out, st = oracle.lz4_block_decode(comp, len(want))
        assert st == 0, c["name"]
        assert out.tobytes() == want, c["name"]
    else:
        out, st = oracle.lz4_block_decode(comp, c["out_len"])
        assert st == c["status"], c["name"]


@pytest.mark.skipif(liblz4() is None, reason="system liblz4 not present")
def test_lz4_handmade_strict_cases_agree_with_liblz4(golden_dir):
    for c in _lz4_cases(golden_dir):
        if c["status"] == 0 and c.get("strict"):
            want = _expected_out(c)
            assert lz4_lib_decompress(hexbytes(c["comp"]), len(want)) == want, c["name"]


@pytest.mark.skipif(liblz4() is None, reason="system liblz4 not present")
@pytest.mark.parametrize("kind", ["zeros", "random", "0xab", "int4_law", "text", "short"])
def test_lz4_decodes_liblz4_output(kind):
    n = 65536
    if kind == "zeros":
        data = bytes(n)
    elif kind == "random":
        data = RNG.integers(0, 256, n, dtype=np.uint8).tobytes()
    elif kind == "0xab":
        data = b"\xab" * n
    elif kind == "int4_law":
        from weight_dequantization_b200.synth import int4_gauss_groups_packed
        data = int4_gauss_groups_packed(11, 2 * n).tobytes()
    elif kind == "text":
        words = [b"alpha", b"beta", b"gamma", b"delta", b"lz4", b"block"]
        data = b" ".join(words[i] for i in RNG.integers(0, len(words), 20000))[:n]
    else:
        data = b"abcdefghijklm"
    comp = lz4_lib_compress(data)
    out, st = oracle.lz4_block_decode(comp, len(data))
    assert st == 0 and out.tobytes() == data


@pytest.mark.skipif(liblz4() is None, reason="system liblz4 not present")
def test_generator_lz4_output_accepted_by_liblz4():
    # the roadmap's 64 KB test block (0xAB x 65536), a literal-only random
    # block, and the INT4 workload law: the input generator's compressor must
    # emit blocks that an outside decoder reads back exactly
    from weight_dequantization_b200.synth import int4_gauss_groups_packed, lz4_compress_block
    cases = [b"\xab" * 65536, RNG.integers(0, 256, 65536, dtype=np.uint8).tobytes(),
             int4_gauss_groups_packed(5, 131072).tobytes(), b"x", b"", bytes(13)]
    for data in cases:
        comp = lz4_compress_block(np.frombuffer(data, np.uint8) if data else np.zeros(0, np.uint8))
        assert lz4_lib_decompress(comp.tobytes(), len(data)) == data
        out, st = oracle.lz4_block_decode(comp, len(data))
        assert st == 0 and out.tobytes() == data
    # 0xAB x 65536 is not stored as 64 KB of literals: one literal + a long
    # offset-1 match
    comp = lz4_compress_block(np.full(65536, 0xAB, np.uint8))
    assert comp.size < 300


def test_lz4_literal_only_64k_block():
    from weight_dequantization_b200.synth import lz4_compress_block
    data = RNG.integers(0, 256, 65536, dtype=np.uint8)
    comp = lz4_compress_block(data, force_literals=True)
    # token + 256 extension bytes for 65536 - 15 + the literals
    assert comp.size == 1 + (65536 - 15) // 255 + 1 + 65536
    out, st = oracle.lz4_block_decode(comp, data.size)
    assert st == 0 and np.array_equal(out, data)


def test_lz4_match_at_maximum_offset():
    # a match reaching back exactly 65535 bytes
    head = RNG.integers(0, 256, 65535, dtype=np.uint8).tobytes()
    tok_lit = bytes([0xF4]) + bytes([255] * ((65535 - 15) // 255)) + bytes([(65535 - 15) % 255])
    comp = tok_lit + head + bytes([0xFF, 0xFF]) + bytes([0x50]) + b"tail!"
    # token 0xF4: 65535 literals, match length 8 at offset 65535, then 5 literals
    out, st = oracle.lz4_block_decode(comp, 65535 + 8 + 5)
    assert st == 0
    assert out.tobytes() == head + head[:8] + b"tail!"
    if liblz4() is not None:
        assert lz4_lib_decompress(comp, 65535 + 8 + 5) == out.tobytes()


def test_lz4_blocks_and_fused_equal_decompress_then_dequant():
    from weight_dequantization_b200.synth import fp16_uniform, int4_gauss_groups_packed, lz4_compress_blocks, u8_uniform
    rows, cols, G = 48, 4096, 128
    n = rows * cols
    packed = int4_gauss_groups_packed(3, n)
    comp, off = lz4_compress_blocks(packed, 16384)
    s = fp16_uniform(3, n // G, 0.001, 0.1, stream=1)
    z = u8_uniform(3, n // G, 0, 15, stream=2)
    raw, st = oracle.lz4_decode_blocks(comp, off, 16384, packed.size)
    assert st == 0 and np.array_equal(raw, packed)
    fused, st = oracle.lz4_int4_decode(comp, off, 16384, s, z, rows, cols, G)
    assert st == 0
    # independent dequant of the raw packed bytes through numpy
    codes = np.empty(n, np.int64)
    codes[0::2] = packed & 0xF
    codes[1::2] = packed >> 4
    sv = s.view(np.float16).astype(np.float64)
    expect = ((codes.reshape(-1, G) - z[:, None].astype(np.int64)) * sv[:, None]).ravel()
    assert np.array_equal(fused, _np_f16_bits(expect))


def test_lz4_corrupt_block_is_reported_not_crashing():
    from weight_dequantization_b200.synth import int4_gauss_groups_packed, lz4_compress_block
    data = int4_gauss_groups_packed(9, 131072)
    comp = lz4_compress_block(data)
    bad = 0
    for i in range(200):
        c = comp.copy()
        pos = int(RNG.integers(0, c.size))
        c[pos] ^= np.uint8(1 << int(RNG.integers(0, 8)))
        out, st = oracle.lz4_block_decode(c, data.size)
        if st != 0:
            bad += 1
        else:
            # a flip inside a literal decodes fine but differs from the input
            assert not np.array_equal(out, data) or c.tobytes() == comp.tobytes()
    assert bad > 0
    # truncation always fails
    for cut in (1, 2, 10, comp.size // 2):
        _, st = oracle.lz4_block_decode(comp[:-cut], data.size)
        assert st != 0


def test_lz4_random_sequence_blocks_match_direct_simulation():
    # blocks assembled sequence by sequence in every match regime; expected
    # bytes from a direct simulation of the format, and the system library
    from tests._lz4gen import random_blocks
    comp, offs, raw = random_blocks(101, 12, 65536, last=40000)
    out, st = oracle.lz4_decode_blocks(comp, offs, 65536, raw.size)
    assert st == 0 and np.array_equal(out, raw)
    if liblz4() is not None:
        for b in range(len(offs) - 1):
            c = comp[int(offs[b]):int(offs[b + 1])].tobytes()
            want = raw[b * 65536:(b + 1) * 65536].tobytes()
            assert lz4_lib_decompress(c, len(want)) == want


# ---------------------------------------------------------------------------
# XXH3-64 and the HCT v2 container (roadmap Phase 6.1)
# ---------------------------------------------------------------------------

needs_xxhash = pytest.mark.skipif(libxxhash() is None, reason="system libxxhash not present")


@needs_xxhash
@pytest.mark.parametrize("secret_len", [136, 192, 193, 256])
def test_xxh3_matches_libxxhash_in_every_length_class(secret_len):
    # 0, 1-3, 4-8, 9-16, 17-128, 129-240 and the striped path, across the
    # boundaries of the secret's scramble blocks ((secret_len - 64) / 8
    # stripes of 64 bytes)
    secret = RNG.integers(0, 256, secret_len, dtype=np.uint8).tobytes()
    block = 64 * ((secret_len - 64) // 8)
    lengths = list(range(0, 260)) + [block - 1, block, block + 1, 2 * block, 2 * block + 63, 2 * block + 64,
                                     4096, 47_000, 65_536, 100_003]
    for n in lengths:
        data = RNG.integers(0, 256, n, dtype=np.uint8).tobytes()
        assert oracle.xxh3_64(data, secret) == xxh3_lib(data, secret), n


@needs_xxhash
def test_xxh3_structured_inputs():
    secret = bytes((7 * i + 3) & 0xFF for i in range(192))
    for data in (b"", b"\0", b"\0" * 17, b"\xff" * 241, b"\0" * 65536, bytes(range(256)) * 300):
        assert oracle.xxh3_64(data, secret) == xxh3_lib(data, secret), len(data)


def _lz4_int4_container(secret_len=192):
    # a small LZ4+INT4 matrix: 8 x 8192 codes = 32 KB packed in 4 blocks of 8 KB
    from weight_dequantization_b200.synth import (fp16_uniform, int4_gauss_groups_packed, lz4_compress_blocks,
                                                  u8_uniform)
    rows, cols, G, bs = 8, 8192, 128, 8192
    packed = int4_gauss_groups_packed(9, rows * cols)
    comp, offs = lz4_compress_blocks(packed, bs)
    blocks = [comp[offs[b]:offs[b + 1]].tobytes() for b in range(len(offs) - 1)]
    n_groups = rows * cols // G
    scales = fp16_uniform(9, n_groups, 0.001, 0.1, stream=1).tobytes()
    zeros = u8_uniform(9, n_groups, 0, 15, stream=2).tobytes()
    secret = RNG.integers(0, 256, secret_len, dtype=np.uint8).tobytes()
    return hct2_build(blocks, bs, rows, cols, G, 1, scales, zeros, secret), blocks


@needs_xxhash
def test_hct2_checksum_valid():
    c, _ = _lz4_int4_container()
    assert oracle.hct2_validate(c) == (oracle.HCT_OK, None)


@needs_xxhash
def test_hct2_checksum_detects_corruption():
    c, _ = _lz4_int4_container()
    bad = bytearray(c)
    bad[100] ^= 0xFF  # the page's flipped byte
    assert oracle.hct2_validate(bytes(bad))[0] != oracle.HCT_OK


@needs_xxhash
def test_hct2_every_flipped_byte_is_reported():
    c, blocks = _lz4_int4_container(secret_len=136)
    _, _, sec = oracle.hct2_meta(c)
    for i in range(len(c)):
        bad = bytearray(c)
        bad[i] ^= 0x5A
        st, blk = oracle.hct2_validate(bytes(bad))
        assert st != oracle.HCT_OK, i
        if i >= sec["payload"]:  # a payload byte: the block holding it, found by its hash
            rel = i - sec["payload"]
            ends = np.cumsum([len(b) for b in blocks])
            assert (st, blk) == (oracle.HCT_BLOCK_MISMATCH, int(np.searchsorted(ends, rel, side="right"))), i


@needs_xxhash
def test_hct2_metadata():
    c, blocks = _lz4_int4_container()
    st, meta, sec = oracle.hct2_meta(c)
    assert st == oracle.HCT_OK
    assert meta["compression"] == 1 and meta["quantization"] == 1  # LZ4, INT4
    assert meta["block_size"] == 8192 and meta["rows"] == 8 and meta["cols"] == 8192 and meta["group_size"] == 128
    assert meta["n_blocks"] == len(blocks) and meta["payload_bytes"] == sum(len(b) for b in blocks)
    assert meta["n_groups"] == 512 and sec["end"] == len(c)
    assert all(v % 16 == 0 for k, v in sec.items() if k != "end")
    # the page's block size through the same header
    c2 = hct2_build([b"\x10"], 65536, 1, 2, 2, 1, b"\x00\x3c", b"\x00", bytes(136))
    assert oracle.hct2_meta(c2)[1]["block_size"] == 65536


@needs_xxhash
def test_hct2_header_and_size_errors():
    c, _ = _lz4_int4_container()
    assert oracle.hct2_validate(c[:-1])[0] == oracle.HCT_TRUNCATED
    assert oracle.hct2_validate(c + b"\0")[0] == oracle.HCT_TRUNCATED
    assert oracle.hct2_validate(b"HCT1" + c[4:])[0] == oracle.HCT_BAD_HEADER
    assert oracle.hct2_validate(c[:40])[0] == oracle.HCT_BAD_HEADER
    short_secret = hct2_build([b"ab"], 64, 1, 2, 2, 1, b"\0\0", b"\0", bytes(135))
    assert oracle.hct2_validate(short_secret)[0] == oracle.HCT_BAD_HEADER


# ---------------------------------------------------------------------------
# decode -> matrix multiply (roadmap Phase 4.1: input.matmul(weights))
# ---------------------------------------------------------------------------

def _np_int4_dequant(packed, scales, zeros, K, N, G):
    # numpy's own path: nibbles low first, (q - z) * s exact in double,
    # rounded by numpy's binary16 conversion
    codes = np.stack([packed & 0xF, packed >> 4], axis=1).ravel()[: K * N].astype(np.float64)
    z = np.repeat(zeros.astype(np.float64), G)
    s = np.repeat(scales.view(np.float16).astype(np.float64), G)
    return ((codes - z) * s).astype(np.float16).astype(np.float64).reshape(K, N)


def _int4_operands(seed, M, K, N, G):
    rng = np.random.default_rng(seed)
    packed = rng.integers(0, 256, K * N // 2, dtype=np.uint8)
    scales = rng.uniform(0.001, 0.1, K * N // G).astype(np.float16).view(np.uint16)
    zeros = rng.integers(0, 16, K * N // G, dtype=np.uint8)
    x = rng.standard_normal((M, K)).astype(np.float16)
    return x, packed, scales, zeros


def test_int4_matmul_identity_input_returns_the_decoded_matrix():
    K, N, G = 48, 40, 8
    _, packed, scales, zeros = _int4_operands(1, K, K, N, G)
    eye = np.eye(K, dtype=np.float16)
    out, absum, st = oracle.int4_matmul(eye.view(np.uint16), K, packed, scales, zeros, K, N, G)
    assert st == 0
    w = _np_int4_dequant(packed, scales, zeros, K, N, G)
    assert np.array_equal(out, w) and np.array_equal(absum, np.abs(w))


def test_int4_matmul_matches_numpy_matmul():
    M, K, N, G = 24, 256, 96, 32  # M, K, N distinct: a transposed operand cannot pass
    x, packed, scales, zeros = _int4_operands(2, M, K, N, G)
    out, absum, st = oracle.int4_matmul(x.view(np.uint16), M, packed, scales, zeros, K, N, G)
    assert st == 0
    w = _np_int4_dequant(packed, scales, zeros, K, N, G)
    xd = x.astype(np.float64)
    assert np.all(np.abs(out - xd @ w) <= 1e-13 * absum + 1e-300)
    assert np.allclose(absum, np.abs(xd) @ np.abs(w), rtol=1e-13, atol=0)


def test_int4_matmul_small_integers_are_exact():
    M, K, N, G = 5, 64, 32, 16
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, K * N)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    zeros = rng.integers(0, 16, K * N // G, dtype=np.uint8)
    scales = np.full(K * N // G, 0x3C00, np.uint16)  # 1.0
    xi = rng.integers(-8, 9, (M, K))
    out, _, st = oracle.int4_matmul(xi.astype(np.float16).view(np.uint16), M, packed, scales, zeros, K, N, G)
    assert st == 0
    wi = codes.reshape(K, N) - np.repeat(zeros.astype(np.int64), G).reshape(K, N)
    assert np.array_equal(out, (xi @ wi).astype(np.float64))


def test_int4_matmul_worked_example_row(golden_dir):
    # the INT4 worked example as a 1 x 8 weight; an input of [[2.0]] doubles it
    g = json.load(open(os.path.join(golden_dir, "int4_worked_example.json")))
    out, _, st = oracle.int4_matmul(np.array([[0x4000]], np.uint16), 1, np.array(g["packed"], np.uint8),
                                    np.array([g["scale_f16_bits"]], np.uint16), np.array([g["zero_point"]], np.uint8),
                                    1, 8, 8)
    assert st == 0 and list(out[0]) == [2 * v for v in g["expected_values"]]
