"""GPU parity: per-block XXH3-64 checksums vs the CPU oracle, and their
verification against the hashes stored in an HCT v2 container."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests._gpu import dev, need_gpu, torch
from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import int4_gauss_groups_packed, lz4_compress_blocks

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(17)
NONE = np.uint64(0xFFFFFFFFFFFFFFFF)


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def device_hashes(data: np.ndarray, offsets: np.ndarray, secret: np.ndarray, expected=None):
    """(hashes, status, first bad block) from the device."""
    n = offsets.size - 1
    hashes = torch.zeros(max(n, 1), dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.from_numpy(np.array([NONE]).view(np.int64)).cuda()
    d = dev(data) if data.size else None
    L.lt_xxh3_blocks(d, data.size, dev(offsets), n, dev(secret), secret.size, hashes,
                     None if expected is None else dev(expected), status, first)
    torch.cuda.synchronize()
    return (hashes.cpu().numpy().view(np.uint64)[:n], int(status.item()),
            int(first.cpu().numpy().view(np.uint64)[0]))


def oracle_hashes(data, offsets, secret):
    return np.array([oracle.xxh3_64(data[offsets[b]:offsets[b + 1]], secret) for b in range(offsets.size - 1)],
                    np.uint64)


@pytest.mark.parametrize("secret_len", [136, 192, 256])
def test_every_length_class(secret_len):
    secret = RNG.integers(0, 256, secret_len, dtype=np.uint8)
    block = 64 * ((secret_len - 64) // 8)
    lengths = list(range(0, 300)) + [block - 1, block, block + 1, 3 * block + 5, 47_000, 65_536]
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.uint64)
    data = RNG.integers(0, 256, int(offsets[-1]), dtype=np.uint8)
    got, st, first = device_hashes(data, offsets, secret)
    assert st == 0 and first == int(NONE)
    want = oracle_hashes(data, offsets, secret)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{bad.size} hashes differ, first at length {lengths[bad[0]]}"


def test_lz4_blocks_verify_and_report_the_first_mismatch():
    packed = int4_gauss_groups_packed(4, 2 * 64 * 65536)  # 64 blocks of 64 KB
    comp, offs = lz4_compress_blocks(packed, 65536)
    secret = RNG.integers(0, 256, 192, dtype=np.uint8)
    want = oracle_hashes(comp, offs, secret)
    got, st, first = device_hashes(comp, offs, secret, expected=want)
    assert st == 0 and first == int(NONE) and np.array_equal(got, want)
    stored = want.copy()
    stored[[41, 17]] ^= np.uint64(1)
    _, st, first = device_hashes(comp, offs, secret, expected=stored)
    assert st == L.LT_ERR_CHECKSUM and first == 17


def test_flipped_payload_byte_is_found_in_its_block():
    packed = int4_gauss_groups_packed(5, 2 * 8 * 65536)
    comp, offs = lz4_compress_blocks(packed, 65536)
    secret = RNG.integers(0, 256, 136, dtype=np.uint8)
    stored = oracle_hashes(comp, offs, secret)
    for pos in (0, int(offs[3]) + 100, comp.size - 1):
        bad = comp.copy()
        bad[pos] ^= 0xFF
        _, st, first = device_hashes(bad, offs, secret, expected=stored)
        blk = int(np.searchsorted(offs[1:], pos, side="right"))
        assert (st, first) == (L.LT_ERR_CHECKSUM, blk), pos


def test_offsets_past_the_stream_are_reported():
    data = RNG.integers(0, 256, 1000, dtype=np.uint8)
    secret = RNG.integers(0, 256, 192, dtype=np.uint8)
    offsets = np.array([0, 500, 1001, 900], np.uint64)  # block 1 ends past the data, block 2 runs backwards
    got, st, _ = device_hashes(data, offsets, secret)
    assert st == L.LT_ERR_CORRUPT_STREAM
    assert got[0] == oracle.xxh3_64(data[:500], secret)


def _container_parts():
    from weight_dequantization_b200.synth import fp16_uniform, u8_uniform
    rows, cols, G, bs = 16, 8192, 128, 16384
    packed = int4_gauss_groups_packed(6, rows * cols)
    comp, offs = lz4_compress_blocks(packed, bs)
    blocks = [comp[offs[b]:offs[b + 1]].tobytes() for b in range(len(offs) - 1)]
    n_groups = rows * cols // G
    scales = fp16_uniform(6, n_groups, 0.001, 0.1, stream=1)
    zeros = u8_uniform(6, n_groups, 0, 15, stream=2)
    secret = RNG.integers(0, 256, 192, dtype=np.uint8).tobytes()
    return blocks, bs, rows, cols, G, scales, zeros, secret


def test_container_written_on_the_device_is_the_reference_layout():
    from tests._pins import hct2_build, libxxhash
    from weight_dequantization_b200 import hct
    if libxxhash() is None:
        pytest.skip("system libxxhash not present")
    blocks, bs, rows, cols, G, scales, zeros, secret = _container_parts()
    c = hct.write(blocks, bs, rows, cols, hct.QUANT_INT4, G, scales, zeros, secret)
    assert c == hct2_build(blocks, bs, rows, cols, G, 1, scales.tobytes(), zeros.tobytes(), secret)
    assert oracle.hct2_validate(c) == (oracle.HCT_OK, None)


def test_container_verified_on_the_device():
    from weight_dequantization_b200 import hct
    blocks, bs, rows, cols, G, scales, zeros, secret = _container_parts()
    c = hct.write(blocks, bs, rows, cols, hct.QUANT_INT4, G, scales, zeros, secret)
    assert hct.verify(c) == (True, None, True)
    sec = hct.sections(hct.read_header(c))
    ends = np.cumsum([len(b) for b in blocks])
    for rel in (0, int(ends[2]) + 7, int(ends[-1]) - 1):
        bad = bytearray(c)
        bad[sec["payload"] + rel] ^= 0xFF
        assert hct.verify(bytes(bad)) == (False, int(np.searchsorted(ends, rel, side="right")), True), rel
    bad = bytearray(c)
    bad[100] ^= 0xFF  # a byte of the secret: the metadata hash no longer matches
    assert hct.verify(bytes(bad)) == (False, None, False)
    assert oracle.hct2_validate(bytes(bad))[0] == oracle.HCT_META_MISMATCH


def _f16_bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).ravel()


def test_container_decodes_like_the_oracle():
    from weight_dequantization_b200 import hct
    blocks, bs, rows, cols, G, scales, zeros, secret = _container_parts()
    c = hct.write(blocks, bs, rows, cols, hct.QUANT_INT4, G, scales, zeros, secret)
    comp = np.frombuffer(b"".join(blocks), np.uint8)
    offs = np.concatenate([[0], np.cumsum([len(b) for b in blocks])]).astype(np.uint64)
    want, st = oracle.lz4_int4_decode(comp, offs, bs, scales, zeros, rows, cols, G)
    assert st == 0
    assert np.array_equal(_f16_bits(hct.decode(c)), want)
    # a damaged payload byte: the checked decode names its block
    bad = bytearray(c)
    bad[-1] ^= 0xFF
    with pytest.raises(hct.HctError, match=f"checksum mismatch in block {len(blocks) - 1}$"):
        hct.decode(bytes(bad))
    # a damaged byte of the secret: the metadata hash no longer matches
    bad = bytearray(c)
    bad[100] ^= 0xFF
    with pytest.raises(hct.HctError, match="metadata checksum mismatch"):
        hct.decode(bytes(bad))


def test_uncompressed_and_raw_containers_decode_like_the_oracle():
    from weight_dequantization_b200 import hct
    from weight_dequantization_b200.synth import fp16_uniform, int8_normal, relu_runs, u8_uniform
    secret = RNG.integers(0, 256, 136, dtype=np.uint8).tobytes()
    # INT4 without compression, payload in two checksummed blocks
    rows, cols, G = 8, 1024, 64
    packed = int4_gauss_groups_packed(8, rows * cols)
    s4 = fp16_uniform(8, rows * cols // G, 0.001, 0.1, stream=1)
    z4 = u8_uniform(8, rows * cols // G, 0, 15, stream=2)
    c = hct.write([packed[:1000].tobytes(), packed[1000:].tobytes()], 4096, rows, cols, hct.QUANT_INT4, G, s4, z4,
                  secret, compression=hct.COMPRESSION_NONE)
    want, _ = oracle.dequant_int4(packed, s4, z4, rows, cols, G)
    assert np.array_equal(_f16_bits(hct.decode(c)), want)
    # INT8 per row without compression
    q = int8_normal(9, 16 * 512, 32.0)
    s8 = fp16_uniform(9, 16, 0.001, 0.02, stream=1)
    c = hct.write([q.view(np.uint8).tobytes()], 8192, 16, 512, hct.QUANT_INT8, 0, s8, None, secret,
                  compression=hct.COMPRESSION_NONE)
    want, _ = oracle.dequant_int8(q, s8, None, True, 16, 512)
    assert np.array_equal(_f16_bits(hct.decode(c)), want)
    # raw fp16 in LZ4 blocks
    x = relu_runs(10, 3 * 32768)
    comp, offs = lz4_compress_blocks(x.view(np.uint8), 65536)
    blocks = [comp[offs[b]:offs[b + 1]].tobytes() for b in range(len(offs) - 1)]
    c = hct.write(blocks, 65536, 3, 32768, hct.QUANT_NONE, 0, None, None, secret)
    assert np.array_equal(_f16_bits(hct.decode(c)), x)


# --------------------------------------------------------------------------- checked decode

def _checked(comp, offs, m, secret, expected, ws=True, shift=0):
    n = m["rows"] * m["cols"]
    out = torch.full((n,), float("nan"), dtype=torch.float16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.from_numpy(np.array([NONE]).view(np.int64)).cuda()
    buf = dev(np.concatenate([np.zeros(shift, np.uint8), comp]))[shift:]
    nb = offs.size - 1
    work = torch.empty(L.lt_lz4_workspace_bytes(nb), dtype=torch.uint8, device="cuda") if ws else None
    L.lt_lz4_int4_decode_checked(buf, comp.size, dev(offs), 65536, dev(m["scales"]), dev(m["zeros"]), m["rows"],
                                 m["cols"], m["group_size"], out, dev(secret), secret.size, dev(expected), work,
                                 status, first)
    torch.cuda.synchronize()
    bits = out.cpu().view(torch.int16).numpy().view(np.uint16)
    return bits, int(status.item()), int(first.cpu().numpy().view(np.uint64)[0])


@pytest.mark.parametrize("ws,shift", [(True, 0), (False, 0), (True, 5)])
def test_checked_decode_matches_the_oracle_and_stops_a_damaged_block(ws, shift):
    from weight_dequantization_b200.synth import workloads as W
    m = W.c4_lz4_int4(scale=16 * 8 / 4096, seed=21)  # 16 blocks of 64 KB, C4's law
    comp, offs = m["comp"], m["offsets"]
    secret = RNG.integers(0, 256, 192, dtype=np.uint8)
    stored = oracle_hashes(comp, offs, secret)
    want, st = oracle.lz4_int4_decode(comp, offs, 65536, m["scales"], m["zeros"], m["rows"], m["cols"],
                                      m["group_size"])
    assert st == 0
    got, st, first = _checked(comp, offs, m, secret, stored, ws, shift)
    assert (st, first) == (0, int(NONE))
    assert np.array_equal(got, want)
    # one flipped byte in block 5: reported as a checksum mismatch at block 5
    # (not as whatever stream error the damage causes); every other block
    # still decodes exactly
    bad = comp.copy()
    bad[int(offs[5]) + 7] ^= 0xFF
    got, st, first = _checked(bad, offs, m, secret, stored, ws, shift)
    assert (st, first) == (L.LT_ERR_CHECKSUM, 5)
    per = 2 * 65536
    keep = np.ones(want.size, bool)
    keep[5 * per:6 * per] = False
    assert np.array_equal(got[keep], want[keep])
