"""HCT v2 container header on the host (no GPU): the library's native
header functions (lt_hct2_layout / read_header / write_header, through the
C ABI) agree with the oracle's reading of containers built byte by byte."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests._pins import hct2_build, libxxhash
from weight_dequantization_b200 import hct
from weight_dequantization_b200 import lt_decode as L

pytestmark = pytest.mark.skipif(libxxhash() is None, reason="system libxxhash not present")
RNG = np.random.default_rng(23)


def _containers():
    sec = RNG.integers(0, 256, 192, dtype=np.uint8).tobytes()
    blocks = [RNG.integers(0, 256, n, dtype=np.uint8).tobytes() for n in (100, 0, 4097, 31)]
    yield hct2_build(blocks, 8192, 4, 8192, 128, 1, bytes(2 * 256), bytes(256), sec)          # INT4
    yield hct2_build(blocks[:1], 65536, 3, 10, 0, 2, bytes(2 * 3), b"", sec[:136])            # INT8
    yield hct2_build([], 65536, 0, 0, 0, 0, b"", b"", sec, compression=0)                     # empty


@pytest.mark.parametrize("idx", range(3))
def test_header_and_sections_match_the_oracle(idx):
    c = list(_containers())[idx]
    st, meta, sec = oracle.hct2_meta(c)
    assert st == oracle.HCT_OK
    h = hct.read_header(c)
    for k in ("compression", "quantization", "block_size", "rows", "cols", "group_size", "secret_len", "n_blocks",
              "payload_bytes", "n_groups", "version", "checksum"):
        assert getattr(h, k) == meta[k], k
    assert hct.sections(h) == sec
    assert L.lt_hct2_write_header(h) == c[:64]


def test_parser_rejects_what_the_oracle_rejects():
    c = next(_containers())
    for bad in (c[:-1], c + b"\0", b"HCT1" + c[4:], c[:40]):
        assert oracle.hct2_validate(bad)[0] in (oracle.HCT_TRUNCATED, oracle.HCT_BAD_HEADER)
        with pytest.raises(hct.HctError):
            hct.read_header(bad)


def test_writer_rejects_bad_arguments_before_any_device_work():
    with pytest.raises(hct.HctError):
        hct.write([b"ab"], 65536, 1, 2, hct.QUANT_INT4, 2, np.zeros(1, np.uint16), np.zeros(1, np.uint8),
                  secret=bytes(135))  # secret too short
    with pytest.raises(hct.HctError):
        hct.write([b"ab"], 65536, 1, 4, hct.QUANT_INT4, 2, np.zeros(1, np.uint16), np.zeros(2, np.uint8),
                  secret=bytes(136))  # 2 groups need 2 scales


@pytest.mark.parametrize("field,offset,value", [
    ("version", 4, b"\x03\x00"), ("compression", 8, b"\x02"), ("quantization", 9, b"\x03"),
    ("checksum", 10, b"\x00"), ("secret_len", 36, (135).to_bytes(4, "little")),
    ("block_size", 12, bytes(4)), ("group_size", 32, (3).to_bytes(4, "little")),
])
def test_parser_rejects_each_bad_field(field, offset, value):
    c = bytearray(next(_containers()))
    c[offset:offset + len(value)] = value
    with pytest.raises(hct.HctError):
        hct.read_header(bytes(c))
    assert oracle.hct2_validate(bytes(c))[0] == oracle.HCT_BAD_HEADER, field


def test_decode_rejects_payloads_that_cannot_hold_the_shape():
    sec = bytes(range(136))
    # INT4 without compression: 4 x 64 codes need 128 payload bytes, 100 given
    short = hct2_build([bytes(100)], 4096, 4, 64, 64, 1, bytes(2 * 4), bytes(4), sec, compression=0)
    with pytest.raises(hct.HctError):
        hct.decode(short, check=False)
    # LZ4 + INT4: 4 x 65536 codes are 128 KB packed, two 64 KB blocks; one given
    one_block = hct2_build([b"\x00" * 8], 65536, 4, 65536, 128, 1, bytes(2 * 2048), bytes(2048), sec)
    with pytest.raises(hct.HctError):
        hct.decode(one_block, check=False)


def test_decode_refuses_lz4_int8_before_any_device_work():
    c = hct2_build([b"\x00"], 65536, 2, 8, 0, 2, bytes(4), b"", bytes(range(136)))
    with pytest.raises(hct.HctError):
        hct.decode(c)
