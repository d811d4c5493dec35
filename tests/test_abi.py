"""The C-ABI library loads and exports what include/lt_decode.h declares.

Runs without a GPU: only symbol lookup and host-side argument checks, which
return before any CUDA call.
"""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from weight_dequantization_b200 import _build
from weight_dequantization_b200 import lt_decode as L

HEADER = os.path.join(_build.ROOT, "include", "lt_decode.h")


@pytest.fixture(scope="module")
def lib():
    _build.build_decode()
    return L.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lt_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert set(names) == set(L.EXPORTED), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_binding_constants_match_the_header():
    text = open(HEADER).read()
    for name in ("LT_NOALLOC_MAX_BLOCKS", "LT_LZ4_BATCH_MAX", "LT_ABI_VERSION"):
        m = re.search(r"#define\s+%s\s+(\d+)" % name, text)
        assert m, name
        want = int(m.group(1))
        got = L.abi_version() if name == "LT_ABI_VERSION" else getattr(L, name)
        assert got == want, (name, got, want)


def test_abi_version_and_status_strings(lib):
    assert L.abi_version() == 6
    for code in range(9):
        s = L.status_string(code)
        assert s and s != "unknown status"
    assert L.status_string(99) == "unknown status"


def test_host_argument_errors_return_synchronously(lib):
    # each of these is rejected before anything touches a device
    P = 0x1000  # never dereferenced
    assert lib.lt_dequant_int4(P, P, None, -1, 8, 8, P, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_dequant_int4(P, P, None, 2, 12, 8, P, None) == L.LT_ERR_INVALID_ARG  # 8 does not divide 12
    assert lib.lt_dequant_int4(P, P, None, 2, 8, 0, P, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_dequant_int4(None, P, None, 2, 8, 8, P, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_dequant_int4(P, P + 1, None, 2, 8, 8, P, None) == L.LT_ERR_MISALIGNED
    assert lib.lt_dequant_int4(P, P, None, 0, 8, 8, P, None) == L.LT_OK  # empty: nothing enqueued
    assert lib.lt_dequant_int8(P, P, None, 2, 4, 4, P, None) == L.LT_ERR_INVALID_ARG  # bad scale mode
    assert lib.lt_dequant_int8(P, P, None, 1, 4, 4, P + 1, None) == L.LT_ERR_MISALIGNED
    assert lib.lt_xxh3_blocks(P, 64, P, 1, P, 135, P, None, None, None, None) == L.LT_ERR_INVALID_ARG  # short secret
    assert lib.lt_xxh3_blocks(P, 64, P, -1, P, 192, P, None, None, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_xxh3_blocks(P, 64, P, 1, P, 192, None, None, None, None, None) == L.LT_ERR_INVALID_ARG  # no output
    assert lib.lt_xxh3_blocks(None, 64, P, 1, P, 192, P, None, None, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_xxh3_blocks(P, 64, P + 4, 1, P, 192, P, None, None, None, None) == L.LT_ERR_MISALIGNED
    assert lib.lt_xxh3_blocks(P, 64, P, 1, P, 192, None, P + 4, None, None, None) == L.LT_ERR_MISALIGNED
    assert lib.lt_xxh3_blocks(P, 64, P, 0, P, 192, P, None, None, None, None) == L.LT_OK  # empty
    assert lib.lt_hct2_layout(None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_hct2_read_header(None, 64, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_hct2_read_header(b"HCT2" + bytes(60), 64, ctypes.byref(L.LtHct2Header())) == L.LT_ERR_INVALID_ARG
    assert lib.lt_hct2_write_header(ctypes.byref(L.LtHct2Header()), None) == L.LT_ERR_INVALID_ARG
    for bits in (0, 3, 5, 16, -4):
        assert lib.lt_value_dict_decode(P, bits, P, 64, P, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_value_dict_decode(P, 4, P, -1, P, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_value_dict_decode(P, 4, None, 64, P, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_value_dict_decode(None, 4, P, 64, P, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_value_dict_decode(P, 4, P + 1, 64, P, None) == L.LT_ERR_MISALIGNED
    assert lib.lt_value_dict_decode(P, 4, P, 64, P + 1, None) == L.LT_ERR_MISALIGNED
    assert lib.lt_value_dict_decode(P, 4, P, (1 << 62), P, None) == L.LT_ERR_INVALID_ARG  # n * bits overflows
    assert lib.lt_value_dict_decode(None, 4, None, 0, None, None) == L.LT_OK  # empty: nothing enqueued
    assert lib.lt_zrle_decode(P, 16, P, 100, 0, P, None, None) == L.LT_ERR_UNSUPPORTED
    assert lib.lt_zrle_decode(P, 16, P, 100, 65536, P, None, None) == L.LT_ERR_UNSUPPORTED
    assert lib.lt_zrle_decode(P, 16, P + 4, 100, 4096, P, None, None) == L.LT_ERR_MISALIGNED
    assert lib.lt_zrle_decode(P, 16, P, -1, 4096, P, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_int4_decode(P, 16, P, 65537, P, None, 1, 8, 8, P, None, 0, None, None) == L.LT_ERR_UNSUPPORTED
    assert lib.lt_lz4_int4_decode(P, 16, P, 1000, P, None, 1, 8, 8, P, None, 0, None, None) == L.LT_ERR_UNSUPPORTED
    assert lib.lt_lz4_int4_decode(P, 16, P, 65536, P, None, 1, 8, 3, P, None, 0, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_int4_decode(P, 16, P + 2, 65536, P, None, 1, 8, 8, P, None, 0, None, None) == L.LT_ERR_MISALIGNED
    assert lib.lt_lz4_int4_decode(P, 16, P, 65536, P, None, 1, 8, 8, P, P + 4, 1 << 20, None, None) == \
        L.LT_ERR_MISALIGNED
    assert lib.lt_lz4_decode(P, 16, P, 8, P, 100, None, 0, None, None) == L.LT_ERR_UNSUPPORTED
    arr = (L.LtLz4Int4Desc * (L.LT_LZ4_BATCH_MAX + 1))()
    assert lib.lt_lz4_int4_decode_batch(arr, L.LT_LZ4_BATCH_MAX + 1, None, 0, None, None) == L.LT_ERR_UNSUPPORTED
    assert lib.lt_lz4_int4_decode_batch(arr, 0, None, 0, None, None) == L.LT_ERR_INVALID_ARG
    # the two-step decode: index and expand
    assert lib.lt_lz4_index_batch(arr, 0, P, 1 << 20, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_index_batch(arr, L.LT_LZ4_BATCH_MAX + 1, P, 1 << 20, None) == L.LT_ERR_UNSUPPORTED
    one = (L.LtLz4Int4Desc * 2)()
    for i in range(2):  # 16 x 8192 codes = 64 KB packed = one 64 KB block each
        one[i] = L.LtLz4Int4Desc(P, 16, P, P, None, P, 16, 8192, 128, 65536)
    need = lib.lt_lz4_workspace_bytes(2)
    assert lib.lt_lz4_index_batch(one, 2, P, need - 1, None) == L.LT_ERR_INVALID_ARG  # index too small
    assert lib.lt_lz4_index_batch(one, 2, None, need, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_index_batch(one, 2, P + 8, need, None) == L.LT_ERR_MISALIGNED
    # expanding descriptor 1 of a 2-block index starts at block 1; block 2 is past its end
    assert lib.lt_lz4_int4_expand_batch(one, 1, P, need, 2, 2, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_int4_expand_batch(one, 2, P, need, 2, 1, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_int4_expand_batch(one, 1, P, need, 2, -1, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_int4_expand_batch(one, 1, P, need - 1, 2, 1, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_int4_expand_batch(one, 1, None, need, 2, 1, None, None) == L.LT_ERR_INVALID_ARG
    assert lib.lt_lz4_int4_expand_batch(one, 1, P, need, 2, 1, P + 2, None) == L.LT_ERR_MISALIGNED
    # workspace sizing: a 16-byte index header plus 512 descriptors per block
    assert lib.lt_lz4_workspace_bytes(0) == 0
    assert lib.lt_lz4_workspace_bytes(448) >= 448 * (16 + 16 * 512)


def test_binding_rejects_host_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(TypeError):
        L.lt_dequant_int4(x, x, None, 1, 32, 32, x, stream=0)


def test_gemm_host_argument_errors(lib):
    P = 0x1000  # never dereferenced: every call below is refused before any CUDA call
    ok = dict(x=P, M=4, K=128, packed=P, scales=P, zeros=None, N=512, G=128, out=P)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.lt_int4_gemm(a["x"], a["M"], a["K"], a["packed"], a["scales"], a["zeros"], a["N"], a["G"],
                                a["out"], None, 0, None, None)

    assert call(N=384) == L.LT_ERR_UNSUPPORTED     # N not a multiple of 256
    assert call(K=96) == L.LT_ERR_UNSUPPORTED      # K not a multiple of 64
    assert call(G=16) == L.LT_ERR_UNSUPPORTED      # group not a multiple of 32
    assert call(G=96) == L.LT_ERR_UNSUPPORTED      # group does not divide N
    assert call(M=-1) == L.LT_ERR_INVALID_ARG
    assert call(x=None) == L.LT_ERR_INVALID_ARG
    assert call(x=P + 8) == L.LT_ERR_MISALIGNED   # x must be 16-byte aligned (tiled copies)
    assert call(out=P + 2) == L.LT_ERR_MISALIGNED
    assert call(M=0) == L.LT_OK                    # empty: nothing enqueued
    # a split of K is offered only when the output has fewer tiles than SMs
    assert L.lt_int4_gemm_workspace_bytes(1, 8192, 8192) > 0
    assert L.lt_int4_gemm_workspace_bytes(4096, 8192, 8192) == 0
    assert L.lt_int4_gemm_workspace_bytes(1, 8192, 100) == 0
