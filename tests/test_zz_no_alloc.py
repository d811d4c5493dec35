"""The fused LZ4 -> INT4 decode for callers that may not allocate device memory.

lt_lz4_int4_decode_noalloc keeps the sequence index the decode needs in a
scratch array built into the library instead of a caller-provided workspace,
so a caller whose device memory is budgeted up front (an engine plugin, a
component that does not own the allocator) can still use the fast path. This
file is collected after the decoders' parity tests on purpose: a failure here
leaves them already run.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import fp16_uniform, int4_gauss_groups_packed, lz4_compress_blocks, u8_uniform


def _matrix(seed: int, rows: int, cols: int = 8192, G: int = 128):
    n = rows * cols
    packed = int4_gauss_groups_packed(seed, n)
    comp, offs = lz4_compress_blocks(packed, 65536)
    return dict(rows=rows, cols=cols, G=G, comp=comp, offs=offs,
                scales=fp16_uniform(seed, n // G, 0.001, 0.1, stream=1), zeros=u8_uniform(seed, n // G, 0, 15, stream=2))


def test_noalloc_rejects_more_blocks_than_its_scratch_holds():
    # returns before touching any device: no GPU needed
    lib = L.load_library()
    P = 0x1000  # never dereferenced
    rows, cols = (L.LT_NOALLOC_MAX_BLOCKS + 1) * 16, 8192  # 16 rows of 8192 codes = one 64 KB block
    st = lib.lt_lz4_int4_decode_noalloc(P, 16, P, 65536, P, None, rows, cols, 128, P, None, None)
    assert st == L.LT_ERR_UNSUPPORTED
    # the largest accepted request is exactly the stated maximum
    assert lib.lt_lz4_workspace_bytes(L.LT_NOALLOC_MAX_BLOCKS) > 0


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    torch = pytest.importorskip("torch")
    from tests._gpu import assert_f16_parity, dev, host_bits, need_gpu

    need_gpu()
    lib = L.load_library()
    # two different matrices, decoded one after the other through the C ABI:
    # the second call finds the scratch holding the first call's index
    cases = [_matrix(41, 448 * 16 // 2), _matrix(42, L.LT_NOALLOC_MAX_BLOCKS * 16)]
    stream = torch.cuda.current_stream().cuda_stream
    for m in cases:
        n_blocks = len(m["offs"]) - 1
        assert n_blocks <= L.LT_NOALLOC_MAX_BLOCKS
        n = m["rows"] * m["cols"]
        comp, offs, sc, ze = dev(m["comp"]), dev(m["offs"]), dev(m["scales"]), dev(m["zeros"])
        ref = torch.empty(n, dtype=torch.float16, device="cuda")
        got = torch.full((n,), float("nan"), dtype=torch.float16, device="cuda")
        st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
        st_got = torch.zeros(1, dtype=torch.int32, device="cuda")
        ws = torch.empty(L.lt_lz4_workspace_bytes(n_blocks), dtype=torch.uint8, device="cuda")
        rc = lib.lt_lz4_int4_decode(comp.data_ptr(), int(m["comp"].size), offs.data_ptr(), 65536, sc.data_ptr(),
                                    ze.data_ptr(), m["rows"], m["cols"], m["G"], ref.data_ptr(), ws.data_ptr(),
                                    ctypes.c_uint64(ws.numel()), st_ref.data_ptr(), stream)
        assert rc == L.LT_OK
        rc = lib.lt_lz4_int4_decode_noalloc(comp.data_ptr(), int(m["comp"].size), offs.data_ptr(), 65536,
                                            sc.data_ptr(), ze.data_ptr(), m["rows"], m["cols"], m["G"],
                                            got.data_ptr(), st_got.data_ptr(), stream)
        assert rc == L.LT_OK
        torch.cuda.synchronize()
        assert int(st_ref.item()) == 0 and int(st_got.item()) == 0
        assert_f16_parity(host_bits(got), host_bits(ref), what="no-allocation entry point")
