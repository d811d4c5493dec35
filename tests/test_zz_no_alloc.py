"""The fused LZ4 -> INT4 decode for callers that may not allocate device memory.

lt_lz4_int4_decode_noalloc keeps the sequence index the decode needs in a
scratch array built into the library instead of a caller-provided workspace,
so a caller whose device memory is budgeted up front (an engine plugin, a
component that does not own the allocator) can still use the fast path. This
file is collected after the decoders' parity tests on purpose: a failure here
leaves them already run.
"""
from __future__ import annotations

import os
import re

import numpy as np
import pytest

from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import fp16_uniform, int4_gauss_groups_packed, lz4_compress_blocks, u8_uniform


def _matrix(seed: int, rows: int, cols: int = 8192, G: int = 128, block_bytes: int = 65536):
    n = rows * cols
    packed = int4_gauss_groups_packed(seed, n)
    comp, offs = lz4_compress_blocks(packed, block_bytes)
    return dict(rows=rows, cols=cols, G=G, block_bytes=block_bytes, comp=comp, offs=offs,
                scales=fp16_uniform(seed, n // G, 0.001, 0.1, stream=1), zeros=u8_uniform(seed, n // G, 0, 15, stream=2))


def _header_limit() -> int:
    """LT_NOALLOC_MAX_BLOCKS as include/lt_decode.h defines it (the library's
    own limit; the binding's constant is checked against it in test_abi)."""
    text = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                             "lt_decode.h")).read()
    return int(re.search(r"#define\s+LT_NOALLOC_MAX_BLOCKS\s+(\d+)", text).group(1))


def test_noalloc_rejects_more_blocks_than_its_scratch_holds():
    # returns before touching any device: no GPU needed. The request is one
    # block over the header's limit, whatever that limit is, so the call can
    # never get past the check and launch on the placeholder pointers.
    lib = L.load_library()
    P = 0x1000  # never dereferenced
    limit = _header_limit()
    rows, cols = (limit + 1) * 16, 8192  # 16 rows of 8192 codes = one 64 KB block
    st = lib.lt_lz4_int4_decode_noalloc(P, 16, P, 65536, P, None, rows, cols, 128, P, None, None)
    assert st == L.LT_ERR_UNSUPPORTED
    # with smaller blocks the same code count is more blocks: still refused
    st = lib.lt_lz4_int4_decode_noalloc(P, 16, P, 32768, P, None, (limit // 2 + 1) * 16, cols, 128, P, None, None)
    assert st == L.LT_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_noalloc_matches_the_oracle_on_two_calls_in_a_row():
    torch = pytest.importorskip("torch")
    import oracle
    from tests._gpu import assert_f16_parity, dev, host_bits, need_gpu

    need_gpu()
    lib = L.load_library()
    limit = _header_limit()
    # two matrices decoded one after the other through the C ABI. The first
    # fills the scratch with the largest index it can hold (64 KB blocks);
    # the second is smaller and has 32 KB blocks, so it starts from the
    # first call's leftover entries and a different window size.
    cases = [_matrix(42, limit * 16), _matrix(41, 600, block_bytes=32768)]
    stream = torch.cuda.current_stream().cuda_stream
    for m in cases:
        n_blocks = len(m["offs"]) - 1
        assert n_blocks <= limit
        n = m["rows"] * m["cols"]
        want, st_want = oracle.lz4_int4_decode(m["comp"], m["offs"], m["block_bytes"], m["scales"], m["zeros"],
                                               m["rows"], m["cols"], m["G"])
        assert st_want == 0
        comp, offs, sc, ze = dev(m["comp"]), dev(m["offs"]), dev(m["scales"]), dev(m["zeros"])
        got = torch.full((n,), float("nan"), dtype=torch.float16, device="cuda")
        st_got = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = lib.lt_lz4_int4_decode_noalloc(comp.data_ptr(), int(m["comp"].size), offs.data_ptr(), m["block_bytes"],
                                            sc.data_ptr(), ze.data_ptr(), m["rows"], m["cols"], m["G"],
                                            got.data_ptr(), st_got.data_ptr(), stream)
        assert rc == L.LT_OK
        torch.cuda.synchronize()
        assert int(st_got.item()) == 0
        assert_f16_parity(host_bits(got), want, what=f"no-allocation entry point, {n_blocks} blocks")
